// C ABI of librkv: argument validation, cache layout and binding, kernel dispatch.
// Every entry point returns an rkv_status and never throws; see include/rkv.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "launchers.h"
#include "rkv.h"
#include "rkv_internal.h"

using namespace rkv;

namespace {

// An NVTX range around one entry point, so a profile of the whole path splits by API call.
// Costs a few nanoseconds when no profiler is attached.
struct ApiRange {
    explicit ApiRange(const char* name) { nvtxRangePushA(name); }
    ~ApiRange() { nvtxRangePop(); }
    ApiRange(const ApiRange&) = delete;
    ApiRange& operator=(const ApiRange&) = delete;
};

uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---- reference schedule on the host ----------------------------------------------------

rkv_status make_phases(const rkv_config& c, int64_t max_len, Phases& ph)
{
    std::memset(&ph, 0, sizeof(ph));
    auto magic = [&](int i) {
        div_magic(ph.stride[i], ph.m_stride[i], ph.sh_stride[i]);
        div_magic(ph.stride[i] - 1, ph.m_per[i], ph.sh_per[i]);
    };
    if (c.refs_per_phase <= 0) {
        ph.n = 1;
        ph.stride[0] = c.stride0;
        magic(0);
        return RKV_OK;
    }
    int64_t start = 0, stride = c.stride0, ord = 0;
    int n = 0;
    do {
        if (n >= kMaxPhases || stride > INT32_MAX / 2 || start > INT32_MAX)
            return RKV_ERR_UNSUPPORTED;
        ph.start[n] = static_cast<int32_t>(start);
        ph.stride[n] = static_cast<int32_t>(stride);
        ph.first_ord[n] = static_cast<int32_t>(ord);
        ph.first_slot[n] = static_cast<int32_t>(start - ord);
        magic(n);
        ++n;
        start += static_cast<int64_t>(c.refs_per_phase) * stride;
        ord += c.refs_per_phase;
        stride *= 2;
    } while (start < max_len);
    ph.n = n;
    return RKV_OK;
}

// references at positions <= p
int64_t host_refs_upto(const Phases& ph, int64_t p)
{
    int q = 0;
    for (int i = 1; i < ph.n; ++i)
        if (p >= ph.start[i])
            q = i;
    return ph.first_ord[q] + (p - ph.start[q]) / ph.stride[q] + 1;
}

int64_t host_ref_count(const Phases& ph, int64_t n) { return n <= 0 ? 0 : host_refs_upto(ph, n - 1); }

// ---- validation ---------------------------------------------------------------------

rkv_status validate_config(const rkv_config* c)
{
    if (!c)
        return RKV_ERR_INVALID_ARG;
    if (c->n_kv_heads <= 0 || c->n_q_heads <= 0 || c->n_q_heads % c->n_kv_heads != 0 || c->batch <= 0 ||
        c->max_len < 0 || c->k <= 0 || c->stride0 < 2 || c->refs_per_phase < 0 || c->group <= 0)
        return RKV_ERR_INVALID_ARG;
    if (c->in_dtype != RKV_DTYPE_BF16 && c->in_dtype != RKV_DTYPE_F32)
        return RKV_ERR_INVALID_ARG;
    if (c->out_dtype != RKV_DTYPE_BF16 && c->out_dtype != RKV_DTYPE_F32)
        return RKV_ERR_INVALID_ARG;
    if (c->bits != 4 && c->bits != 8)
        return RKV_ERR_UNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128)
        return RKV_ERR_UNSUPPORTED;
    if (c->group != 32 || c->k > RKV_MAX_K || c->batch > RKV_MAX_BATCH)
        return RKV_ERR_UNSUPPORTED;
    if (c->n_q_heads / c->n_kv_heads > 16)
        return RKV_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(c->batch) * c->n_kv_heads > 65535)
        return RKV_ERR_UNSUPPORTED;
    if (c->ref_bits != 0 && c->ref_bits != 16 && c->ref_bits != 4)
        return RKV_ERR_UNSUPPORTED;
    if (c->coder != 0 && c->coder != 1)
        return RKV_ERR_UNSUPPORTED;
    if (c->coder == 1 && (c->head_dim != 128 || c->bits != 4 || c->in_dtype != RKV_DTYPE_BF16 || c->ref_bits == 4 ||
                          c->n_q_heads / c->n_kv_heads > 8 || c->k > 8))
        return RKV_ERR_UNSUPPORTED;
    return RKV_OK;
}

// Splits of the gather decode over a position list: about 32 positions per CTA (8 per warp;
// each position is a chain of dependent gathers), within the workspace reserved for them.
int sparse_splits_max(int n_units) { return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(256, 65536 / n_units))); }

int sparse_splits(int n_units, int max_sel)
{
    return static_cast<int>(std::min<int64_t>(sparse_splits_max(n_units), std::max<int64_t>(1, ceil_div(max_sel, 32))));
}

int decode_splits(int n_units, int max_tokens)
{
    int s = static_cast<int>(ceil_div(4 * 148, n_units));
    s = std::max(1, std::min(s, 64));
    s = std::min<int64_t>(s, std::max<int64_t>(1, ceil_div(max_tokens, 256)));
    return s;
}

CacheArgs make_args(const Desc& d);

rkv_status compute_layout(const rkv_config* c, const int32_t* lengths, Desc& d)
{
    rkv_status st = validate_config(c);
    if (st != RKV_OK)
        return st;
    if (!lengths)
        return RKV_ERR_INVALID_ARG;
    std::memset(&d, 0, sizeof(d));
    d.magic = kDescMagic;
    d.cfg = *c;
    int max_n = 0;
    for (int b = 0; b < c->batch; ++b) {
        if (lengths[b] < 0 || lengths[b] > c->max_len)
            return RKV_ERR_INVALID_ARG;
        max_n = std::max(max_n, lengths[b]);
    }
    st = make_phases(*c, std::max(1, max_n), d.ph);
    if (st != RKV_OK)
        return st;
    const int D = c->head_dim, Hkv = c->n_kv_heads, G = c->n_q_heads / c->n_kv_heads;
    d.kc = search_width(c->k);
    d.code_bytes = D * c->bits / 8;
    d.n_groups = D / c->group;
    d.n_units = c->batch * Hkv;
    d.max_n = max_n;
    int64_t ref_rows = 0, cmp_rows = 0, tiles = 0, pairs = 0;
    for (int b = 0; b < c->batch; ++b) {
        const int64_t n = lengths[b];
        const int64_t R = host_ref_count(d.ph, n);
        if (R > RKV_MAX_REFS)
            return RKV_ERR_UNSUPPORTED;
        d.len[b] = static_cast<int32_t>(n);
        d.cur_len[b] = static_cast<int32_t>(n);
        d.R[b] = static_cast<int32_t>(R);
        d.C[b] = static_cast<int32_t>(n - R);
        d.Rpad[b] = static_cast<int32_t>(align_up(R, kRefPad));
        d.Cpad[b] = static_cast<int32_t>(align_up(n - R, kCmpPad));
        d.ref_seq_row[b] = ref_rows;
        d.cmp_seq_row[b] = cmp_rows;
        ref_rows += static_cast<int64_t>(Hkv) * d.Rpad[b];
        cmp_rows += static_cast<int64_t>(Hkv) * d.Cpad[b];
        tiles += static_cast<int64_t>(Hkv) * ceil_div(n, kPosTile);
        pairs += static_cast<int64_t>(Hkv) * ceil_div(n, 2 * kPosTile);
        d.max_R = std::max<int32_t>(d.max_R, d.R[b]);
        d.max_C = std::max<int32_t>(d.max_C, d.C[b]);
    }
    if (tiles > INT32_MAX)
        return RKV_ERR_UNSUPPORTED;
    d.total_ref_rows = ref_rows;
    d.total_cmp_rows = cmp_rows;
    d.n_tiles = static_cast<int32_t>(tiles);
    d.n_pairs = static_cast<int32_t>(pairs);
    uint64_t off = 0;
    auto take = [&](uint64_t bytes) {
        const uint64_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    Sections& s = d.sec;
    s.err = take(256);
    s.units = take(sizeof(UnitMeta) * d.n_units);
    s.tiles = take(sizeof(Tile) * std::max<int64_t>(1, tiles));
    s.pairs = take(sizeof(Tile) * std::max<int64_t>(1, pairs));
    const bool r4 = c->ref_bits == 4;
    s.ref_K = take(r4 ? ref_rows * D / 2 : 2ull * ref_rows * D);
    s.ref_V = take(r4 ? ref_rows * D / 2 : 2ull * ref_rows * D);
    s.ref_sK = take(r4 ? 2ull * ref_rows * (D / 32) : 0);
    s.ref_sV = take(r4 ? 2ull * ref_rows * (D / 32) : 0);
    s.ref_hn = take(4ull * (ref_rows + 256));  // tail slack: tile scans read up to 32 entries past a unit
    s.ref_aug = take(32ull * ref_rows);
    s.ref_pos = take(4ull * ref_rows);
    s.codes_K = take(static_cast<uint64_t>(cmp_rows) * d.code_bytes);
    s.codes_V = take(static_cast<uint64_t>(cmp_rows) * d.code_bytes);
    s.scale_K = take(2ull * cmp_rows * d.n_groups);
    s.scale_V = take(2ull * cmp_rows * d.n_groups);
    s.idx = take(2ull * cmp_rows * c->k);
    s.append = take(append_scratch_bytes(d.n_units));   // per-unit candidate lists of rkv_append
    s.hn_max = take(4ull * d.n_units);
    s.end = off;
    d.ws_select = align_up(2ull * cmp_rows * d.kc, 256) + align_up(4ull * cmp_rows * d.kc, 256);
    if (r4)
        d.ws_select += align_up(2ull * ref_rows * D, 256);   // the stored keys as bf16 rows (search operand)
    d.ws_fix_off = d.ws_select;                                // the encoder's deferred-token list
    d.ws_select += align_up(8ull + 8ull * cmp_rows, 256);
    d.ws_latent_off = d.ws_select;                             // the learned coder's exact-pass list
    if (c->coder == 1)
        d.ws_select += align_up(encode_latent_list_bytes(cmp_rows), 256);
    const int splits = std::max(decode_splits(d.n_units, max_n), sparse_splits_max(d.n_units));
    d.ws_decode = align_up(4ull * d.n_units * splits * G * (D + 2), 256);
    const CacheArgs a = make_args(d);
    if (decode_mma_supported(a))
        d.ws_decode = std::max<uint64_t>(d.ws_decode, decode_mma_ws_bytes(a, d.total_ref_rows));
    return RKV_OK;
}

const Desc* get_desc(const rkv_cache_desc* h)
{
    if (!h)
        return nullptr;
    const Desc* d = reinterpret_cast<const Desc*>(h->opaque);
    return d->magic == kDescMagic ? d : nullptr;
}

CacheArgs make_args(const Desc& d)
{
    CacheArgs a;
    std::memset(&a, 0, sizeof(a));
    const rkv_config& c = d.cfg;
    a.D = c.head_dim;
    a.Hkv = c.n_kv_heads;
    a.Hq = c.n_q_heads;
    a.G = c.n_q_heads / c.n_kv_heads;
    a.k = c.k;
    a.bits = c.bits;
    a.group = c.group;
    a.in_dtype = c.in_dtype;
    a.out_dtype = c.out_dtype;
    a.n_units = d.n_units;
    a.code_bytes = d.code_bytes;
    a.n_groups = d.n_groups;
    a.kc = d.kc;
    a.max_len = c.max_len;
    a.max_refs = d.max_R;
    a.ph = d.ph;
    char* base = static_cast<char*>(d.base);
    a.err = reinterpret_cast<int32_t*>(base + d.sec.err);
    a.units = reinterpret_cast<const UnitMeta*>(base + d.sec.units);
    a.ref_K = reinterpret_cast<uint16_t*>(base + d.sec.ref_K);
    a.ref_V = reinterpret_cast<uint16_t*>(base + d.sec.ref_V);
    a.ref_bits = (d.cfg.ref_bits == 4) ? 4 : 16;
    a.coder = d.cfg.coder;
    for (int i = 0; i < 8; ++i)
        a.cw[i] = d.coder_w[i];
    a.ref_sK = (a.ref_bits == 4) ? reinterpret_cast<uint16_t*>(base + d.sec.ref_sK) : nullptr;
    a.ref_sV = (a.ref_bits == 4) ? reinterpret_cast<uint16_t*>(base + d.sec.ref_sV) : nullptr;
    a.ref_hn = reinterpret_cast<float*>(base + d.sec.ref_hn);
    a.ref_hn_max = reinterpret_cast<float*>(base + d.sec.hn_max);
    a.ref_aug = reinterpret_cast<uint16_t*>(base + d.sec.ref_aug);
    a.ref_pos = reinterpret_cast<int32_t*>(base + d.sec.ref_pos);
    a.codes_K = reinterpret_cast<uint8_t*>(base + d.sec.codes_K);
    a.codes_V = reinterpret_cast<uint8_t*>(base + d.sec.codes_V);
    a.scale_K = reinterpret_cast<uint16_t*>(base + d.sec.scale_K);
    a.scale_V = reinterpret_cast<uint16_t*>(base + d.sec.scale_V);
    a.idx = reinterpret_cast<uint16_t*>(base + d.sec.idx);
    return a;
}

// A failed CUDA call becomes RKV_ERR_CUDA; with RKV_DEBUG set in the environment its
// CUDA error string is also printed to stderr.
rkv_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess)
        return RKV_OK;
    static const bool verbose = std::getenv("RKV_DEBUG") != nullptr;
    if (verbose)
        std::fprintf(stderr, "librkv: CUDA error %d: %s\n", static_cast<int>(e), cudaGetErrorString(e));
    return RKV_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" {

int32_t rkv_abi_version(void) { return RKV_ABI_VERSION; }

const char* rkv_status_string(rkv_status s)
{
    switch (s) {
    case RKV_OK: return "ok";
    case RKV_ERR_INVALID_ARG: return "invalid argument";
    case RKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case RKV_ERR_WORKSPACE: return "buffer too small";
    case RKV_ERR_CUDA: return "CUDA error";
    case RKV_ERR_CORRUPT: return "corrupted cache contents";
    case RKV_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

rkv_status rkv_schedule(const rkv_config* cfg, int32_t n, int32_t* pos, int64_t cap, int32_t* n_ref)
{
    rkv_status st = validate_config(cfg);
    if (st != RKV_OK)
        return st;
    if (n < 0 || !n_ref)
        return RKV_ERR_INVALID_ARG;
    Phases ph;
    st = make_phases(*cfg, std::max(1, n), ph);
    if (st != RKV_OK)
        return st;
    const int64_t R = host_ref_count(ph, n);
    *n_ref = static_cast<int32_t>(R);
    if (pos) {
        int64_t w = 0;
        for (int q = 0; q < ph.n && w < std::min<int64_t>(cap, R); ++q) {
            const int64_t cnt = (q + 1 < ph.n) ? (ph.first_ord[q + 1] - ph.first_ord[q]) : R - ph.first_ord[q];
            for (int64_t m = 0; m < cnt && w < std::min<int64_t>(cap, R); ++m)
                pos[w++] = static_cast<int32_t>(ph.start[q] + m * ph.stride[q]);
        }
    }
    return RKV_OK;
}

rkv_status rkv_cache_size(const rkv_config* cfg, const int32_t* lengths, uint64_t* cache_bytes,
                          uint64_t* workspace_bytes)
{
    if (!cache_bytes || !workspace_bytes)
        return RKV_ERR_INVALID_ARG;
    Desc* d = new (std::nothrow) Desc;
    if (!d)
        return RKV_ERR_INVALID_ARG;
    const rkv_status st = compute_layout(cfg, lengths, *d);
    if (st == RKV_OK) {
        *cache_bytes = d->sec.end;
        *workspace_bytes = std::max(d->ws_select, d->ws_decode);
    }
    delete d;
    return st;
}

rkv_status rkv_cache_bind(const rkv_config* cfg, const int32_t* lengths, void* dev_buf, uint64_t bytes,
                          rkv_cache_desc* desc)
{
    if (!desc || !dev_buf || !aligned(dev_buf, 256))
        return RKV_ERR_INVALID_ARG;
    Desc* d = reinterpret_cast<Desc*>(desc->opaque);
    std::memset(desc, 0, sizeof(*desc));
    rkv_status st = compute_layout(cfg, lengths, *d);
    if (st != RKV_OK) {
        std::memset(desc, 0, sizeof(*desc));
        return st;
    }
    if (bytes < d->sec.end) {
        std::memset(desc, 0, sizeof(*desc));
        return RKV_ERR_WORKSPACE;
    }
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        std::memset(desc, 0, sizeof(*desc));
        return RKV_ERR_CUDA;
    }
    if (major != 10 || minor != 0) {
        std::memset(desc, 0, sizeof(*desc));
        return RKV_ERR_UNSUPPORTED;
    }
    d->base = dev_buf;
    d->bytes = bytes;
    // unit table and the selection tiles, heaviest first
    const int Hkv = cfg->n_kv_heads;
    std::vector<UnitMeta> units(d->n_units);
    std::vector<std::pair<int64_t, Tile>> work;
    work.reserve(d->n_tiles);
    for (int b = 0; b < cfg->batch; ++b)
        for (int h = 0; h < Hkv; ++h) {
            const int u = b * Hkv + h;
            UnitMeta& m = units[u];
            m.n = d->len[b];
            m.R = d->R[b];
            m.C = d->C[b];
            m.seq = b;
            m.ref_row = d->ref_seq_row[b] + static_cast<int64_t>(h) * d->Rpad[b];
            m.cmp_row = d->cmp_seq_row[b] + static_cast<int64_t>(h) * d->Cpad[b];
            const int nt = static_cast<int>(ceil_div(m.n, kPosTile));
            for (int t = 0; t < nt; ++t) {
                const int64_t last = std::min<int64_t>(static_cast<int64_t>(t + 1) * kPosTile, m.n) - 1;
                work.push_back({host_refs_upto(d->ph, last), Tile{u, t}});
            }
        }
    auto heavier = [](const std::pair<int64_t, Tile>& x, const std::pair<int64_t, Tile>& y) { return x.first > y.first; };
    std::stable_sort(work.begin(), work.end(), heavier);
    std::vector<Tile> tiles(work.size());
    for (size_t i = 0; i < work.size(); ++i)
        tiles[i] = work[i].second;
    std::vector<std::pair<int64_t, Tile>> pwork;
    pwork.reserve(d->n_pairs);
    for (int u = 0; u < d->n_units; ++u) {
        const int np = static_cast<int>(ceil_div(units[u].n, 2 * kPosTile));
        for (int t = 0; t < np; ++t) {
            const int64_t last = std::min<int64_t>(static_cast<int64_t>(t + 1) * 2 * kPosTile, units[u].n) - 1;
            pwork.push_back({host_refs_upto(d->ph, last), Tile{u, t}});
        }
    }
    std::stable_sort(pwork.begin(), pwork.end(), heavier);
    std::vector<Tile> pairs(pwork.size());
    for (size_t i = 0; i < pwork.size(); ++i)
        pairs[i] = pwork[i].second;
    char* base = static_cast<char*>(dev_buf);
    cudaError_t e = cudaMemset(base + d->sec.err, 0, 256);
    if (e == cudaSuccess)
        e = cudaMemcpy(base + d->sec.units, units.data(), sizeof(UnitMeta) * units.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !tiles.empty())
        e = cudaMemcpy(base + d->sec.tiles, tiles.data(), sizeof(Tile) * tiles.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !pairs.empty())
        e = cudaMemcpy(base + d->sec.pairs, pairs.data(), sizeof(Tile) * pairs.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        std::memset(desc, 0, sizeof(*desc));
        return RKV_ERR_CUDA;
    }
    return RKV_OK;
}

rkv_status rkv_unit_view_get(const rkv_cache_desc* desc, int32_t seq, int32_t kv_head, rkv_unit_view* out)
{
    const Desc* d = get_desc(desc);
    if (!d || !out || seq < 0 || seq >= d->cfg.batch || kv_head < 0 || kv_head >= d->cfg.n_kv_heads)
        return RKV_ERR_INVALID_ARG;
    const CacheArgs a = make_args(*d);
    const int64_t ref_row = d->ref_seq_row[seq] + static_cast<int64_t>(kv_head) * d->Rpad[seq];
    const int64_t cmp_row = d->cmp_seq_row[seq] + static_cast<int64_t>(kv_head) * d->Cpad[seq];
    std::memset(out, 0, sizeof(*out));
    const int64_t ncur = d->cur_len[seq];
    const int64_t rcur = host_ref_count(d->ph, ncur);
    out->n = static_cast<int32_t>(ncur);
    out->n_ref = static_cast<int32_t>(rcur);
    out->n_cmp = static_cast<int32_t>(ncur - rcur);
    out->k = d->cfg.k;
    out->code_bytes = d->code_bytes;
    out->n_groups = d->n_groups;
    out->ref_bits = a.ref_bits;
    if (a.ref_bits == 4) {
        out->ref_K = reinterpret_cast<uint8_t*>(a.ref_K) + ref_row * (a.D / 2);
        out->ref_V = reinterpret_cast<uint8_t*>(a.ref_V) + ref_row * (a.D / 2);
        out->ref_scale_K = a.ref_sK + ref_row * (a.D / 32);
        out->ref_scale_V = a.ref_sV + ref_row * (a.D / 32);
    } else {
        out->ref_K = a.ref_K + ref_row * a.D;
        out->ref_V = a.ref_V + ref_row * a.D;
    }
    out->ref_half_norm = a.ref_hn + ref_row;
    out->ref_pos = a.ref_pos + ref_row;
    out->codes_K = a.codes_K + cmp_row * d->code_bytes;
    out->codes_V = a.codes_V + cmp_row * d->code_bytes;
    out->scale_K = a.scale_K + cmp_row * d->n_groups;
    out->scale_V = a.scale_V + cmp_row * d->n_groups;
    out->idx = a.idx + cmp_row * d->cfg.k;
    return RKV_OK;
}

rkv_status rkv_build_refs(const rkv_cache_desc* desc, const void* K, const void* V, void* stream)
{
    const ApiRange range("rkv_build_refs");
    const Desc* d = get_desc(desc);
    if (!d || !K || !V || !aligned(K, 16) || !aligned(V, 16))
        return RKV_ERR_INVALID_ARG;
    const CacheArgs a = make_args(*d);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the units' largest reference half norms are maxima over this call's rows
    const cudaError_t e = cudaMemsetAsync(a.ref_hn_max, 0, 4ull * d->n_units, st);
    if (e != cudaSuccess)
        return RKV_ERR_CUDA;
    return cuda_status(launch_refs_copy(a, d->max_R, K, V, st));
}

static rkv_status check_stage_args(const Desc* d, const void* K, const void* V, const void* workspace,
                                   uint64_t workspace_bytes)
{
    if (!d || !K || !aligned(K, 16) || (V && !aligned(V, 16)) || (!workspace && d->ws_select > 0) ||
        !aligned(workspace, 256))
        return RKV_ERR_INVALID_ARG;
    if (workspace_bytes < d->ws_select)
        return RKV_ERR_WORKSPACE;
    return RKV_OK;
}

static uint16_t* cand_idx_of(const Desc* d, void* ws) { return static_cast<uint16_t*>(ws); }

static float* cand_t_of(const Desc* d, void* ws)
{
    return reinterpret_cast<float*>(static_cast<char*>(ws) + align_up(2ull * d->total_cmp_rows * d->kc, 256));
}

// A learned-coder cache needs its weights bound before compression, decode or reconstruction.
static bool coder_ready(const Desc* d) { return d->cfg.coder == 0 || d->coder_w[0] != nullptr; }

rkv_status rkv_search(const rkv_cache_desc* desc, const void* K, void* workspace, uint64_t workspace_bytes,
                      void* stream)
{
    const ApiRange range("rkv_search");
    const Desc* d = get_desc(desc);
    const rkv_status s = check_stage_args(d, K, nullptr, workspace, workspace_bytes);
    if (s != RKV_OK)
        return s;
    const CacheArgs a = make_args(*d);
    const Tile* tiles = reinterpret_cast<const Tile*>(static_cast<char*>(d->base) + d->sec.tiles);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (select_tc_supported(a) && !(d->cfg.flags & RKV_FLAG_SELECT_SIMT)) {
        const int64_t in_rows = static_cast<int64_t>(d->n_units) * d->cfg.max_len;
        const Tile* pairs = reinterpret_cast<const Tile*>(static_cast<char*>(d->base) + d->sec.pairs);
        const uint16_t* refB = a.ref_K;
        if (a.ref_bits == 4) {
            // bf16 copy of the stored keys, after the candidate lists in the workspace
            uint16_t* copy = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) +
                                                         align_up(2ull * d->total_cmp_rows * d->kc, 256) +
                                                         align_up(4ull * d->total_cmp_rows * d->kc, 256));
            const cudaError_t e = launch_refs_bf16(a, d->total_ref_rows, copy, st);
            if (e != cudaSuccess)
                return cuda_status(e);
            refB = copy;
        }
        return cuda_status(launch_select_tc(a, pairs, d->n_pairs, K, refB, in_rows, d->total_ref_rows,
                                            cand_idx_of(d, workspace), cand_t_of(d, workspace), st));
    }
    return cuda_status(launch_select_simt(a, tiles, d->n_tiles, K, cand_idx_of(d, workspace),
                                          cand_t_of(d, workspace), st));
}

rkv_status rkv_encode(const rkv_cache_desc* desc, const void* K, const void* V, void* workspace,
                      uint64_t workspace_bytes, void* stream)
{
    const ApiRange range("rkv_encode");
    const Desc* d = get_desc(desc);
    if (!V)
        return RKV_ERR_INVALID_ARG;
    const rkv_status s = check_stage_args(d, K, V, workspace, workspace_bytes);
    if (s != RKV_OK)
        return s;
    if (!coder_ready(d))
        return RKV_ERR_INVALID_ARG;
    const CacheArgs a = make_args(*d);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* fix = reinterpret_cast<int*>(static_cast<char*>(workspace) + d->ws_fix_off);
    cudaError_t e = launch_encode(a, d->max_C, K, V, cand_idx_of(d, workspace), cand_t_of(d, workspace), fix,
                                  static_cast<int>(d->total_cmp_rows), st);
    if (e == cudaSuccess && a.coder == 1) {
        // the latent residuals replace the codes
        int total = 0;
        for (int b = 0; b < d->cfg.batch; ++b) {
            const int n = d->cur_len[b];
            total += d->cfg.n_kv_heads * encode_latent_tiles(n - static_cast<int>(host_ref_count(d->ph, n)));
        }
        e = launch_encode_latent(a, K, V, total,
                                 reinterpret_cast<int*>(static_cast<char*>(workspace) + d->ws_latent_off), st);
    }
    return cuda_status(e);
}

rkv_status rkv_compress(const rkv_cache_desc* desc, const void* K, const void* V, void* workspace,
                        uint64_t workspace_bytes, void* stream)
{
    const ApiRange range("rkv_compress");
    if (!V)
        return RKV_ERR_INVALID_ARG;
    const rkv_status s = rkv_search(desc, K, workspace, workspace_bytes, stream);
    return s != RKV_OK ? s : rkv_encode(desc, K, V, workspace, workspace_bytes, stream);
}

rkv_status rkv_decode_attn(const rkv_cache_desc* desc, const void* q, void* out, void* workspace,
                           uint64_t workspace_bytes, void* stream)
{
    const ApiRange range("rkv_decode_attn");
    const Desc* d = get_desc(desc);
    if (!d || !q || !out || !workspace || !aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256))
        return RKV_ERR_INVALID_ARG;
    if (workspace_bytes < d->ws_decode)
        return RKV_ERR_WORKSPACE;
    if (!coder_ready(d))
        return RKV_ERR_INVALID_ARG;
    const CacheArgs a = make_args(*d);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (a.coder == 1 && ((d->cfg.flags & (RKV_FLAG_DECODE_DIRECT | RKV_FLAG_DECODE_SIMT)) || !decode_mma_supported(a)))
        return RKV_ERR_UNSUPPORTED;   // fd is folded into the tensor-core decode only
    if (!(d->cfg.flags & (RKV_FLAG_DECODE_DIRECT | RKV_FLAG_DECODE_SIMT)) && decode_mma_supported(a) &&
        workspace_bytes >= decode_mma_ws_bytes(a, d->total_ref_rows))
        return cuda_status(launch_decode_mma(a, d->total_ref_rows, d->total_cmp_rows, q, out, workspace, st));
    if (decode_fact_supported(a) && !(d->cfg.flags & RKV_FLAG_DECODE_DIRECT)) {
        int dev = 0, sms = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = launch_decode_fact(a, decode_fact_cluster(a, sms), q, out, st);
        return cuda_status(e);
    }
    const int splits = decode_splits(d->n_units, d->max_n);
    float* part = static_cast<float*>(workspace);
    cudaError_t e = launch_decode_direct(a, splits, q, part, st);
    if (e == cudaSuccess)
        e = launch_decode_combine(a, d->cfg.batch, splits, part, out, st);
    return cuda_status(e);
}

rkv_status rkv_set_coder(rkv_cache_desc* desc, const void* const* w)
{
    const Desc* cd = get_desc(desc);
    if (!cd || !w || cd->cfg.coder != 1)
        return RKV_ERR_INVALID_ARG;
    for (int i = 0; i < 8; ++i)
        if (!w[i] || !aligned(w[i], 16))
            return RKV_ERR_INVALID_ARG;
    Desc* d = const_cast<Desc*>(cd);
    for (int i = 0; i < 8; ++i)
        d->coder_w[i] = static_cast<const uint16_t*>(w[i]);
    return RKV_OK;
}

rkv_status rkv_cache_set_lengths(rkv_cache_desc* desc, const int32_t* lengths, void* stream)
{
    const ApiRange range("rkv_cache_set_lengths");
    const Desc* cd = get_desc(desc);
    if (!cd || !lengths)
        return RKV_ERR_INVALID_ARG;
    Desc* d = const_cast<Desc*>(cd);
    for (int b = 0; b < d->cfg.batch; ++b)
        if (lengths[b] < 0 || lengths[b] > d->len[b])
            return RKV_ERR_INVALID_ARG;
    const int Hkv = d->cfg.n_kv_heads;
    std::vector<UnitMeta> units(d->n_units);
    for (int b = 0; b < d->cfg.batch; ++b)
        for (int h = 0; h < Hkv; ++h) {
            UnitMeta& m = units[b * Hkv + h];
            m.n = lengths[b];
            m.R = static_cast<int32_t>(host_ref_count(d->ph, lengths[b]));
            m.C = m.n - m.R;
            m.seq = b;
            m.ref_row = d->ref_seq_row[b] + static_cast<int64_t>(h) * d->Rpad[b];
            m.cmp_row = d->cmp_seq_row[b] + static_cast<int64_t>(h) * d->Cpad[b];
        }
    // pageable source: the copy has read it when the call returns
    const cudaError_t e = cudaMemcpyAsync(static_cast<char*>(d->base) + d->sec.units, units.data(),
                                          sizeof(UnitMeta) * units.size(), cudaMemcpyHostToDevice,
                                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return RKV_ERR_CUDA;
    for (int b = 0; b < d->cfg.batch; ++b)
        d->cur_len[b] = lengths[b];
    return RKV_OK;
}

rkv_status rkv_append(rkv_cache_desc* desc, const void* K_new, const void* V_new, const uint8_t* active,
                      void* stream)
{
    const ApiRange range("rkv_append");
    const Desc* cd = get_desc(desc);
    if (!cd || !K_new || !V_new || !aligned(K_new, 16) || !aligned(V_new, 16))
        return RKV_ERR_INVALID_ARG;
    Desc* d = const_cast<Desc*>(cd);
    if (d->cfg.coder != 0)
        return RKV_ERR_UNSUPPORTED;
    uint32_t bits[8] = {};
    bool any = false;
    for (int b = 0; b < d->cfg.batch; ++b) {
        if (active && !active[b])
            continue;
        if (d->cur_len[b] >= d->len[b])
            return RKV_ERR_INVALID_ARG;            // capacity reached: nothing is launched
        bits[b >> 5] |= 1u << (b & 31);
        any = true;
    }
    if (!any)
        return RKV_OK;
    const CacheArgs a = make_args(*d);
    const cudaError_t e = launch_append(a, K_new, V_new, bits, static_cast<char*>(d->base) + d->sec.append,
                                        static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return RKV_ERR_CUDA;
    for (int b = 0; b < d->cfg.batch; ++b)
        if (bits[b >> 5] >> (b & 31) & 1u)
            ++d->cur_len[b];
    return RKV_OK;
}

rkv_status rkv_decode_attn_sparse(const rkv_cache_desc* desc, const void* q, const int32_t* positions,
                                  const int32_t* counts, int32_t max_sel, void* out, void* workspace,
                                  uint64_t workspace_bytes, void* stream)
{
    const ApiRange range("rkv_decode_attn_sparse");
    const Desc* d = get_desc(desc);
    if (!d || !q || !out || !positions || !counts || max_sel < 1 || !workspace || !aligned(q, 16) ||
        !aligned(out, 16) || !aligned(workspace, 256) || !aligned(positions, 4) || !aligned(counts, 4))
        return RKV_ERR_INVALID_ARG;
    if (workspace_bytes < d->ws_decode)
        return RKV_ERR_WORKSPACE;
    if (d->cfg.coder != 0)
        return RKV_ERR_UNSUPPORTED;
    const CacheArgs a = make_args(*d);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int splits = sparse_splits(d->n_units, std::min<int>(max_sel, std::max(1, d->max_n)));
    float* part = static_cast<float*>(workspace);
    cudaError_t e = launch_decode_direct(a, splits, q, part, st, positions, counts, max_sel);
    if (e == cudaSuccess)
        e = launch_decode_combine(a, d->cfg.batch, splits, part, out, st);
    return cuda_status(e);
}

rkv_status rkv_reconstruct(const rkv_cache_desc* desc, int32_t seq, int32_t kv_head, const int32_t* positions,
                           int64_t n_pos, void* K_out, void* V_out, int32_t out_dtype, void* stream)
{
    const ApiRange range("rkv_reconstruct");
    const Desc* d = get_desc(desc);
    if (!d || seq < 0 || seq >= d->cfg.batch || kv_head < 0 || kv_head >= d->cfg.n_kv_heads || n_pos < 0)
        return RKV_ERR_INVALID_ARG;
    if (out_dtype != RKV_DTYPE_BF16 && out_dtype != RKV_DTYPE_F32)
        return RKV_ERR_INVALID_ARG;
    if (!positions && n_pos != d->cur_len[seq])
        return RKV_ERR_INVALID_ARG;
    if ((K_out && !aligned(K_out, 16)) || (V_out && !aligned(V_out, 16)) || (positions && !aligned(positions, 4)))
        return RKV_ERR_INVALID_ARG;
    if (n_pos == 0)
        return RKV_OK;
    if (!K_out && !V_out)
        return RKV_ERR_INVALID_ARG;
    if (!coder_ready(d))
        return RKV_ERR_INVALID_ARG;
    const CacheArgs a = make_args(*d);
    return cuda_status(launch_reconstruct(a, seq * d->cfg.n_kv_heads + kv_head, positions, n_pos, K_out, V_out,
                                          out_dtype, static_cast<cudaStream_t>(stream)));
}

rkv_status rkv_selftest_wait_timeout(int32_t* err_dev, void* stream)
{
    if (!err_dev || !aligned(err_dev, 4))
        return RKV_ERR_INVALID_ARG;
    return cuda_status(launch_wait_timeout_selftest(err_dev, static_cast<cudaStream_t>(stream)));
}

rkv_status rkv_read_device_error(const rkv_cache_desc* desc, void* stream, int32_t* device_status)
{
    const ApiRange range("rkv_read_device_error");
    const Desc* d = get_desc(desc);
    if (!d || !device_status)
        return RKV_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return RKV_ERR_CUDA;
    int32_t* err = reinterpret_cast<int32_t*>(static_cast<char*>(d->base) + d->sec.err);
    int32_t v = 0;
    if (cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
        return RKV_ERR_CUDA;
    if (v != 0 && cudaMemset(err, 0, sizeof(int32_t)) != cudaSuccess)
        return RKV_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess)
        return RKV_ERR_CUDA;
    *device_status = v;
    return RKV_OK;
}

// ---- compress without a workspace ------------------------------------------------------
// For callers that cannot allocate (see rkv_compress_noalloc in rkv.h): the candidate lists
// live in this file-scope device array.  Host code only ever uses its device address, looked
// up with cudaGetSymbolAddress once per CUDA context, with that context current.

}  // extern "C"

static __device__ __align__(256) unsigned char g_noalloc_scratch[RKV_NOALLOC_SCRATCH_BYTES];

namespace {

// The array's address belongs to a loaded module, and a module belongs to one CUDA context:
// after cudaDeviceReset, or with another context current on the same device, the array may
// sit elsewhere.  So the cached address is keyed by the current context's unique id (never
// reused within a process, unlike a context handle), not by the device ordinal, and it is
// looked up again whenever a context without an entry is current.
constexpr int kMaxContexts = 64;
struct ScratchAddr {
    unsigned long long ctx_id;
    void* ptr;
};
ScratchAddr g_noalloc_addr[kMaxContexts];
int g_noalloc_count = 0;
int g_noalloc_next = 0;
std::mutex g_noalloc_mutex;

// The two driver calls, resolved through the runtime (the library does not link the driver).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name)
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(fn);
}

rkv_status current_context_id(unsigned long long* id)
{
    static const CtxGetCurrentFn cuCtxGetCurrent = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn cuCtxGetId = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!cuCtxGetCurrent || !cuCtxGetId)
        return RKV_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (cuCtxGetCurrent(&ctx) != CUDA_SUCCESS)
        return RKV_ERR_CUDA;
    if (!ctx) {
        // no context on this thread yet: a runtime call that needs one makes the current
        // device's primary context current (it neither allocates nor launches)
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess)
            return RKV_ERR_CUDA;
        void* probe = nullptr;
        if (cudaGetSymbolAddress(&probe, g_noalloc_scratch) != cudaSuccess)
            return RKV_ERR_CUDA;
        if (cuCtxGetCurrent(&ctx) != CUDA_SUCCESS || !ctx)
            return RKV_ERR_CUDA;
    }
    return cuCtxGetId(ctx, id) == CUDA_SUCCESS ? RKV_OK : RKV_ERR_CUDA;
}

// Device address of the scratch array in the current context (looked up on first use).
rkv_status noalloc_scratch(void** out)
{
    unsigned long long id = 0;
    const rkv_status st = current_context_id(&id);
    if (st != RKV_OK)
        return st;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    for (int i = 0; i < g_noalloc_count; ++i)
        if (g_noalloc_addr[i].ctx_id == id) {
            *out = g_noalloc_addr[i].ptr;
            return RKV_OK;
        }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
        return RKV_ERR_CUDA;
    // a full table replaces its entries in turn (a context without an entry just looks up again)
    const int slot = g_noalloc_count < kMaxContexts ? g_noalloc_count++ : g_noalloc_next++ % kMaxContexts;
    g_noalloc_addr[slot] = ScratchAddr{id, p};
    *out = p;
    return RKV_OK;
}

}  // namespace

extern "C" {

rkv_status rkv_compress_noalloc(const rkv_cache_desc* desc, const void* K, const void* V, void* stream)
{
    const ApiRange range("rkv_compress_noalloc");
    const Desc* d = get_desc(desc);
    if (!d || !V)
        return RKV_ERR_INVALID_ARG;
    if (d->ws_select > RKV_NOALLOC_SCRATCH_BYTES)
        return RKV_ERR_WORKSPACE;
    void* scratch = nullptr;
    const rkv_status st = noalloc_scratch(&scratch);
    if (st != RKV_OK)
        return st;
    return rkv_compress(desc, K, V, scratch, RKV_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
