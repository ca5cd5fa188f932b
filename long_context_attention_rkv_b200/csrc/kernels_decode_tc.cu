// Compressed tokens of a decode step on the 5th-generation tensor cores (ResidualKV paper
// summary page, "Practical Deployment via Sparse-vLLM": reconstruction fused into attention;
// news page, "How ResidualKV Works": tokens rebuilt on the fly when attention needs them).
//
// The factorised algebra of the scores and refs kernels (kernels_decode_mma.cu) is kept; this
// kernel does the per-token part, with one thread per compressed token:
//   logit_i = cK * sum_g sK_ig (q . codeK_i)_g + mean_{j in S(i)} s_j,   p_i = 2^(logit_i - m)
//   O      += sum_i p_i sum_g sV_ig codeV_i|g,   W_j += p_i / k_eff (j in S(i)),   L += p_i
// Persistent, one CTA per SM over a contiguous range of 128-token tiles.  Warps:
//   0     TMA producer: a tile's int4 codes (K and V, 64-byte swizzle), scales and ordinals
//         into a 3-stage ring;
//   1     TMEM allocator and the K-side MMA issuer (one thread);
//   2-13  three teams of four token warps taking the tiles in turn; thread = token = TMEM lane;
//   14    the V-side MMA issuer (one thread).
// Per tile a team
//   1. turns its tokens' codes into bf16 (136 + v, exact: the bf16 bit pattern of 128 + the
//      offset nibble): the K codes straight into TMEM (tcgen05.st, one lane per token), where
//      they are the A operand of the K-side product, then, once its previous tile's V-side
//      MMAs have completed (at Gp 8 the team waits for them before the K codes), the V codes
//      into shared memory as the MN-major A operand of the V side;
//   2. the MMA thread forms D_K[token][(head, group)] = codes x qblock, M 128, N 4 Gp, K 128,
//      with qblock the query split by scale group (block-diagonal, bf16, exact);
//   3. each thread turns its D_K row into the logits, p, the reference weights (vector
//      reductions to global memory) and the V-side B operand p * sV as a hi + lo bf16 pair
//      (about 16 significant bits), written as its token's row of an MN-major shared-memory
//      tile;
//   4. the MMA thread accumulates D_V[channel][(head, group) hi | lo] += codes^T x B, M 128,
//      N 8 Gp, K 128 tokens, over all the tiles of a unit.
// The channel order inside the MMAs follows the nibble order of the code words (pairs of
// nibbles i and i + 4 make one bf16 pair, one mask-xor each); the query block and the output
// use the same order.  The K side keeps the offset 136 in its operand and takes it off with
// the query's group sums (one 128-term product per tile).  The V side accumulates over all of
// a unit's tiles (up to a million tokens), so its operand holds the exact codes v (one packed
// bf16 subtraction of 136 per pair): the accumulator then carries sums of the size of the
// result instead of 136 times the softmax mass, whose rounding the final subtraction of the
// offset would have exposed.  At the end of a unit's tiles team 0 reads D_V and adds the
// unit's partial output and softmax sum to global memory.
// Every mbarrier wait is bounded (2 s); a wait that gives up records RKV_ERR_TIMEOUT, the roles
// go on through the CTA's barriers without work, and the MMAs and copies in flight are waited
// for before TMEM is freed.
#include <cudaTypedefs.h>

#include <cfloat>

#include "decode_mma.h"
#include "device_common.cuh"
#include "launchers.h"
#include "sm100_ptx.cuh"

namespace rkv {

namespace {

using namespace sm100;
using namespace decode_detail;

constexpr int kD = 128;
constexpr int kT = 128;                        // tokens per tile (TMEM lanes, MMA M of the K side)
constexpr int kTeams = 3;
constexpr int kTokWarps = 4 * kTeams;
constexpr int kVWarp = 2 + kTokWarps;           // the V-side MMA issuer
constexpr int kThreads = 96 + 32 * kTokWarps;  // producer, two MMA issuers, token warps
constexpr int kSyncThreads = 64 + 32 * kTokWarps;   // the issuers and the token warps (named barrier 1)
constexpr int kCodeRow = 64;                   // bytes of one int4 code row
constexpr int kNst = 3;                        // ring stages
constexpr int kStageBytes = 2 * kT * kCodeRow + 2 * kT * 8 + kT * 8 * 2;   // codes, scales, ordinals (k <= 8)
constexpr uint32_t kNibMask = 0x000F000Fu;
constexpr uint32_t kNibMagic = 0x43084308u;
constexpr float kCodeOffset = 136.0f;
constexpr uint32_t kTmemCols = 512;

template <int Gp>
struct TcLayout {
    static constexpr int NK = 4 * Gp;          // K side: (head, group) columns
    static constexpr int NV = 2 * NK;          // V side: hi and lo halves
    static constexpr uint32_t stages = 0;
    static constexpr uint32_t vtile = stages + kNst * kStageBytes;            // per team: 32 KB
    static constexpr uint32_t bv = vtile + kTeams * 32768;                   // per team: kT * NV * 2
    static constexpr uint32_t bk = bv + kTeams * kT * NV * 2;                // NK rows x 256 B
    static constexpr uint32_t qs = bk + NK * 256;                            // q of the unit, bf16 [Gp][D]
    static constexpr uint32_t red = qs + Gp * kD * 2;                        // [kTokWarps][Gp] floats
    static constexpr uint32_t misc = red + kTokWarps * Gp * 4;              // qc[NK], m[Gp], key[Gp]
    static constexpr uint32_t bars = (misc + (NK + 2 * Gp) * 4 + 15) / 16 * 16;
    static constexpr uint32_t tab = bars + 256;                              // score table (ST)
    static constexpr uint32_t total = tab;
    static constexpr uint32_t alloc = total + 1024;
    static_assert(vtile % 1024 == 0 && bv % 1024 == 0 && bk % 1024 == 0, "operand alignment");
};

struct TcBars {
    uint64_t full[kNst];
    uint64_t empty[kNst];
    uint64_t a_ready[kTeams];
    uint64_t k_done[kTeams];
    uint64_t p_ready[kTeams];
    uint64_t v_done[kTeams];
    uint64_t dv_full;
    uint64_t done;
    uint64_t done_v;
    uint32_t tmem_base;
    int abort;
    int issued;
};
static_assert(sizeof(TcBars) <= 256, "barrier block");

// Channel of MMA slot m (0 .. 127): slot pair j = m / 2 is the bf16 pair made of nibbles i and
// i + 4 of code word j / 4 (channels 8 (j / 4) + i, + 4).  The groups of 32 channels stay
// contiguous (slots 32 g .. 32 g + 31).
__host__ __device__ __forceinline__ int slot_channel(int m)
{
    const int j = m >> 1;
    return 8 * (j >> 2) + (j & 3) + 4 * (m & 1);
}

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void named_sync(int id, int n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void red_global_v4(float* p, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory matrix descriptor with explicit leading / stride byte offsets and layout type.
__device__ __forceinline__ uint64_t smem_desc(uint32_t start, uint32_t lbo, uint32_t sbo, uint32_t layout)
{
    return static_cast<uint64_t>((start >> 4) & 0x3fff) | (static_cast<uint64_t>((lbo >> 4) & 0x3fff) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3fff) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(layout) << 61);
}

// 32 consecutive 32-bit columns of this warp's 32 TMEM lanes from registers (one lane per thread).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// N consecutive fp32 columns (16, 32 or 64) of this warp's TMEM lanes.
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N])
{
    if constexpr (N == 16) {
        tmem_ld16(taddr, v);
    } else if constexpr (N == 32) {
        tmem_ld32(taddr, v);
    } else {
        float a[32], b[32];
        tmem_ld32(taddr, a);
        tmem_ld32(taddr + 32, b);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[i] = a[i];
            v[32 + i] = b[i];
        }
    }
}

// Byte offset of (row, 16-byte chunk) in a 64-byte-row tile written by TMA with the 64-byte swizzle.
__device__ __forceinline__ uint32_t sw64(int row, int chunk)
{
    return static_cast<uint32_t>(row * kCodeRow + ((chunk ^ ((row >> 1) & 3)) << 4));
}

// Half hf (code bytes 32 hf .. 32 hf + 31) of one token's code row (stage tile, 64-byte
// swizzle) as 32 bf16 pairs {136 + v_i, 136 + v_i+4}: pair 4 wd + i of code word wd (the
// words 8 hf .. 8 hf + 7 of the row) holds nibbles i and i + 4.
__device__ __forceinline__ void convert_half(const unsigned char* tile, int tok, int hf, uint32_t (&out)[32])
{
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(tile + sw64(tok, 2 * hf + c));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int wd = 4 * c + x;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                out[4 * wd + i] = ((w[x] >> (4 * i)) & kNibMask) ^ kNibMagic;
        }
    }
}

// The unit's first tile end, as in the tile partition (units' rows padded to whole tiles).
__device__ __forceinline__ int unit_end_tile(const CacheArgs& a, int uu)
{
    const UnitMeta m = a.units[uu];
    return static_cast<int>((m.cmp_row + ((m.C + kT - 1) / kT) * kT) / kT);
}

// The first unit from u0 on whose tiles reach past tile T (warp-wide, 32 units per round trip).
__device__ __forceinline__ int unit_after(const CacheArgs& a, int u0, int T, int lane)
{
    for (int base = u0; base < a.n_units; base += 32) {
        const bool past = base + lane < a.n_units && T < unit_end_tile(a, base + lane);
        const unsigned bal = __ballot_sync(0xffffffffu, past);
        if (bal)
            return base + __ffs(bal) - 1;
    }
    return a.n_units;
}

// ST: the units' reference-score tables are copied into shared memory (they fit), else read
// from L2.
template <int Gp, int KK, bool ST>
__global__ void __launch_bounds__(kThreads, 1)
    tokens_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const CacheArgs a, const void* __restrict__ q, const MmaWs w)
{
    using L = TcLayout<Gp>;
    constexpr int NK = L::NK, NV = L::NV;
    // K conversion of a tile before the wait for the team's previous V side (Gp 4; at Gp 8 the
    // values it keeps live across that wait spill)
    constexpr bool kEarlyK = Gp == 4;
    extern __shared__ unsigned char tc_smem_raw[];
    const uint32_t raw_addr = smem_addr(tc_smem_raw);
    unsigned char* sm = tc_smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
    TcBars* bars = reinterpret_cast<TcBars*>(sm + L::bars);
    volatile int* abort = &bars->abort;
    uint16_t* q_sm = reinterpret_cast<uint16_t*>(sm + L::qs);
    float* red = reinterpret_cast<float*>(sm + L::red);
    float* qc_sm = reinterpret_cast<float*>(sm + L::misc);
    float* m_sm = qc_sm + NK;
    uint32_t* key_sm = reinterpret_cast<uint32_t*>(m_sm + Gp);
    const float* tab_sm = reinterpret_cast<const float*>(sm + L::tab);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = gridDim.x, b = blockIdx.x;
    const int t_lo = static_cast<int>(static_cast<int64_t>(w.n_tiles) * b / nb);
    const int t_hi = static_cast<int>(static_cast<int64_t>(w.n_tiles) * (b + 1) / nb);
    const int n_local = t_hi - t_lo;
    if (n_local <= 0)
        return;
    const uint32_t idx_bytes = static_cast<uint32_t>(kT * a.k * 2);
    const uint32_t tx = 2 * kT * kCodeRow + 2 * kT * 8 + idx_bytes;

    if (tid == 0) {
        for (int s = 0; s < kNst; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 128);
        }
        for (int t = 0; t < kTeams; ++t) {
            mbar_init(&bars->a_ready[t], 128);
            mbar_init(&bars->k_done[t], 1);
            mbar_init(&bars->p_ready[t], 128);
            mbar_init(&bars->v_done[t], 1);
        }
        mbar_init(&bars->dv_full, 1);
        mbar_init(&bars->done, 1);
        mbar_init(&bars->done_v, 1);
        bars->abort = 0;
        bars->issued = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t tm_ak = tmem;                         // team t: columns 64 t .. 64 t + 63 (K-side A)
    const uint32_t tm_dk = tmem + 64 * kTeams;           // team t: 32 columns from 64 kTeams + 32 t (K-side D)
    const uint32_t tm_dv = tmem + 96 * kTeams;           // V-side D (NV <= 64 columns)

    if (warp == 0) {
        // ---------------- TMA producer (runs ahead of the scores kernel: codes do not depend on it)
        if (lane == 0) {
            int last = -1;
            for (int j = 0; j < n_local; ++j) {
                const int s = j % kNst;
                if (j >= kNst && !mbar_wait_sleep(&bars->empty[s], ((j / kNst) - 1) & 1, abort)) {
                    if (!*abort)
                        report(a.err, RKV_ERR_TIMEOUT);
                    *abort = 1;
                    break;
                }
                unsigned char* st = sm + L::stages + s * kStageBytes;
                const int64_t row0 = static_cast<int64_t>(t_lo + j) * kT;
                mbar_arrive_expect_tx(&bars->full[s], tx);
                tma_load_2d(st, &tmK, 0, static_cast<int>(row0), &bars->full[s]);
                tma_load_2d(st + kT * kCodeRow, &tmV, 0, static_cast<int>(row0), &bars->full[s]);
                bulk_load(st + 2 * kT * kCodeRow, a.scale_K + row0 * 4, kT * 8, &bars->full[s]);
                bulk_load(st + 2 * kT * kCodeRow + kT * 8, a.scale_V + row0 * 4, kT * 8, &bars->full[s]);
                bulk_load(st + 2 * kT * kCodeRow + 2 * kT * 8, a.idx + row0 * a.k, idx_bytes, &bars->full[s]);
                last = j;
            }
            bars->issued = last + 1;
        }
        grid_dep_wait();
        grid_dep_launch();
    } else if (warp == 1 || warp == kVWarp) {
        // ---------------- MMA issuers: warp 1 the K side, warp kVWarp the V side.  Each sleeps on
        // the barrier of the next tile it serves, so the token warps keep their issue slots.
        // A tile's K side precedes its V side (the team writes its B operand only after it has
        // read D_K), and a team converts its next tile only after its previous V side has
        // completed (v_done); the V sides go in tile order, the first of a unit clearing D_V.
        grid_dep_wait();
        grid_dep_launch();
        const bool kside = warp == 1;
        constexpr uint32_t idescK = idesc_bf16_f32(kT, NK);
        constexpr uint32_t idescV = idesc_bf16_f32(kT, NV) | (1u << 15) | (1u << 16);   // A and B MN-major
        bool issued_any = false;
        int t = t_lo;
        int u = unit_after(a, 0, t_lo, lane);
        while (t < t_hi && u < a.n_units) {
            const int seg_end = min(t_hi, unit_end_tile(a, u));
            named_sync(1, kSyncThreads);   // A: the previous unit is read out
            named_sync(1, kSyncThreads);   // B: this unit's query block is in shared memory
            if (lane == 0) {
                const uint32_t bkb = smem_addr(sm + L::bk);
                for (int i = t; i < seg_end && !*abort; ++i) {
                    const int li = i - t_lo, tm = li % kTeams;
                    uint64_t* bar = kside ? &bars->a_ready[tm] : &bars->p_ready[tm];
                    if (!mbar_wait_sleep(bar, (li / kTeams) & 1, abort)) {
                        if (!*abort)
                            report(a.err, RKV_ERR_TIMEOUT);
                        *abort = 1;
                        break;
                    }
                    tc_fence_after();
                    if (kside) {
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk)
                            mma_f16_ts(tm_dk + 32 * tm, tm_ak + 64 * tm + 8 * kk,
                                       smem_desc_sw128(bkb + (kk / 4) * (NK * 128) + (kk % 4) * 32), idescK,
                                       kk > 0 ? 1u : 0u);
                        mma_commit(&bars->k_done[tm]);
                    } else {
                        const uint32_t av = smem_addr(sm + L::vtile + tm * 32768);
                        const uint32_t bvb = smem_addr(sm + L::bv + tm * (kT * NV * 2));
#pragma unroll
                        for (int kk = 0; kk < kT / 16; ++kk)
                            mma_f16(tm_dv, smem_desc(av + kk * 2048, 16384, 1024, 2),
                                    smem_desc(bvb + kk * 256, 128, 2048, 0), idescV, (i > t || kk > 0) ? 1u : 0u);
                        mma_commit(&bars->v_done[tm]);
                    }
                    issued_any = true;
                }
                if (!kside && !*abort)
                    mma_commit(&bars->dv_full);
            }
            __syncwarp();
            t = seg_end;
            u = unit_after(a, u, t, lane);
        }
        if (lane == 0 && issued_any) {
            // every MMA this thread issued has completed before TMEM is released
            volatile int never = 0;
            uint64_t* done = kside ? &bars->done : &bars->done_v;
            mma_commit(done);
            mbar_wait(done, 0, &never);
        }
    } else {
        // ---------------- token warps: thread = token of the tile = TMEM lane
        const int tw = warp - 2;                 // 0 .. kTokWarps - 1
        const int tm = tw >> 2;                  // team
        const int qd = warp & 3;                 // TMEM lane quarter this warp may access
        const int tok = 32 * qd + lane;
        const int tt = tm * 128 + (tw & 3) * 32 + lane;   // 0 .. 255 among the token threads
        const uint32_t lane_off = static_cast<uint32_t>(32 * qd) << 16;
        const int G = a.G;
        grid_dep_wait();   // reference scores, unit maxima and zeroed accumulators of the scores kernel
        grid_dep_launch();
        bool overflow = false, corrupt = false;
        int t = t_lo, seg = 0;
        int u = unit_after(a, 0, t_lo, lane);
        while (t < t_hi && u < a.n_units) {
            const UnitMeta um = a.units[u];
            const int seg_end = min(t_hi, unit_end_tile(a, u));
            const int kvh = u - um.seq * a.Hkv;
            named_sync(1, kSyncThreads);   // A
            // ---- unit setup: query, query block (K-major, 128-byte swizzle), offsets
            if (tt < Gp)
                key_sm[tt] = 0u;
            for (int x = tt; x < Gp * kD; x += 32 * kTokWarps) {
                const int h = x / kD, c = x % kD;
                q_sm[x] = (h < G) ? static_cast<const uint16_t*>(q)[(static_cast<int64_t>(um.seq) * a.Hq + kvh * G + h) *
                                                                     kD + c]
                                  : static_cast<uint16_t>(0);
            }
            named_sync(2, 32 * kTokWarps);
            unit_max_fold<Gp>(w, u, um.R, tt, 32 * kTokWarps, key_sm);
            for (int x = tt; x < NK * (kD / 2); x += 32 * kTokWarps) {
                // word x: row n = x / 64 ((head, group)), slot pair j = x % 64
                const int n = x / (kD / 2), j = x % (kD / 2);
                const int h = n >> 2, g = n & 3;
                uint32_t word = 0u;
                if (h < G && (2 * j) / 32 == g)
                    word = static_cast<uint32_t>(q_sm[h * kD + slot_channel(2 * j)]) |
                           (static_cast<uint32_t>(q_sm[h * kD + slot_channel(2 * j + 1)]) << 16);
                const int m = 2 * j;   // first slot of the pair
                const uint32_t off = (m / 64) * (NK * 128) + (n / 8) * 1024 + (n % 8) * 128 +
                                     ((((m % 64) / 8) ^ (n % 8)) << 4) + (m % 8) * 2;
                *reinterpret_cast<uint32_t*>(sm + L::bk + off) = word;
            }
            if constexpr (ST) {
                // the unit's reference scores (written by the scores kernel, read through L2)
                const float4* src = reinterpret_cast<const float4*>(w.s_tab + um.ref_row * Gp);
                float4* dst = reinterpret_cast<float4*>(sm + L::tab);
                for (int x = tt; x < um.R * Gp / 4; x += 32 * kTokWarps)
                    dst[x] = __ldcg(src + x);
            }
            if (tt < NK) {
                const int h = tt >> 2, g = tt & 3;
                float sum = 0.0f;
                for (int c = 0; c < 32; ++c)
                    sum += bf16_bits_to_f32(q_sm[h * kD + 32 * g + c]);
                qc_sm[tt] = kCodeOffset * sum;
            }
            fence_proxy_async_smem();
            named_sync(2, 32 * kTokWarps);
            if (tt < Gp)
                m_sm[tt] = unit_m(key_sm, tt);
            named_sync(1, kSyncThreads);   // B
            float qc[NK], mh[Gp], lsum[Gp];
#pragma unroll
            for (int n = 0; n < NK; ++n)
                qc[n] = qc_sm[n];
#pragma unroll
            for (int h = 0; h < Gp; ++h) {
                mh[h] = m_sm[h];
                lsum[h] = 0.0f;
            }
            const float* s_tab = w.s_tab + um.ref_row * Gp;
            float* Wt = w.W + um.ref_row * Gp;
            const int R = um.R;

            // ---- this team's tiles of the unit
            for (int i = t + (tm - (t - t_lo) % kTeams + kTeams) % kTeams; i < seg_end; i += kTeams) {
                const int li = i - t_lo, s = li % kNst, use = li / kTeams;
                bool ok = !*abort;
                if (!kEarlyK && ok && use > 0 && !mbar_wait_sleep(&bars->v_done[tm], (use - 1) & 1, abort))
                    ok = false;
                if (ok && !mbar_wait_sleep(&bars->full[s], (li / kNst) & 1, abort))
                    ok = false;
                if (!ok) {
                    if (!*abort)
                        report(a.err, RKV_ERR_TIMEOUT);
                    *abort = 1;
                }
                // the TMEM stores below are warp-collective: the warp goes on (or skips) as one
                if (!__all_sync(0xffffffffu, ok))
                    continue;
                const unsigned char* st = sm + L::stages + s * kStageBytes;
                const int c_tok = static_cast<int>(static_cast<int64_t>(i) * kT - um.cmp_row) + tok;
                const bool valid = c_tok < um.C;
                // 0. the chosen references and their scores, first: the lookups (shared memory
                //    when the unit's table fits there, else L2) land while the codes convert
                const uint16_t* ix = reinterpret_cast<const uint16_t*>(st + 2 * kT * kCodeRow + 2 * kT * 8) + tok * a.k;
                int oi[KK];
                if (KK == 4 && a.k == 4) {
                    const uint2 v = *reinterpret_cast<const uint2*>(ix);
                    oi[0] = v.x & 0xffff; oi[1] = v.x >> 16; oi[KK > 2 ? 2 : 0] = v.y & 0xffff;
                    oi[KK > 3 ? 3 : 0] = v.y >> 16;
                } else if (KK == 8 && a.k == 8) {
                    const uint4 v = *reinterpret_cast<const uint4*>(ix);
                    oi[0] = v.x & 0xffff; oi[1] = v.x >> 16; oi[KK > 2 ? 2 : 0] = v.y & 0xffff;
                    oi[KK > 3 ? 3 : 0] = v.y >> 16; oi[KK > 4 ? 4 : 0] = v.z & 0xffff;
                    oi[KK > 5 ? 5 : 0] = v.z >> 16; oi[KK > 6 ? 6 : 0] = v.w & 0xffff;
                    oi[KK > 7 ? 7 : 0] = v.w >> 16;
                } else {
#pragma unroll
                    for (int j = 0; j < KK; ++j)
                        oi[j] = (j < a.k) ? static_cast<int>(ix[j]) : static_cast<int>(RKV_IDX_UNUSED);
                }
                int keff = 0;
                float4 sraw[KK][Gp / 4];
#pragma unroll
                for (int j = 0; j < KK; ++j) {
                    const bool has = valid && oi[j] != RKV_IDX_UNUSED;
                    corrupt |= has && oi[j] >= R;
                    const bool use_j = has && oi[j] < R;
                    oi[j] = use_j ? oi[j] : -1;
                    keff += use_j ? 1 : 0;
                    const int oc = use_j ? oi[j] : 0;
#pragma unroll
                    for (int h4 = 0; h4 < Gp / 4; ++h4)
                        sraw[j][h4] = ST ? reinterpret_cast<const float4*>(tab_sm + oc * Gp)[h4]
                                         : __ldg(reinterpret_cast<const float4*>(s_tab + oc * Gp) + h4);
                }
                // 1. codes -> bf16: K side into TMEM, V side into the team's MN-major tile
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t wk[32];
                    convert_half(st, tok, hf, wk);
                    tmem_st32(tm_ak + 64 * tm + 32 * hf + lane_off, wk);
                }
                // the K side can start: its A operand is in TMEM
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars->a_ready[tm]);
                // the team's previous V-side MMAs read its V tile and B operand: they complete
                // before either is rewritten (with kEarlyK the K side above overlapped them)
                if constexpr (kEarlyK) {
                    const bool vd = use == 0 || mbar_wait_sleep(&bars->v_done[tm], (use - 1) & 1, abort);
                    if (!vd) {
                        if (!*abort)
                            report(a.err, RKV_ERR_TIMEOUT);
                        *abort = 1;
                    }
                    if (!__all_sync(0xffffffffu, vd))
                        continue;
                }
                // V codes while the K-side MMAs run (made visible to the tensor cores by the fence
                // before p_ready)
                // V: pair words 32 hf .. 32 hf + 31 are MMA slots 64 hf .. 64 hf + 63, the
                // 64-slot MN block hf of the tile (eight 16-byte chunks of this token's row)
                unsigned char* vt = sm + L::vtile + tm * 32768 + (tok >> 3) * 1024 + (tok & 7) * 128;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t wv[32];
                    convert_half(st + kT * kCodeRow, tok, hf, wv);
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        // (136 + v) - 136 = v, exact in bf16
                        __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&wv[x]);
                        pr = __hsub2(pr, __floats2bfloat162_rn(kCodeOffset, kCodeOffset));
                        wv[x] = *reinterpret_cast<const uint32_t*>(&pr);
                    }
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        *reinterpret_cast<uint4*>(vt + hf * 16384 + ((cc ^ (tok & 7)) << 4)) =
                            make_uint4(wv[4 * cc], wv[4 * cc + 1], wv[4 * cc + 2], wv[4 * cc + 3]);
                }
                const uint2 skw = *reinterpret_cast<const uint2*>(st + 2 * kT * kCodeRow + tok * 8);
                const uint2 svw = *reinterpret_cast<const uint2*>(st + 2 * kT * kCodeRow + kT * 8 + tok * 8);
                mbar_arrive(&bars->empty[s]);

                // 2. the mean reference score of each head
                float sref[Gp];
#pragma unroll
                for (int h = 0; h < Gp; ++h)
                    sref[h] = 0.0f;
#pragma unroll
                for (int j = 0; j < KK; ++j) {
                    const bool use_j = oi[j] >= 0;
#pragma unroll
                    for (int h4 = 0; h4 < Gp / 4; ++h4) {
                        sref[4 * h4] += use_j ? sraw[j][h4].x : 0.0f;
                        sref[4 * h4 + 1] += use_j ? sraw[j][h4].y : 0.0f;
                        sref[4 * h4 + 2] += use_j ? sraw[j][h4].z : 0.0f;
                        sref[4 * h4 + 3] += use_j ? sraw[j][h4].w : 0.0f;
                    }
                }
                const float rk = __frcp_rn(static_cast<float>(max(keff, 1)));
                const float sk[4] = {__half2float(__ushort_as_half(static_cast<unsigned short>(skw.x & 0xffffu))),
                                     __half2float(__ushort_as_half(static_cast<unsigned short>(skw.x >> 16))),
                                     __half2float(__ushort_as_half(static_cast<unsigned short>(skw.y & 0xffffu))),
                                     __half2float(__ushort_as_half(static_cast<unsigned short>(skw.y >> 16)))};
                const float sv[4] = {__half2float(__ushort_as_half(static_cast<unsigned short>(svw.x & 0xffffu))),
                                     __half2float(__ushort_as_half(static_cast<unsigned short>(svw.x >> 16))),
                                     __half2float(__ushort_as_half(static_cast<unsigned short>(svw.y & 0xffffu))),
                                     __half2float(__ushort_as_half(static_cast<unsigned short>(svw.y >> 16)))};

                // 3. the K-side products, softmax, reference weights, V-side B operand
                const bool kd = mbar_wait_sleep(&bars->k_done[tm], use & 1, abort);
                if (!kd) {
                    if (!*abort)
                        report(a.err, RKV_ERR_TIMEOUT);
                    *abort = 1;
                }
                if (!__all_sync(0xffffffffu, kd))
                    continue;
                tc_fence_after();
                float dk[NK];
                tmem_ld<NK>(tm_dk + 32 * tm + lane_off, dk);
                float p[Gp];
#pragma unroll
                for (int h = 0; h < Gp; ++h) {
                    float acc = 0.0f;
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        acc = fmaf(sk[g], dk[4 * h + g] - qc[4 * h + g], acc);
                    const float logit = fmaf(w.cK, acc, sref[h] * rk);
                    const float ex = logit - mh[h];
                    const bool live = valid && keff > 0 && h < G;
                    overflow |= live && ex > 100.0f;
                    p[h] = live ? exp2f(fminf(ex, 100.0f)) : 0.0f;
                    lsum[h] += p[h];
                }
#pragma unroll
                for (int j = 0; j < KK; ++j) {
                    if (oi[j] >= 0) {
#pragma unroll
                        for (int h4 = 0; h4 < Gp; h4 += 4)
                            red_global_v4(Wt + oi[j] * Gp + h4, p[h4] * rk, p[h4 + 1] * rk, p[h4 + 2] * rk,
                                          p[h4 + 3] * rk);
                    }
                }
                // B operand row of this token: columns n = (head, group) hi, then NK + n lo
                uint32_t hi[NK / 2], lo[NK / 2];
#pragma unroll
                for (int n = 0; n < NK; n += 2) {
                    // p = 0 for rows past the unit's tokens, whose scales are not written: zero,
                    // not 0 * (whatever the padding holds)
                    const float v0 = p[n >> 2] != 0.0f ? p[n >> 2] * sv[n & 3] : 0.0f;
                    const float v1 = p[(n + 1) >> 2] != 0.0f ? p[(n + 1) >> 2] * sv[(n + 1) & 3] : 0.0f;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
                    const uint32_t hw = *reinterpret_cast<const uint32_t*>(&h2);
                    const float h0 = __uint_as_float(hw << 16), h1 = __uint_as_float(hw & 0xffff0000u);
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(v0 - h0, v1 - h1);
                    const uint32_t lw = *reinterpret_cast<const uint32_t*>(&l2);
                    hi[n / 2] = hw;
                    lo[n / 2] = lw;
                }
                unsigned char* bvr = sm + L::bv + tm * (kT * NV * 2) + (tok >> 3) * 128 + (tok & 7) * 16;
#pragma unroll
                for (int cb = 0; cb < NK / 8; ++cb) {
                    *reinterpret_cast<uint4*>(bvr + cb * 2048) =
                        make_uint4(hi[4 * cb], hi[4 * cb + 1], hi[4 * cb + 2], hi[4 * cb + 3]);
                    *reinterpret_cast<uint4*>(bvr + (NK / 8 + cb) * 2048) =
                        make_uint4(lo[4 * cb], lo[4 * cb + 1], lo[4 * cb + 2], lo[4 * cb + 3]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bars->p_ready[tm]);
            }

            // ---- end of the unit's tiles: softmax sums over the token threads
#pragma unroll
            for (int h = 0; h < Gp; ++h) {
                float v = lsum[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0)
                    red[tw * Gp + h] = v;
            }
            named_sync(2, 32 * kTokWarps);
            if (tm == 0) {
                // team 0 reads D_V: lane = MMA slot m = tok (channel slot_channel(m), group m / 32)
                bool got = !*abort;
                if (got && !mbar_wait_sleep(&bars->dv_full, seg & 1, abort)) {
                    if (!*abort)
                        report(a.err, RKV_ERR_TIMEOUT);
                    *abort = 1;
                    got = false;
                }
                if (__all_sync(0xffffffffu, got)) {
                    tc_fence_after();
                    float dv[NV];
                    tmem_ld<NV>(tm_dv + lane_off, dv);
                    const int m = tok, g = m >> 5, ch = slot_channel(m);
                    float* Ou = w.O + static_cast<int64_t>(u) * Gp * kD;
                    for (int h = 0; h < G; ++h) {
                        const int n = 4 * h + g;
                        float val = 0.0f;
#pragma unroll
                        for (int n2 = 0; n2 < NK; ++n2)
                            val = (n2 == n) ? dv[n2] + dv[NK + n2] : val;
                        atomicAdd(&Ou[h * kD + ch], val);
                    }
                    if (tt < G) {
                        float ls = 0.0f;
#pragma unroll
                        for (int x = 0; x < kTokWarps; ++x)
                            ls += red[x * Gp + tt];
                        atomicAdd(&w.L[u * Gp + tt], ls);
                    }
                }
                tc_fence_before();
            }
            t = seg_end;
            u = unit_after(a, u, t, lane);
            ++seg;
        }
        if (__any_sync(0xffffffffu, overflow) && lane == 0)
            report(a.err, RKV_ERR_UNSUPPORTED);
        if (__any_sync(0xffffffffu, corrupt) && lane == 0)
            report(a.err, RKV_ERR_CORRUPT);
    }

    // the copies of the last stages land before the CTA may exit (only after an abort can one
    // still be in flight here)
    __syncthreads();
    if (tid == 0) {
        volatile int never = 0;
        const int n = bars->issued;
        for (int j = (n > kNst ? n - kNst : 0); j < n; ++j)
            mbar_wait(&bars->full[j % kNst], (j / kNst) & 1, &never);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn map_encoder()
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeFn>(fn);
}

// Byte-typed 2D map over the int4 code rows (64 bytes each), 128-row boxes, 64-byte swizzle.
bool codes_map(EncodeFn enc, CUtensorMap* m, const void* base, int64_t rows)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kCodeRow), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kCodeRow)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kCodeRow), static_cast<cuuint32_t>(kT)};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shared memory the score table may take next to the rest of the layout.
constexpr uint32_t kSmemOptin = 232448;

template <int Gp, int KK, bool ST>
cudaError_t launch_t(const CUtensorMap& mK, const CUtensorMap& mV, const CacheArgs& a, const void* q, const MmaWs& w,
                     cudaStream_t st)
{
    auto kern = tokens_tc_kernel<Gp, KK, ST>;
    const uint32_t smem = TcLayout<Gp>::alloc + (ST ? static_cast<uint32_t>(a.max_refs) * Gp * 4 : 0u);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(w.n_cta);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mK, mV, a, q, w);
}

template <int Gp, int KK>
cudaError_t launch_st(const CUtensorMap& mK, const CUtensorMap& mV, const CacheArgs& a, const void* q,
                      const MmaWs& w, cudaStream_t st)
{
    const bool fits = TcLayout<Gp>::alloc + static_cast<uint64_t>(a.max_refs) * Gp * 4 <= kSmemOptin;
    return fits ? launch_t<Gp, KK, true>(mK, mV, a, q, w, st) : launch_t<Gp, KK, false>(mK, mV, a, q, w, st);
}

}  // namespace

cudaError_t launch_tokens_tc(const CacheArgs& a, const MmaWs& w, const void* q, int Gp, cudaStream_t st)
{
    if (w.n_tiles <= 0)
        return cudaSuccess;
    EncodeFn enc = map_encoder();
    if (!enc)
        return cudaErrorNotSupported;
    alignas(64) CUtensorMap mK;
    alignas(64) CUtensorMap mV;
    const int64_t rows = static_cast<int64_t>(w.n_tiles) * kT;
    if (!codes_map(enc, &mK, a.codes_K, rows) || !codes_map(enc, &mV, a.codes_V, rows))
        return cudaErrorInvalidValue;
    if (Gp == 4)
        return a.k <= 4 ? launch_st<4, 4>(mK, mV, a, q, w, st) : launch_st<4, 8>(mK, mV, a, q, w, st);
    return a.k <= 4 ? launch_st<8, 4>(mK, mV, a, q, w, st) : launch_st<8, 8>(mK, mV, a, q, w, st);
}

}  // namespace rkv
