// Reference search on the 5th-generation tensor cores (ResidualKV paper summary
// page, "DeltaKV Framework Architecture": top-k nearest references by L2
// distance; "Practical Deployment via Sparse-vLLM": a batched L2 distance
// kernel for the reference search).
//
// |k - r|^2 = |k|^2 - 2 t with t = k.r - |r|^2/2, and |k|^2 is the same for all
// candidates of a position, so the nearest references are those of largest t.
// t is one GEMM: the position rows [k, 1, 1, 1, 0..] times the reference rows
// [r, -hi, -mid, -lo, 0..] where hi + mid + lo = |r|^2/2 (three bf16 terms of
// the fp32 value).  The extra 16-wide K block rides along as one more
// tcgen05.mma, so the epilogue reads t straight from TMEM.
//
// Work item: two consecutive 128-position tiles of one unit, so every
// reference tile fetched from L2 feeds two MMAs (M = 2 x 128, N = 128).  Only
// references at earlier positions are candidates: an item needs the reference
// tiles up to its last position's count, and columns past a row's own count are
// masked.
//
// Persistent kernel, one CTA per SM, warp-specialised:
//   warp 0      TMA producer (no multicast): both position tiles of an item
//               (128-byte swizzle) and a 2-stage ring of reference tiles plus their
//               augmented block (32-byte swizzle); L2 prefetch of the next item
//   warp 1      TMEM allocator and MMA issuer (one thread)
//   warps 2-17  epilogue: warps (quarter q, tile a, half h) read TMEM lanes 32q..32q+31
//               of tile a, columns 64h .. 64h+63 of every reference tile: two threads
//               per position
// Two accumulator sets (2 tiles x 128 columns each) let the MMAs of the next
// reference tile overlap the epilogue of the previous one.
//
// Top-kc per position (ties to the lower ordinal): per 32 columns a thread forms the bit
// mask of the t above its threshold (one subtraction and one funnel shift per element: the
// sign bit of threshold - t), and only the set bits are inserted, in column order, into its
// sorted list in registers (the chunk's values parked in the thread's own shared-memory
// slots so that a set bit can fetch its value).  Most chunks of a row hold no t above the
// threshold, so the per-element cost is the two instructions of the mask.
//
// Every wait is bounded; a wait that gives up records RKV_ERR_TIMEOUT, the CTA
// winds down (waiting, again bounded, for its own copies and MMAs) and frees its
// TMEM.  The pipeline waits sleep in the barrier (a suspend-time hint) instead of
// polling, so a waiting role leaves its scheduler's issue slots to the epilogue.
#include <cudaTypedefs.h>

#include <cfloat>

#include "device_common.cuh"
#include "launchers.h"
#include "sm100_ptx.cuh"

namespace rkv {

namespace {

using namespace sm100;

constexpr int kM = 128;           // positions per tile = TMEM lanes
constexpr int kTiles = 2;         // position tiles per work item
constexpr int kN = 128;           // references per stage = TMEM columns per accumulator
constexpr int kStagesB = 2;
constexpr int kAcc = 2;           // accumulator sets (each kTiles x kN columns)
constexpr int kHalves = 2;        // column halves of a reference tile (a position's two threads)
constexpr int kHalfCols = kN / kHalves;
constexpr int kEpiWarps = 4 * kTiles * kHalves;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kPairs = kEpiWarps / kHalves;   // warp pairs sharing a set of positions
constexpr int kThreads = 64 + kEpiThreads;
constexpr int kSlots = 10;        // 16-byte shared-memory slots per epilogue thread (>= 8, >= KC / 2)
constexpr uint32_t kTmemCols = kAcc * kTiles * kN;  // 512

template <int D>
struct Layout {
    static constexpr uint32_t a_tile = kM * D * 2;
    static constexpr uint32_t b_main = kN * D * 2;
    static constexpr uint32_t b_stage = b_main + kN * 32;            // + augmented block
    static constexpr uint32_t a_off = 0;
    static constexpr uint32_t b_off = a_off + kTiles * a_tile;
    static constexpr uint32_t aaug_off = b_off + kStagesB * b_stage;
    static constexpr uint32_t q_off = aaug_off + kM * 32;
    static constexpr uint32_t thr_off = q_off + kSlots * kEpiThreads * 16;   // [kHalves][kTiles * kM]
    static constexpr uint32_t bar_off = thr_off + kHalves * kTiles * kM * 4;
    static constexpr uint32_t total = bar_off + 256;
    static constexpr uint32_t alloc = total + 1024;  // slack for 1024-byte alignment
    static_assert(b_stage % 1024 == 0 && a_tile % 1024 == 0, "stage alignment");
};
static_assert(2 * kSlots >= 20, "the merge hands over up to 20 (t, ordinal) pairs");

struct Bars {
    uint64_t full_a;
    uint64_t empty_a;
    uint64_t full_b[kStagesB];
    uint64_t empty_b[kStagesB];
    uint64_t acc_full[kAcc];
    uint64_t acc_empty[kAcc];
    uint64_t done;
    uint64_t pair[kPairs];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Inserts t into the list kept in descending t.  Exact ties of t are not ordered here: the
// encoder re-ranks every candidate within its error bound of the k-th by exact distance
// and ordinal, and rescans all candidates when the kept list could be incomplete.
template <int KC>
__device__ __forceinline__ void topk_insert(float (&tv)[KC], int (&ti)[KC], float t, int j)
{
    float cv = t;
    int ci = j;
#pragma unroll
    for (int s = 0; s < KC; ++s) {
        const bool before = cv > tv[s];
        const float ft = tv[s];
        const int it = ti[s];
        tv[s] = before ? cv : ft;
        ti[s] = before ? ci : it;
        cv = before ? ft : cv;
        ci = before ? it : ci;
    }
}

// Orders entries of equal t by ascending ordinal (odd-even transposition passes).
template <int KC>
__device__ __forceinline__ void order_ties(float (&tv)[KC], int (&ti)[KC])
{
#pragma unroll
    for (int pass = 0; pass < KC; ++pass) {
#pragma unroll
        for (int s = pass & 1; s + 1 < KC; s += 2) {
            const bool sw = tv[s] == tv[s + 1] && ti[s] > ti[s + 1];
            const int x = ti[s];
            ti[s] = sw ? ti[s + 1] : x;
            ti[s + 1] = sw ? x : ti[s + 1];
        }
    }
}

// Item taken by this CTA in round r: rounds alternate direction over the
// heaviest-first list, so every CTA gets a balanced share of the work.
__device__ __forceinline__ int item_of(int r)
{
    const int g = static_cast<int>(gridDim.x);
    const int b = static_cast<int>(blockIdx.x);
    return r * g + ((r & 1) ? (g - 1 - b) : b);
}

// Candidates of the last position of an item (its causal limit).
__device__ __forceinline__ int item_candidates(const CacheArgs& a, const UnitMeta& um, int p0)
{
    const int p_last = min(p0 + kTiles * kM, um.n) - 1;
    return min(refs_upto(a.ph, p_last), um.R);
}

__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Maxima of the kHalfCols / 16 blocks of 16 columns starting at TMEM column col (this thread's
// row); columns j0 + c at or past ncand count as -inf.
__device__ __forceinline__ void half_maxima(uint32_t col, int j0, int ncand, float* mx)
{
#pragma unroll
    for (int c0 = 0; c0 < kHalfCols; c0 += 32) {
        float v[32];
        tmem_ld32(col + c0, v);
        if (j0 + c0 + 32 > ncand) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                v[i] = (j0 + c0 + i < ncand) ? v[i] : -FLT_MAX;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float* b = v + 16 * h;
            const float m0 = fmax3(b[0], b[1], b[2]), m1 = fmax3(b[3], b[4], b[5]);
            const float m2 = fmax3(b[6], b[7], b[8]), m3 = fmax3(b[9], b[10], b[11]);
            const float m4 = fmax3(b[12], b[13], b[14]);
            mx[c0 / 16 + h] = fmax3(fmax3(m0, m1, m2), fmax3(m3, m4, b[15]), -FLT_MAX);
        }
    }
}

// (m << 1) | sign bit of x: one funnel shift.
__device__ __forceinline__ uint32_t shl_sign(uint32_t m, float x)
{
    uint32_t r;
    asm("shf.l.wrap.b32 %0, %1, %2, 1;" : "=r"(r) : "r"(__float_as_uint(x)), "r"(m));
    return r;
}

// Sorts 16 values in descending order (bitonic network).
__device__ __forceinline__ void sort16_desc(float (&x)[16])
{
#pragma unroll
    for (int k = 2; k <= 16; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const float a = x[i], b = x[l];
                    const bool desc = (i & k) == 0;
                    x[i] = desc ? fmaxf(a, b) : fminf(a, b);
                    x[l] = desc ? fminf(a, b) : fmaxf(a, b);
                }
            }
}

template <int D, int KC>
__global__ void __launch_bounds__(kThreads, 1)
    select_tc_kernel(const CacheArgs a, const Tile* __restrict__ items, int n_items,
                     const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmAug, uint16_t* __restrict__ cand_idx,
                     float* __restrict__ cand_t)
{
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
    uint8_t* sA = smem + L::a_off;
    uint8_t* sB = smem + L::b_off;
    uint8_t* sAaug = smem + L::aaug_off;
    float4* sQ = reinterpret_cast<float4*>(smem + L::q_off);   // [kSlots][kEpiThreads]
    float* sThr = reinterpret_cast<float*>(smem + L::thr_off);
    Bars* bars = reinterpret_cast<Bars*>(smem + L::bar_off);
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->full_a, 1);
        mbar_init(&bars->empty_a, 1);
        for (int s = 0; s < kStagesB; ++s) {
            mbar_init(&bars->full_b[s], 1);
            mbar_init(&bars->empty_b[s], 1);
        }
        for (int s = 0; s < kAcc; ++s) {
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], kEpiThreads);
        }
        mbar_init(&bars->done, 1);
        for (int s = 0; s < kPairs; ++s)
            mbar_init(&bars->pair[s], 64);
        bars->abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmAug);
    }
    if (warp >= 2 && threadIdx.x - 64 < kM) {
        // augmented block of the position rows: [1, 1, 1, 0 ... 0] per row, 32-byte swizzle
        // (the 16-byte half that holds the ones is the physical half (row >> 2) & 1)
        const int r = threadIdx.x - 64;
        uint4* row = reinterpret_cast<uint4*>(sAaug + r * 32);
        const uint4 ones = make_uint4(0x3f803f80u, 0x00003f80u, 0u, 0u);
        const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
        const int phys = (r >> 2) & 1;
        row[phys] = ones;
        row[phys ^ 1] = zero;
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t it_b = 0, ni = 0;
            int last_a = -1;
            int last_b[kStagesB];
            for (int s = 0; s < kStagesB; ++s)
                last_b[s] = -1;
            bool ok = true;
            for (int rnd = 0, w = item_of(0); w < n_items && ok; w = item_of(++rnd)) {
                const Tile it = items[w];
                const UnitMeta um = a.units[it.unit];
                const int p0 = it.tile * kTiles * kM;
                const int nrt = (item_candidates(a, um, p0) + kN - 1) / kN;
                if (!(ok = mbar_wait_sleep(&bars->empty_a, (ni & 1) ^ 1, abort)))
                    break;
                mbar_arrive_expect_tx(&bars->full_a, kTiles * L::a_tile);
                const int row0 = it.unit * a.max_len + p0;
#pragma unroll
                for (int t = 0; t < kTiles; ++t)
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb)
                        tma_load_2d(sA + t * L::a_tile + kb * (kM * 128), &tmA, kb * 64, row0 + t * kM,
                                    &bars->full_a);
                last_a = static_cast<int>(ni);
                ++ni;
                if (item_of(rnd + 1) < n_items) {
                    const Tile nx = items[item_of(rnd + 1)];
                    const int nrow = nx.unit * a.max_len + nx.tile * kTiles * kM;
#pragma unroll
                    for (int t = 0; t < kTiles; ++t)
#pragma unroll
                        for (int kb = 0; kb < D / 64; ++kb)
                            prefetch_tile_2d(&tmA, kb * 64, nrow + t * kM);
                }
                for (int r = 0; r < nrt; ++r) {
                    const int sb = it_b % kStagesB;
                    if (!(ok = mbar_wait_sleep(&bars->empty_b[sb], ((it_b / kStagesB) & 1) ^ 1, abort)))
                        break;
                    mbar_arrive_expect_tx(&bars->full_b[sb], L::b_stage);
                    const int rrow = static_cast<int>(um.ref_row) + r * kN;
                    uint8_t* dst = sB + sb * L::b_stage;
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb)
                        tma_load_2d(dst + kb * (kN * 128), &tmB, kb * 64, rrow, &bars->full_b[sb]);
                    tma_load_2d(dst + L::b_main, &tmAug, 0, rrow, &bars->full_b[sb]);
                    last_b[sb] = static_cast<int>(it_b / kStagesB);
                    ++it_b;
                }
            }
            if (!ok) {
                *abort = 1;
                report(a.err, RKV_ERR_TIMEOUT);
                // let the copies this thread issued land before the CTA exits
                volatile int never = 0;
                if (last_a >= 0)
                    mbar_wait(&bars->full_a, last_a & 1, &never);
                for (int s = 0; s < kStagesB; ++s)
                    if (last_b[s] >= 0)
                        mbar_wait(&bars->full_b[s], last_b[s] & 1, &never);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kM, kN);
            const uint64_t aaug_desc = smem_desc_sw32(smem_addr(sAaug));
            uint32_t it_b = 0, it_c = 0, ni = 0;
            bool ok = true;
            bool issued = false;
            for (int rnd = 0, w = item_of(0); w < n_items && ok; w = item_of(++rnd)) {
                const Tile it = items[w];
                const UnitMeta um = a.units[it.unit];
                const int nrt = (item_candidates(a, um, it.tile * kTiles * kM) + kN - 1) / kN;
                if (!(ok = mbar_wait_sleep(&bars->full_a, ni & 1, abort)))
                    break;
                tc_fence_after();
                const uint32_t a_base = smem_addr(sA);
                for (int r = 0; r < nrt; ++r) {
                    const int sb = it_b % kStagesB;
                    const int acc = it_c % kAcc;
                    if (!(ok = mbar_wait_sleep(&bars->full_b[sb], (it_b / kStagesB) & 1, abort)))
                        break;
                    if (!(ok = mbar_wait_sleep(&bars->acc_empty[acc], ((it_c / kAcc) & 1) ^ 1, abort)))
                        break;
                    tc_fence_after();
                    const uint32_t b_base = smem_addr(sB + sb * L::b_stage);
                    const uint64_t baug_desc = smem_desc_sw32(b_base + L::b_main);
#pragma unroll
                    for (int t = 0; t < kTiles; ++t) {
                        const uint32_t d_tmem = tmem_base + (acc * kTiles + t) * kN;
                        const uint32_t at = a_base + t * L::a_tile;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off_a = (kk / 4) * (kM * 128) + (kk % 4) * 32;
                            const uint32_t off_b = (kk / 4) * (kN * 128) + (kk % 4) * 32;
                            mma_f16(d_tmem, smem_desc_sw128(at + off_a), smem_desc_sw128(b_base + off_b), idesc,
                                    kk > 0 ? 1u : 0u);
                        }
                        mma_f16(d_tmem, aaug_desc, baug_desc, idesc, 1u);
                    }
                    issued = true;
                    mma_commit(&bars->empty_b[sb]);
                    mma_commit(&bars->acc_full[acc]);
                    ++it_b;
                    ++it_c;
                }
                if (!ok)
                    break;
                mma_commit(&bars->empty_a);
                ++ni;
            }
            if (!ok) {
                *abort = 1;
                report(a.err, RKV_ERR_TIMEOUT);
            }
            if (issued) {
                // every MMA of this CTA has completed before TMEM is released
                volatile int never = 0;
                mma_commit(&bars->done);
                mbar_wait(&bars->done, 0, &never);
            }
        }
    } else {
        // ---------------- epilogue: a position per pair of threads ----------------
        // Warps e and e + kPairs read the same TMEM lanes (positions) of the same tile, the first
        // columns 0 .. 63 of every reference tile, the second 64 .. 127.  Each keeps its own
        // sorted list and shared-memory slots; they share a threshold (the larger of their
        // kc-th best values is a lower bound of the position's kc-th best, so either may filter
        // with it), combine their seeds, and merge their lists at the end of the item.  Pairs
        // synchronise on an mbarrier of their own (bounded waits).
        const int e = warp - 2;                  // 0 .. kEpiWarps-1
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int pi = e % kPairs;               // pair
        const int hf = e / kPairs;               // column half
        const int t = pi >> 2;                   // position tile of the item
        const int row = q * 32 + lane;
        const int trow = t * kM + row;
        const int qi = e * 32 + lane;            // slot column of this thread
        float4* myq = sQ + qi;                                     // this thread's slots
        const float4* otherq = sQ + ((e ^ kPairs) * 32 + lane);   // the partner's slots
        volatile float* thr_own = sThr + hf * (kTiles * kM) + trow;
        volatile float* thr_oth = sThr + (hf ^ 1) * (kTiles * kM) + trow;
        const int cb = hf * kHalfCols;           // first column of this thread's half
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        uint32_t it_c = 0, pph = 0;
        bool ok = true;
        auto pair_sync = [&]() {
            mbar_arrive(&bars->pair[pi]);
            if (!mbar_wait_sleep(&bars->pair[pi], pph & 1, abort))
                ok = false;
            ++pph;
        };
        // (no early exit from the item loop: after a wait gives up every later wait returns at
        // once, and both threads of a pair still take the same synchronisations)
        for (int rnd = 0, w = item_of(0); w < n_items; w = item_of(++rnd)) {
            const Tile it = items[w];
            const UnitMeta um = a.units[it.unit];
            const int p0 = it.tile * kTiles * kM;
            const int nc_max = item_candidates(a, um, p0);
            const int nrt = (nc_max + kN - 1) / kN;
            const int p = p0 + t * kM + row;
            const bool valid = (p < um.n) && !is_ref_pos(a.ph, p);
            const int ncand = valid ? refs_upto(a.ph, p) : 0;
            float tv[KC];
            int ti[KC];
#pragma unroll
            for (int s = 0; s < KC; ++s) {
                tv[s] = -FLT_MAX;
                ti[s] = 0x7fffffff;
            }
            float seed_lo = -FLT_MAX;
            *thr_own = -FLT_MAX;
            pair_sync();   // both halves start the item with no threshold
            for (int r = 0; r < nrt; ++r) {
                const int acc = it_c % kAcc;
                // one lane waits, the warp follows: the TMEM loads below are warp-collective
                int got = 1;
                if (lane == 0)
                    got = (ok && mbar_wait_sleep(&bars->acc_full[acc], (it_c / kAcc) & 1, abort)) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, got, 0) != 0;
                tc_fence_after();
                const int j0 = r * kN + cb;
                const uint32_t col0 = lane_base + (acc * kTiles + t) * kN + cb;
                if (r == 0 && nrt >= 2 && KC <= 16) {
                    // the KC-th largest of the sixteen block maxima of the first two reference
                    // tiles (distinct elements; eight from each half) bounds the kc-th best t
                    // from below; the first tile stays in TMEM while the second is read
                    float mx[16];
                    const int acc1 = (it_c + 1) % kAcc;
                    int got1 = 1;
                    if (lane == 0)
                        got1 = (ok && mbar_wait_sleep(&bars->acc_full[acc1], ((it_c + 1) / kAcc) & 1, abort)) ? 1 : 0;
                    ok = __shfl_sync(0xffffffffu, got1, 0) != 0;
                    tc_fence_after();
                    if (ok) {
                        half_maxima(col0, j0, ncand, mx);
                        half_maxima(lane_base + (acc1 * kTiles + t) * kN + cb, j0 + kN, ncand, mx + 4);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            mx[i] = -FLT_MAX;
                    }
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        myq[i * kEpiThreads] = make_float4(mx[4 * i], mx[4 * i + 1], mx[4 * i + 2], mx[4 * i + 3]);
                    pair_sync();
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const float4 o = otherq[i * kEpiThreads];
                        mx[8 + 4 * i] = o.x;
                        mx[8 + 4 * i + 1] = o.y;
                        mx[8 + 4 * i + 2] = o.z;
                        mx[8 + 4 * i + 3] = o.w;
                    }
                    pair_sync();   // the partner has read this thread's maxima (the slots are reused)
                    sort16_desc(mx);
                    const float seed = mx[KC - 1];
                    seed_lo = (seed > -FLT_MAX) ? nextafterf(seed, -FLT_MAX) : -FLT_MAX;
                }
                for (int c0 = 0; ok && c0 < kHalfCols && j0 + c0 < nc_max; c0 += 32) {
                    float v[32];
                    tmem_ld32(col0 + c0, v);
                    // one compare per element: seed_lo is just below the seed, so the element that
                    // defines the seed still passes; the partner's kc-th best bounds this
                    // position's kc-th best as well
                    // (+0 turns a threshold of -0 into +0: the sign of thr - t is then set exactly
                    // when t > thr)
                    const float thr = __fadd_rn(fmax3(tv[KC - 1], seed_lo, *thr_oth), 0.0f);
                    uint32_t hit = 0u;   // bit 31 - k: column c0 + k is above thr
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        hit = shl_sign(hit, __fsub_rn(thr, v[k]));
                    // columns at or past this row's own candidate count are not candidates
                    const int nvalid = ncand - (j0 + c0);
                    if (nvalid < 32)
                        hit = (nvalid <= 0) ? 0u : (hit & ~(0xffffffffu >> nvalid));
                    if (hit != 0u) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            myq[i * kEpiThreads] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                        const float* mine = reinterpret_cast<const float*>(myq);
                        do {
                            const int k = __clz(hit);
                            hit ^= 0x80000000u >> k;
                            const float x = mine[(k >> 2) * (4 * kEpiThreads) + (k & 3)];
                            if (x > tv[KC - 1])
                                topk_insert<KC>(tv, ti, x, j0 + c0 + k);
                        } while (hit != 0u);
                        *thr_own = tv[KC - 1];
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars->acc_empty[acc]);
                ++it_c;
            }
            // merge: the second half hands its list over through its slots (KC <= 2 kSlots)
            if (hf == 1) {
#pragma unroll
                for (int s = 0; s < KC; s += 2)
                    myq[(s / 2) * kEpiThreads] =
                        make_float4(tv[s], __int_as_float(ti[s]), tv[s + 1], __int_as_float(ti[s + 1]));
            }
            pair_sync();
            if (hf == 0) {
#pragma unroll
                for (int s = 0; s < KC; s += 2) {
                    const float4 x = otherq[(s / 2) * kEpiThreads];
                    if (x.x > tv[KC - 1])
                        topk_insert<KC>(tv, ti, x.x, __float_as_int(x.y));
                    if (x.z > tv[KC - 1])
                        topk_insert<KC>(tv, ti, x.z, __float_as_int(x.w));
                }
                order_ties<KC>(tv, ti);
                if (valid && ok) {
                    const int64_t orow = um.cmp_row + (p - ncand);
                    const int nv = min(KC, ncand);
#pragma unroll
                    for (int s = 0; s < KC; ++s) {
                        cand_idx[orow * KC + s] = (s < nv) ? static_cast<uint16_t>(ti[s])
                                                           : static_cast<uint16_t>(RKV_IDX_UNUSED);
                        cand_t[orow * KC + s] = (s < nv) ? tv[s] : -FLT_MAX;
                    }
                }
            }
            pair_sync();   // the second half's column is free again
        }
        if (!ok) {
            *abort = 1;
            report(a.err, RKV_ERR_TIMEOUT);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn tensor_map_encoder()
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeFn>(fn);
}

// 2D bf16 tensor map over rows x cols with a (box_cols x box_rows) box.
bool make_map(EncodeFn enc, CUtensorMap* m, const void* base, int64_t rows, int cols, int box_cols, int box_rows,
              CUtensorMapSwizzle sw)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int KC>
cudaError_t launch_t(const CacheArgs& a, const Tile* items, int n_items, const CUtensorMap& mA, const CUtensorMap& mB,
                     const CUtensorMap& mAug, uint16_t* ci, float* ct, int grid, cudaStream_t st)
{
    auto kern = select_tc_kernel<D, KC>;
    const uint32_t smem = Layout<D>::alloc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    kern<<<grid, kThreads, smem, st>>>(a, items, n_items, mA, mB, mAug, ci, ct);
    return cudaGetLastError();
}

}  // namespace

bool select_tc_supported(const CacheArgs& a) { return a.in_dtype == RKV_DTYPE_BF16 && (a.D == 128 || a.D == 64); }

cudaError_t launch_select_tc(const CacheArgs& a, const Tile* items, int n_items, const void* K, const uint16_t* refB,
                             int64_t in_rows, int64_t ref_rows, uint16_t* cand_idx, float* cand_t, cudaStream_t st)
{
    if (n_items <= 0)
        return cudaSuccess;
    EncodeFn enc = tensor_map_encoder();
    if (!enc)
        return cudaErrorNotSupported;
    alignas(64) CUtensorMap mA;
    alignas(64) CUtensorMap mB;
    alignas(64) CUtensorMap mAug;
    if (!make_map(enc, &mA, K, in_rows, a.D, 64, kM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(enc, &mB, refB, ref_rows, a.D, 64, kN, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(enc, &mAug, a.ref_aug, ref_rows, 16, 16, kN, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const int grid = n_items < sms ? n_items : sms;
    if (a.D == 128) {
        switch (a.kc) {
        case 8: return launch_t<128, 8>(a, items, n_items, mA, mB, mAug, cand_idx, cand_t, grid, st);
        case 12: return launch_t<128, 12>(a, items, n_items, mA, mB, mAug, cand_idx, cand_t, grid, st);
        default: return launch_t<128, 20>(a, items, n_items, mA, mB, mAug, cand_idx, cand_t, grid, st);
        }
    }
    switch (a.kc) {
    case 8: return launch_t<64, 8>(a, items, n_items, mA, mB, mAug, cand_idx, cand_t, grid, st);
    case 12: return launch_t<64, 12>(a, items, n_items, mA, mB, mAug, cand_idx, cand_t, grid, st);
    default: return launch_t<64, 20>(a, items, n_items, mA, mB, mAug, cand_idx, cand_t, grid, st);
    }
}

}  // namespace rkv
