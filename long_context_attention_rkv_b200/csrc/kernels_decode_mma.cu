// Decode attention over the compressed cache with the two per-token contractions on
// the tensor cores (ResidualKV paper summary page, "Practical Deployment via
// Sparse-vLLM": reconstruction fused into attention; news page, "How ResidualKV
// Works": tokens rebuilt on the fly when attention needs them).
//
// The algebra is the factorised one (reference scores s_j = q.refK_j, reference
// weights w_j = sum of p_i / k_eff over the tokens that chose j):
//   logit_i = mean_{j in S(i)} s_j + sum_g sK_ig * (q . codeK_i)_g
//   out     = (sum_i p_i sum_g sV_ig codeV_i|g + sum_j (p_j + w_j) refV_j) / (sum_i p_i + sum_j p_j)
// with every p taken against one common offset m = max_j s_j per (unit, q-head), so
// partial sums from any number of CTAs add without rescaling.
//
// Per query step a G-head group does 2 * G * D multiply-adds per token against 152
// bytes of codes, scales and ordinals (int4, D = 128, k = 4): at G >= 4 that is more
// arithmetic per byte than the CUDA cores deliver per byte of HBM bandwidth, so the
// per-token dot products run as bf16 MMAs and the CUDA cores only unpack codes and
// run the softmax.  Three kernels, chained with programmatic dependent launch:
//   1. scores:  s_j for every reference (fp32, log2 units) and per-64-reference maxima;
//               zeroes the weight and output accumulators;
//   2. tokens:  persistent, one CTA per SM over a contiguous range of 128-token tiles.
//               Each tile is streamed into a shared-memory ring (codes by TMA with the
//               64-byte swizzle, scales and ordinals by bulk copies); the last of the
//               eight warps to finish a stage refills it, so no warp is spent on loads
//               (two warps per scheduler keep the register file at up to 255 a thread);
//               each warp takes 16 tokens of a tile:
//                 K side  D[tok][(head, group)] = codes (int4 -> bf16, exact) x q, one
//                         m16n8k16 MMA per 16 channels, the group scale applied after;
//                 softmax p = 2^(logit - m), reference weights by shared atomics;
//                 V side  D[channel][(head, group)] = codes^T x (p * sV), the group
//                         scale folded into the B operand (a hi + lo pair of bf16);
//               reference weights go to global memory with vector reductions as they
//               are produced, partial outputs and sums at the end of each unit;
//   3. refs:    sum_j (p_j + w_j) refV_j per 64-reference chunk; the last chunk of a
//               unit to finish normalises and writes the output.
// Codes enter the MMAs as 136 + v (v the signed code; the bf16 bit pattern of 128 + n
// for a nibble n): the constant 136 is taken off afterwards with exact row/column sums.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cfloat>
#include <cmath>

#include "decode_mma.h"
#include "device_common.cuh"
#include "launchers.h"
#include "sm100_ptx.cuh"

namespace rkv {

namespace {

using namespace sm100;
using namespace decode_detail;

constexpr int kTok = 128;            // tokens per pipeline stage (= compressed-row padding)
constexpr int kWarpTok = 16;         // tokens per consumer warp and stage
constexpr int kConsWarps = kTok / kWarpTok;
constexpr int kCodeRow = 64;         // bytes of one int4 code row at D = 128
constexpr uint32_t kNibMask = 0x000F000Fu;
constexpr uint32_t kNibMagic = 0x43084308u;   // bf16 128.0 in each half, sign bit of the nibble flipped
constexpr float kCodeOffset = 136.0f;         // (128 + (v + 8)) - v

// Stage layout (bytes): codes K | codes V (64-byte swizzle, 1024-aligned) | scales K | scales V | ordinals
constexpr int kStCodes = kTok * kCodeRow;                 // 8192
constexpr int kStScale = kTok * 4 * 2;                    // 4 groups x fp16
constexpr int kStIdxMax = kTok * 8 * 2;                   // k <= 8 ordinals x u16
constexpr int kStageBytes = 2 * kStCodes + 2 * kStScale + kStIdxMax;   // 20480

// ---- small PTX wrappers ------------------------------------------------------------------

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// One-dimensional bulk copy global -> shared, completion counted on bar (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two nibbles (bits 0-3 and 16-19 of w) to a bf16 pair {136 + v_lo, 136 + v_hi}.
__device__ __forceinline__ uint32_t nib2(uint32_t w) { return (w & kNibMask) ^ kNibMagic; }

// A pair of fp32 values as two bf16 pairs, hi = bf16(x) and lo = bf16(x - hi), so that
// hi + lo carries about 16 significant bits; sum accumulates the four values exactly as
// the MMAs will see them.
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo, float& sum)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - h0, x1 - h1);
    lo = *reinterpret_cast<const uint32_t*>(&l);
    sum += (h0 + __uint_as_float(lo << 16)) + (h1 + __uint_as_float(lo & 0xffff0000u));
}

__device__ __forceinline__ float half_bits_to_f32(uint32_t b) { return __half2float(__ushort_as_half(static_cast<unsigned short>(b))); }

__device__ __forceinline__ void red_shared(float* p, float v)
{
    asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(smem_addr(p)), "f"(v) : "memory");
}

__device__ __forceinline__ void red_global_v4(float* p, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// Bytes offset of (row, 16-byte chunk) in a 64-byte-row tile written by TMA with the 64-byte swizzle.
__device__ __forceinline__ uint32_t sw64(int row, int chunk)
{
    return static_cast<uint32_t>(row * kCodeRow + ((chunk ^ ((row >> 1) & 3)) << 4));
}

}  // namespace

namespace {

// ==== 1. reference scores ==================================================================

template <int Gp, int RB, bool LC>
__global__ void __launch_bounds__(128) mma_scores_kernel(const CacheArgs a, const void* __restrict__ q, const MmaWs w)
{
    // s[r][h] = cK * (refK_r . q_h) as m16n8k16 MMAs: one warp per 16 references, columns are
    // the (up to 8) q-heads.  The k-slot -> channel map gives lane tq the 32 channels
    // 32 tq .. 32 tq + 31 in every k-block (k-block kb, slots 2tq, 2tq+1 -> channels
    // 32 tq + 4 kb + {0, 1}; slots 2tq+8, 2tq+9 -> + {2, 3}), so A and B fragments are
    // four 16-byte loads of a row each.
    grid_dep_launch();
    constexpr int D = 128;
    __shared__ float wmax[4][Gp];
    const int u = blockIdx.y, ch = blockIdx.x;
    const UnitMeta um = a.units[u];
    const int kvh = u - um.seq * a.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, tq = lane & 3;
    const int R = um.R;
    const int r0 = ch * kRefChunk;
    const int r1 = min(R, r0 + kRefChunk);
    const int rw = r0 + warp * 16;               // first reference of this warp
    // A rows gid and gid + 8 (zero past the unit), B column gid (zero past the group)
    // With the int4 reference store (RB 4) the stored values code * 2^e are exact bf16
    // numbers: the A fragments are built from the codes and scales.
    uint4 ar[2][4], bq[4];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int r = rw + gid + 8 * rr;
        if constexpr (RB != 4) {
            const uint4* src = reinterpret_cast<const uint4*>(a.ref_K + (um.ref_row + r) * D + 32 * tq);
#pragma unroll
            for (int x = 0; x < 4; ++x)
                ar[rr][x] = (r < r1) ? src[x] : make_uint4(0u, 0u, 0u, 0u);
        } else {
            uint32_t hw[16];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    v[i] = 0.0f;
                if (r < r1)
                    load_ref<16, 4>(a, 0, um.ref_row + r, 32 * tq + 16 * half, v);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    hw[8 * half + i] = f32_to_bf16_bits(v[2 * i]) | (uint32_t(f32_to_bf16_bits(v[2 * i + 1])) << 16);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
                ar[rr][x] = make_uint4(hw[4 * x], hw[4 * x + 1], hw[4 * x + 2], hw[4 * x + 3]);
        }
    }
    {
        const uint4* src = reinterpret_cast<const uint4*>(
            static_cast<const uint16_t*>(q) + (static_cast<int64_t>(um.seq) * a.Hq + kvh * a.G + gid) * D + 32 * tq);
#pragma unroll
        for (int x = 0; x < 4; ++x)
            bq[x] = (gid < a.G) ? src[x] : make_uint4(0u, 0u, 0u, 0u);
    }
    if (ch == 0) {
        for (int i = tid; i < Gp * D; i += 128)
            w.O[static_cast<int64_t>(u) * Gp * D + i] = 0.0f;
        if (tid < Gp)
            w.L[u * Gp + tid] = 0.0f;
        if (tid == 0)
            w.cnt[u] = 0u;
        if (LC) {
            // learned-coder shapes: the compressed tokens' codes are latent, so they meet
            // q' = Wd_K^T q (fd folded into the query); the latent output sums start at zero
            for (int i = tid; i < Gp * D; i += 128)
                w.Olat[static_cast<int64_t>(u) * Gp * D + i] = 0.0f;
            // thread l: q'[g][l] = sum_c Wd_K[c][l] q[g][c]; Wd_K (32 KB) staged in shared
            // memory with 16-byte loads first
            __shared__ float qs[8][D];
            __shared__ __align__(16) uint16_t wds[LC ? D * D : 8];
            const uint16_t* Wd = a.cw[3];
            const uint16_t* qb = static_cast<const uint16_t*>(q) + (static_cast<int64_t>(um.seq) * a.Hq + kvh * a.G) * D;
            uint16_t* qo = w.qlat + (static_cast<int64_t>(um.seq) * a.Hq + kvh * a.G) * D;
            if constexpr (LC) {
#pragma unroll 4
                for (int i = tid; i < D * D / 8; i += 128)
                    reinterpret_cast<uint4*>(wds)[i] = reinterpret_cast<const uint4*>(Wd)[i];
            }
            for (int i = tid; i < 8 * D; i += 128)
                qs[i / D][i % D] = (i < a.G * D) ? bf16_bits_to_f32(qb[i]) : 0.0f;
            __syncthreads();
            float acc[8];
#pragma unroll
            for (int g = 0; g < 8; ++g)
                acc[g] = 0.0f;
#pragma unroll 8
            for (int c = 0; c < D; ++c) {
                const float wv = bf16_bits_to_f32(wds[LC ? c * D + tid : 0]);
#pragma unroll
                for (int g = 0; g < 8; ++g)
                    acc[g] = fmaf(wv, qs[g][c], acc[g]);
            }
            for (int g = 0; g < a.G; ++g)
                qo[g * D + tid] = f32_to_bf16_bits(acc[g]);
        }
    }
    for (int i = tid; i < (r1 - r0) * Gp; i += 128)
        w.W[(um.ref_row + r0) * Gp + i] = 0.0f;
    float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    auto word = [](const uint4 (&v)[4], int i) {
        const uint4 x = v[i >> 2];
        return (i & 3) == 0 ? x.x : (i & 3) == 1 ? x.y : (i & 3) == 2 ? x.z : x.w;
    };
#pragma unroll
    for (int kb = 0; kb < 8; ++kb)
        mma_bf16(d, word(ar[0], 2 * kb), word(ar[1], 2 * kb), word(ar[0], 2 * kb + 1), word(ar[1], 2 * kb + 1),
                 word(bq, 2 * kb), word(bq, 2 * kb + 1));
    // d: rows gid / gid + 8, heads 2tq / 2tq + 1
    float mloc[2] = {-FLT_MAX, -FLT_MAX};
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int r = rw + gid + 8 * rr;
        const float s0 = d[2 * rr] * w.cK, s1 = d[2 * rr + 1] * w.cK;
        if (r < r1) {
            if (2 * tq < Gp)
                *reinterpret_cast<float2*>(w.s_tab + (um.ref_row + r) * Gp + 2 * tq) = make_float2(s0, s1);
            if (2 * tq < a.G)
                mloc[0] = fmaxf(mloc[0], s0);
            if (2 * tq + 1 < a.G)
                mloc[1] = fmaxf(mloc[1], s1);
        }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float v = mloc[e];
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        if (gid == 0 && 2 * tq + e < Gp)
            wmax[warp][2 * tq + e] = v;
    }
    __syncthreads();
    if (tid < Gp) {
        float v = -FLT_MAX;
        for (int i = 0; i < 4; ++i)
            v = fmaxf(v, wmax[i][tid]);
        w.mpart[(static_cast<int64_t>(u) * w.n_chunk + ch) * Gp + tid] = v;
    }
}

// ==== 2. compressed tokens ================================================================

// Dynamic shared memory of the tokens kernel (byte offsets from a 1024-aligned base).
struct TokLayout {
    int stages, s_sm, o_sm, p_sm, q_sm, bk_sm, bar, misc, total;
    __host__ __device__ TokLayout(int Gp, int ncons, int R_max, int nst)
    {
        auto up = [](int x) { return (x + 127) & ~127; };
        int off = 0;
        stages = off; off += nst * kStageBytes;
        s_sm = off;   off += 2 * up(R_max * Gp * 4);      // two table buffers
        o_sm = off;   off += up(ncons * Gp * 128 * 4);    // per-warp output partials
        p_sm = off;   off += up(ncons * kWarpTok * Gp * 4);
        q_sm = off;   off += up(Gp * 128 * 2);
        bk_sm = off;  off += 8 * 2 * 8 * 16;     // K-side B operand, ldmatrix layout
        bar = off;    off += 2 * 8 * 8;
        misc = off;   off += up((6 * Gp + 4) * 4);
        total = off;
    }
};

__device__ __forceinline__ void consumer_sync(int n_threads)
{
    asm volatile("bar.sync 1, %0;" ::"r"(n_threads) : "memory");
}

// GT: the units' reference-score tables are read from global memory (L2) instead of being
// copied into shared memory (units with more references than shared memory holds).
template <int Gp, int KK, int NTEAM, bool GT>
__global__ void __launch_bounds__(32 * kConsWarps * NTEAM, 1)
    mma_tokens_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const CacheArgs a, const void* __restrict__ q, const MmaWs w, const int nst)
{
    constexpr int D = 128;
    constexpr int GPS = 8 / Gp;           // scale groups sharing one set of eight MMA columns
    constexpr int NS = 4 / GPS;           // column sets
    constexpr int NH = Gp / 4;            // q-heads per thread in the softmax step
    constexpr int NCT = kConsWarps * NTEAM * 32;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const TokLayout L(Gp, kConsWarps * NTEAM, GT ? 0 : a.max_refs, nst);
    unsigned char* stages = sm + L.stages;
    float* s_buf = reinterpret_cast<float*>(sm + L.s_sm);
    const int s_stride = ((a.max_refs * Gp * 4 + 127) & ~127) / 4;
    float* o_sm = reinterpret_cast<float*>(sm + L.o_sm);
    float* p_sm = reinterpret_cast<float*>(sm + L.p_sm);
    uint16_t* q_sm = reinterpret_cast<uint16_t*>(sm + L.q_sm);
    uint16_t* bk_sm = reinterpret_cast<uint16_t*>(sm + L.bk_sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bar);
    int* done_cnt = reinterpret_cast<int*>(full + 8);        // warps finished with a stage
    uint64_t* tbar = reinterpret_cast<uint64_t*>(done_cnt + 8);   // table buffer loaded
    float* qc_sm = reinterpret_cast<float*>(sm + L.misc);    // [4 groups][Gp]
    float* l_sm = qc_sm + 4 * Gp;
    uint32_t* key_sm = reinterpret_cast<uint32_t*>(l_sm + Gp);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(key_sm + Gp);
    volatile int* zero_flag = abort_flag + 1;
    int* issued = const_cast<int*>(zero_flag + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int nb = gridDim.x, b = blockIdx.x;
    const int t_lo = static_cast<int>(static_cast<int64_t>(w.n_tiles) * b / nb);
    const int t_hi = static_cast<int>(static_cast<int64_t>(w.n_tiles) * (b + 1) / nb);
    const int n_local = t_hi - t_lo;
    const uint32_t idx_bytes = static_cast<uint32_t>(kTok * a.k * 2);
    const uint32_t tx = 2 * kStCodes + 2 * kStScale + idx_bytes;
    // loads local tile j into stage j % nst (one thread)
    auto issue = [&](int j) {
        const int s = j % nst;
        unsigned char* st = stages + s * kStageBytes;
        const int64_t row0 = static_cast<int64_t>(t_lo + j) * kTok;
        mbar_arrive_expect_tx(&full[s], tx);
        tma_load_2d(st, &tmK, 0, static_cast<int>(row0), &full[s]);
        tma_load_2d(st + kStCodes, &tmV, 0, static_cast<int>(row0), &full[s]);
        bulk_load(st + 2 * kStCodes, a.scale_K + row0 * 4, kStScale, &full[s]);
        bulk_load(st + 2 * kStCodes + kStScale, a.scale_V + row0 * 4, kStScale, &full[s]);
        bulk_load(st + 2 * kStCodes + 2 * kStScale, a.idx + row0 * a.k, idx_bytes, &full[s]);
    };

    if (tid == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            done_cnt[s] = 0;
        }
        mbar_init(&tbar[0], 1);
        mbar_init(&tbar[1], 1);
        *abort_flag = 0;
        *zero_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        *issued = n_local < nst ? n_local : nst;
    }
    __syncthreads();
    // the ring fills while the scores kernel may still run (codes do not depend on it): lane j
    // of warp 0 loads local tile j, so the first stages' copies are issued together
    if (warp == 0 && lane < min(n_local, nst))
        issue(lane);

    // ---- consumer warps -----------------------------------------------------------------
    const int team = warp / kConsWarps, wi = warp % kConsWarps;
    const int gid = lane >> 2, tq = lane & 3;
    const int G = a.G;

    // segments: the runs of this CTA's tiles that belong to one unit.  Their score tables
    // are bulk-copied into two alternating buffers, the next one while the current is used.
    auto unit_end = [&](int uu) {
        const UnitMeta m = a.units[uu];
        return static_cast<int>((m.cmp_row + ((m.C + kTok - 1) / kTok) * kTok) / kTok);
    };
    // The first unit from u0 on whose tiles reach past tile T (the units' rows are laid out in
    // order, so their end tiles do not decrease); warp-wide, 32 units per round trip.
    auto unit_after = [&](int u0, int T) {
        for (int base = u0; base < a.n_units; base += 32) {
            const bool past = base + lane < a.n_units && T < unit_end(base + lane);
            const unsigned bal = __ballot_sync(0xffffffffu, past);
            if (bal)
                return base + __ffs(bal) - 1;
        }
        return a.n_units;
    };
    int tables_issued[2] = {0, 0};             // (thread 0)
    auto load_table = [&](int buf, int uu) {   // one thread
        ++tables_issued[buf];
        const UnitMeta m = a.units[uu];
        const uint32_t bytes = static_cast<uint32_t>(m.R * Gp * 4);
        mbar_arrive_expect_tx(&tbar[buf], bytes);
        if (bytes)
            bulk_load(s_buf + buf * s_stride, w.s_tab + m.ref_row * Gp, bytes, &tbar[buf]);
    };
    // the units of the first two segments: the unit layout does not depend on the scores kernel
    int u = unit_after(0, t_lo);
    int u_second = a.n_units;
    if (t_lo < t_hi && u < a.n_units) {
        const int t1 = min(t_hi, unit_end(u));
        if (t1 < t_hi)
            u_second = unit_after(u, t1);
    }
    grid_dep_wait();   // reference scores, maxima and zeroed accumulators of the scores kernel
    // The references kernel may be scheduled once every CTA has passed this wait: the scores
    // kernel has then completed, so the references kernel may read its outputs (through L2)
    // before waiting for this one.
    grid_dep_launch();
    if (!GT && tid == 0 && t_lo < t_hi) {
        load_table(0, u);
        if (u_second < a.n_units)
            load_table(1, u_second);
    }
    bool overflow = false, corrupt = false;
    int t = t_lo, i = 0, seg = 0;
    while (t < t_hi && u < a.n_units) {
        const UnitMeta um = a.units[u];
        const int seg_end = min(t_hi, unit_end(u));
        const float* s_sm = GT ? w.s_tab + um.ref_row * Gp : s_buf + (seg & 1) * s_stride;
        const int R = um.R;
        const int kvh = u - um.seq * a.Hkv;

        // ---- unit setup: q, reference scores, common offsets ------------------------------
        consumer_sync(NCT);
        if (tid < Gp) {
            key_sm[tid] = 0u;
            l_sm[tid] = 0.0f;
        }
        for (int x = tid; x < Gp * D; x += NCT) {
            const int h = x / D, c = x % D;
            q_sm[x] = (h < G) ? static_cast<const uint16_t*>(q)[(static_cast<int64_t>(um.seq) * a.Hq + kvh * G + h) * D + c]
                              : static_cast<uint16_t>(0);
        }
        if (!GT && !*abort_flag && !mbar_wait_sleep(&tbar[seg & 1], (seg >> 1) & 1, abort_flag)) {
            if (!*abort_flag)
                report(a.err, RKV_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        consumer_sync(NCT);
        unit_max_fold<Gp>(w, u, R, tid, NCT, key_sm);
        if (tid < 4 * Gp) {
            const int g = tid / Gp, h = tid % Gp;
            float sum = 0.0f;
#pragma unroll 8
            for (int c = 0; c < 32; ++c)
                sum += bf16_bits_to_f32(q_sm[h * D + 32 * g + c]);
            qc_sm[g * Gp + h] = kCodeOffset * sum;
        }
        // K-side B operand in the ldmatrix layout: matrix (k-block, half) holds rows n (the
        // eight columns: head n / GPS, group residue n % GPS) of eight k-slots; the k-slot
        // order within a group follows the nibble order of the A fragments
        for (int x = tid; x < 8 * 2 * 8 * 8; x += NCT) {
            const int kb = x >> 7, half = (x >> 6) & 1, n = (x >> 3) & 7, slot = x & 7;
            const int g = kb >> 1, sub = kb & 1, tq2 = slot >> 1, e = slot & 1;
            const int nib = 2 * sub + half + 4 * e;
            const int h = n / GPS;
            const bool on = (g % GPS) == (n % GPS) && h < G;
            bk_sm[x] = on ? q_sm[h * D + 32 * g + 8 * tq2 + nib] : static_cast<uint16_t>(0);
        }
        consumer_sync(NCT);
        // ldmatrix row address of this lane for the K-side B operand of group 0 (+512 B per group)
        const uint32_t bk_base = smem_addr(bk_sm) + static_cast<uint32_t>(((lane >> 3) * 8 + (lane & 7)) * 16);
        float m_h[NH], qc_h[4][NH], l_acc[NH];
#pragma unroll
        for (int e = 0; e < NH; ++e) {
            const int h = (Gp == 4) ? tq : 2 * tq + e;
            m_h[e] = unit_m(key_sm, h);
            l_acc[e] = 0.0f;
#pragma unroll
            for (int g = 0; g < 4; ++g)
                qc_h[g][e] = qc_sm[g * Gp + h];
        }
        float dv[8][4];
        float colsum[NS];
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int x = 0; x < 4; ++x)
                dv[mt][x] = 0.0f;
#pragma unroll
        for (int s = 0; s < NS; ++s)
            colsum[s] = 0.0f;

        // ---- the unit's tiles, 16 tokens per warp ---------------------------------------
        for (; t < seg_end; ++t, ++i) {
            if (NTEAM > 1 && (i % NTEAM) != team)
                continue;
            const int s = i % nst;
            if (!*abort_flag && !mbar_wait_sleep(&full[s], (i / nst) & 1, abort_flag)) {
                if (!*abort_flag)
                    report(a.err, RKV_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            if (!*abort_flag) {
                unsigned char* st = stages + s * kStageBytes;
                const uint32_t stK = smem_addr(st), stV = stK + kStCodes;
                const uint16_t* sK = reinterpret_cast<const uint16_t*>(st + 2 * kStCodes);
                const uint16_t* sV = sK + kTok * 4;
                const uint16_t* ix = reinterpret_cast<const uint16_t*>(st + 2 * kStCodes + 2 * kStScale);
                const int rb = wi * kWarpTok;                                   // first row of this warp
                const int tok0 = static_cast<int>(static_cast<int64_t>(t) * kTok - um.cmp_row) + rb;
                float* pw = p_sm + warp * kWarpTok * Gp;

                // K side: D[token][column] per scale group, one MMA per 16 channels
                uint32_t wk0[4], wk1[4];
                ldsm_x4(stK + sw64(rb + (lane & 7), lane >> 3), wk0);
                ldsm_x4(stK + sw64(rb + 8 + (lane & 7), lane >> 3), wk1);
                float dk[4][4];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t bq[4];
                    ldsm_x4(bk_base + g * 512, bq);
                    dk[g][0] = dk[g][1] = dk[g][2] = dk[g][3] = 0.0f;
#pragma unroll
                    for (int sub = 0; sub < 2; ++sub) {
                        const int sh = 8 * sub;
                        mma_bf16(dk[g], nib2(wk0[g] >> sh), nib2(wk1[g] >> sh), nib2(wk0[g] >> (sh + 4)),
                                 nib2(wk1[g] >> (sh + 4)), bq[2 * sub], bq[2 * sub + 1]);
                    }
                }

                // softmax of this thread's two tokens (rows gid, gid + 8) and NH heads
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int row = rb + gid + 8 * rr;
                    const bool valid = tok0 + gid + 8 * rr < um.C;
                    const uint2 skw = *reinterpret_cast<const uint2*>(sK + row * 4);
                    const float sk[4] = {half_bits_to_f32(skw.x & 0xffffu), half_bits_to_f32(skw.x >> 16),
                                         half_bits_to_f32(skw.y & 0xffffu), half_bits_to_f32(skw.y >> 16)};
                    int oi[KK];
                    if (KK == 4 && a.k == 4) {
                        const uint2 v = *reinterpret_cast<const uint2*>(ix + row * 4);
                        oi[0] = v.x & 0xffff; oi[1] = v.x >> 16; oi[2] = v.y & 0xffff; oi[3] = v.y >> 16;
                    } else if (KK == 8 && a.k == 8) {
                        const uint4 v = *reinterpret_cast<const uint4*>(ix + row * 8);
                        oi[0] = v.x & 0xffff; oi[1] = v.x >> 16; oi[2] = v.y & 0xffff; oi[3] = v.y >> 16;
                        oi[KK > 4 ? 4 : 0] = v.z & 0xffff; oi[KK > 5 ? 5 : 0] = v.z >> 16;
                        oi[KK > 6 ? 6 : 0] = v.w & 0xffff; oi[KK > 7 ? 7 : 0] = v.w >> 16;
                    } else {
#pragma unroll
                        for (int j = 0; j < KK; ++j)
                            oi[j] = (j < a.k) ? ix[row * a.k + j] : RKV_IDX_UNUSED;
                    }
                    int keff = 0;
                    float sref[NH];
#pragma unroll
                    for (int e = 0; e < NH; ++e)
                        sref[e] = 0.0f;
#pragma unroll
                    for (int j = 0; j < KK; ++j) {
                        const bool has = valid && oi[j] != RKV_IDX_UNUSED;
                        corrupt |= has && oi[j] >= R;
                        const bool use = has && oi[j] < R;
                        oi[j] = use ? oi[j] : -1;
                        keff += use ? 1 : 0;
                        const int oc = use ? oi[j] : 0;     // unconditional load, selected sum
                        if constexpr (NH == 1) {
                            const float v = GT ? __ldg(s_sm + oc * Gp + tq) : s_sm[oc * Gp + tq];
                            sref[0] += use ? v : 0.0f;
                        } else {
                            const float2 v = GT ? __ldg(reinterpret_cast<const float2*>(s_sm + oc * Gp + 2 * tq))
                                                : *reinterpret_cast<const float2*>(s_sm + oc * Gp + 2 * tq);
                            sref[0] += use ? v.x : 0.0f;
                            sref[1] += use ? v.y : 0.0f;
                        }
                    }
                    const float rk = __frcp_rn(static_cast<float>(max(keff, 1)));
                    float pe[NH];
#pragma unroll
                    for (int e = 0; e < NH; ++e) {
                        const int h = (Gp == 4) ? tq : 2 * tq + e;
                        float acc = 0.0f;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const float raw = (Gp == 4) ? dk[g][(g & 1) + 2 * rr] : dk[g][e + 2 * rr];
                            acc = fmaf(sk[g], raw - qc_h[g][e], acc);
                        }
                        const float logit = fmaf(w.cK, acc, sref[e] * rk);
                        const float ex = logit - m_h[e];
                        const bool live = valid && keff > 0 && h < G;
                        overflow |= live && ex > 100.0f;
                        const float p = live ? exp2f(fminf(ex, 100.0f)) : 0.0f;
                        l_acc[e] += p;
                        pw[(gid + 8 * rr) * Gp + h] = p;
                        pe[e] = p * rk;
                    }
                    // reference weights: the four lanes of the row share all q-heads' p / k_eff,
                    // then lane tq adds them to references tq and tq + 4 with vector reductions
                    float pall[Gp];
#pragma unroll
                    for (int t2 = 0; t2 < 4; ++t2)
#pragma unroll
                        for (int e = 0; e < NH; ++e)
                            pall[NH * t2 + e] = __shfl_sync(0xffffffffu, pe[e], (lane & ~3) | t2);
#pragma unroll
                    for (int jj = 0; jj < KK / 4; ++jj) {
                        const int o = (tq == 0) ? oi[4 * jj] : (tq == 1) ? oi[4 * jj + 1]
                                    : (tq == 2) ? oi[4 * jj + 2] : oi[4 * jj + 3];
                        if (o >= 0) {
                            float* dst = w.W + (um.ref_row + o) * Gp;
#pragma unroll
                            for (int h4 = 0; h4 < Gp; h4 += 4)
                                red_global_v4(dst + h4, pall[h4], pall[h4 + 1], pall[h4 + 2], pall[h4 + 3]);
                        }
                    }
                }
                __syncwarp();

                // V-side B operand: column gid is (head gid / GPS, group residue gid % GPS),
                // k-slots are the tokens 2tq, 2tq+1, 2tq+8, 2tq+9 of the warp's block; p * sV
                // enters as a hi + lo pair of bf16 operands (two MMAs into one accumulator)
                uint32_t bv[NS][2], bl[NS][2];
                {
                    const int hv = gid / GPS, gv = gid % GPS;
                    const int tv[4] = {2 * tq, 2 * tq + 1, 2 * tq + 8, 2 * tq + 9};
                    float pv[4];
                    uint2 svw[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        pv[x] = pw[tv[x] * Gp + hv];
                        svw[x] = *reinterpret_cast<const uint2*>(sV + (rb + tv[x]) * 4);
                    }
#pragma unroll
                    for (int s2 = 0; s2 < NS; ++s2) {
                        const int g = s2 * GPS + gv;
                        float v[4];
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const uint32_t word = (g < 2) ? svw[x].x : svw[x].y;
                            const float sc = half_bits_to_f32((g & 1) ? (word >> 16) : (word & 0xffffu));
                            v[x] = (pv[x] != 0.0f) ? pv[x] * sc : 0.0f;
                        }
                        split_bf16(v[0], v[1], bv[s2][0], bl[s2][0], colsum[s2]);
                        split_bf16(v[2], v[3], bv[s2][1], bl[s2][1], colsum[s2]);
                    }
                }
                __syncwarp();

                // V side: D[channel][column] += codes^T x B, two MMAs (32 channels) per group
                uint32_t xv[2][4];
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    ldsm_x4_t(stV + sw64(rb + 8 * ((lane >> 3) & 1) + (lane & 7), 2 * c + (lane >> 4)), xv[c]);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t xl = xv[g >> 1][(g & 1) * 2], xh = xv[g >> 1][(g & 1) * 2 + 1];
                    const int s2 = g / GPS;
                    const uint32_t a0 = nib2(xl), a1 = nib2(xl >> 4), a2 = nib2(xh), a3 = nib2(xh >> 4);
                    const uint32_t c0 = nib2(xl >> 8), c1 = nib2(xl >> 12), c2 = nib2(xh >> 8), c3 = nib2(xh >> 12);
                    mma_bf16(dv[2 * g], a0, a1, a2, a3, bv[s2][0], bv[s2][1]);
                    mma_bf16(dv[2 * g + 1], c0, c1, c2, c3, bv[s2][0], bv[s2][1]);
                    mma_bf16(dv[2 * g], a0, a1, a2, a3, bl[s2][0], bl[s2][1]);
                    mma_bf16(dv[2 * g + 1], c0, c1, c2, c3, bl[s2][0], bl[s2][1]);
                }
            }
            // the last warp done with the stage refills it with local tile i + nst
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                if (atomicAdd(&done_cnt[s], 1) == kConsWarps - 1) {
                    done_cnt[s] = 0;
                    const int j = i + nst;
                    if (j < n_local && !*abort_flag) {
                        fence_proxy_async_smem();
                        issue(j);
                        atomicMax(issued, j + 1);
                    }
                }
            }
        }

        // ---- flush the unit's partial sums -----------------------------------------------
        consumer_sync(NCT);
        {
            // column sums of the V-side B operand (sum over the four lanes of a column), then
            // the sums of the two columns this thread's accumulators hold
            float cs[NS][2];
#pragma unroll
            for (int s2 = 0; s2 < NS; ++s2) {
                float tot = colsum[s2];
                tot += __shfl_xor_sync(0xffffffffu, tot, 1);
                tot += __shfl_xor_sync(0xffffffffu, tot, 2);
                cs[s2][0] = __shfl_sync(0xffffffffu, tot, (2 * tq) * 4);
                cs[s2][1] = __shfl_sync(0xffffffffu, tot, (2 * tq + 1) * 4);
            }
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int ch = 32 * g + 4 * gid + 2 * hf + rr;
                        const float* d = dv[2 * g + hf];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            // Gp 4: column 2tq + e is (head tq, group residue e); Gp 8: head 2tq + e
                            const int h = (Gp == 4) ? tq : 2 * tq + e;
                            const bool mine = (Gp == 4) ? (e == (g & 1)) : true;
                            if (mine)
                                o_sm[(warp * Gp + h) * D + ch] = d[e + 2 * rr] - kCodeOffset * cs[g / GPS][e];
                        }
                    }
#pragma unroll
            for (int e = 0; e < NH; ++e) {
                float v = l_acc[e];
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                const int h = (Gp == 4) ? tq : 2 * tq + e;
                if (gid == 0 && h < G)
                    red_shared(&l_sm[h], v);
            }
        }
        consumer_sync(NCT);
        // the table buffer of this segment is free: the segment after next loads into it
        if (!GT && warp == 0 && seg_end < t_hi) {
            const int u1 = unit_after(u, seg_end);
            const int t2 = min(t_hi, unit_end(u1));
            if (t2 < t_hi) {
                const int u2 = unit_after(u1, t2);
                if (lane == 0 && !*abort_flag) {
                    fence_proxy_async_smem();
                    load_table(seg & 1, u2);
                }
            }
        }
        if (!*abort_flag) {
            for (int x = tid; x < G * D; x += NCT) {
                float v = 0.0f;
#pragma unroll 4
                for (int wv = 0; wv < kConsWarps * NTEAM; ++wv)
                    v += o_sm[wv * Gp * D + x];
                atomicAdd(&w.O[static_cast<int64_t>(u) * Gp * D + x], v);
            }
            if (tid < G)
                atomicAdd(&w.L[u * Gp + tid], l_sm[tid]);
        }
        t = seg_end;
        u = unit_after(u, t);
        ++seg;
    }
    if (__any_sync(0xffffffffu, overflow) && lane == 0)
        report(a.err, RKV_ERR_UNSUPPORTED);
    if (__any_sync(0xffffffffu, corrupt) && lane == 0)
        report(a.err, RKV_ERR_CORRUPT);
    // the copies of the last stages land before the CTA may exit (only after an abort can
    // one still be in flight here)
    consumer_sync(NCT);
    if (tid == 0) {
        const int n = *issued;
        for (int j = (n > nst ? n - nst : 0); j < n; ++j)
            mbar_wait_sleep(&full[j % nst], (j / nst) & 1, zero_flag);
        for (int bf = 0; bf < 2; ++bf)
            if (tables_issued[bf] > 0)
                mbar_wait_sleep(&tbar[bf], (tables_issued[bf] - 1) & 1, zero_flag);
    }
}

// ==== 3. reference tokens, reference weights, output =========================================

// Chunks of kRefChunk references per CTA of the refs kernel.  One: the kernel is bound by the
// latency of each CTA's chain of dependent loads, so more CTAs in flight beat fewer, longer ones
// (four chunks per CTA measured slower on every workload).
constexpr int kRefBlock = 1;

template <int Gp, int RB, bool LC>
__global__ void __launch_bounds__(256, 4) mma_refs_kernel(const CacheArgs a, void* __restrict__ out, const MmaWs w)
{
    constexpr int D = 128;
    constexpr int RQ = kRefChunk / 4;      // references per thread quarter and chunk
    __shared__ float wt[kRefChunk][Gp];
    __shared__ float red[4][Gp][D];
    __shared__ float lred[Gp];
    __shared__ uint32_t key[Gp];
    __shared__ int last;
    const int u = blockIdx.y, tid = threadIdx.x;
    const UnitMeta um = a.units[u];
    const int R = um.R;
    const int nch = max(1, (R + kRefChunk - 1) / kRefChunk);
    const int nblk = (nch + kRefBlock - 1) / kRefBlock;
    if (static_cast<int>(blockIdx.x) >= nblk)
        return;
    const int G = a.G;
    const int kvh = u - um.seq * a.Hkv;
    const int cp = tid & 63, qq = tid >> 6;
    __shared__ float ssc[RB == 4 ? kRefChunk * (D / 32) : 1];   // int4 store: the chunk's V scales
    if (tid < Gp)
        key[tid] = 0u;
    __syncthreads();
    // the common offsets depend only on the scores kernel (complete once this kernel runs; read
    // through L2), so they are folded before the wait on the tokens kernel
    unit_max_fold<Gp>(w, u, R, tid, 256, key);
    __syncthreads();
    float acc[Gp][2];
#pragma unroll
    for (int h = 0; h < Gp; ++h)
        acc[h][0] = acc[h][1] = 0.0f;
    float lsum = 0.0f;
    constexpr int PJ = kRefChunk * Gp / 256;
    for (int sc = 0; sc < kRefBlock; ++sc) {
        const int ch = static_cast<int>(blockIdx.x) * kRefBlock + sc;
        if (ch >= nch)
            break;
        const int r0 = ch * kRefChunk, r1 = min(R, r0 + kRefChunk);
        // the chunk's reference V rows and the reference tokens' own terms p_r (for the first
        // chunk before the wait on the tokens kernel)
        float rv[RQ][2];
        uint32_t cb[RB == 4 ? RQ : 1];
        if constexpr (RB == 4) {
            // one code byte (channels 2cp, 2cp+1) per row; the rows' scales staged once per chunk
            const uint8_t* codes = reinterpret_cast<const uint8_t*>(a.ref_V);
#pragma unroll
            for (int rr = 0; rr < RQ; ++rr) {
                const int r = r0 + qq * RQ + rr;
                cb[rr] = (r < r1) ? codes[(um.ref_row + r) * (D / 2) + cp] : 0u;
            }
            if (tid < kRefChunk * (D / 32)) {
                const int r = r0 + tid / (D / 32);
                ssc[tid] = (r < r1) ? __half2float(__ushort_as_half(a.ref_sV[(um.ref_row + r) * (D / 32) + tid % (D / 32)]))
                                    : 0.0f;
            }
        } else {
#pragma unroll
            for (int rr = 0; rr < RQ; ++rr) {
                const int r = r0 + qq * RQ + rr;
                rv[rr][0] = rv[rr][1] = 0.0f;
                if (r < r1)
                    load_ref<2, RB>(a, 1, um.ref_row + r, 2 * cp, rv[rr]);
            }
        }
        float pj[PJ > 0 ? PJ : 1];
#pragma unroll
        for (int z = 0; z < PJ; ++z) {
            const int x = tid + 256 * z;
            const int r = r0 + x / Gp, h = x % Gp;
            float v = 0.0f;
            if (r < r1 && h < G)
                v = exp2f(__ldcg(w.s_tab + (um.ref_row + r) * Gp + h) - unit_m(key, h));
            pj[z] = v;
            lsum += v;
        }
        if (sc == 0)
            grid_dep_wait();   // weights and partial sums of the tokens kernel
        // weight of reference r: its own softmax term p_r plus w_r from the tokens that chose it
#pragma unroll
        for (int z = 0; z < PJ; ++z) {
            const int x = tid + 256 * z;
            const int r = r0 + x / Gp, h = x % Gp;
            wt[x / Gp][h] = (r < r1 && h < G) ? w.W[(um.ref_row + r) * Gp + h] + pj[z] : 0.0f;
        }
        __syncthreads();
        if constexpr (RB == 4) {
#pragma unroll
            for (int rr = 0; rr < RQ; ++rr) {
                const float scl = ssc[(qq * RQ + rr) * (D / 32) + cp / 16];
                rv[rr][0] = __fmul_rn(static_cast<float>(static_cast<int>((cb[rr] & 0xfu) ^ 8u) - 8), scl);
                rv[rr][1] = __fmul_rn(static_cast<float>(static_cast<int>((cb[rr] >> 4) ^ 8u) - 8), scl);
            }
        }
        // sum_r wt[r][h] refV[r][c]: thread (channel pair, quarter of the chunk)
#pragma unroll
        for (int rr = 0; rr < RQ; ++rr) {
            const float x0 = rv[rr][0], x1 = rv[rr][1];
            const float* wr = wt[qq * RQ + rr];
#pragma unroll
            for (int h = 0; h < Gp; ++h) {
                acc[h][0] = fmaf(wr[h], x0, acc[h][0]);
                acc[h][1] = fmaf(wr[h], x1, acc[h][1]);
            }
        }
        __syncthreads();   // wt and ssc are refilled by the next chunk
    }
    // per-head sums: entry x holds head x % Gp (256 % Gp == 0)
#pragma unroll
    for (int o = Gp; o < 32; o <<= 1)
        lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    if ((tid & 31) < Gp)
        (&red[0][0][0])[(tid >> 5) * Gp + (tid & 31)] = lsum;   // scratch: 8 warps x Gp
    __syncthreads();
    if (tid < Gp) {
        float v = 0.0f;
        for (int i = 0; i < 8; ++i)
            v += red[0][0][i * Gp + tid];
        lred[tid] = v;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < Gp; ++h) {
        red[qq][h][2 * cp] = acc[h][0];
        red[qq][h][2 * cp + 1] = acc[h][1];
    }
    __syncthreads();
    for (int x = tid; x < G * D; x += 256) {
        const int h = x / D, c = x % D;
        atomicAdd(&w.O[static_cast<int64_t>(u) * Gp * D + x], red[0][h][c] + red[1][h][c] + red[2][h][c] + red[3][h][c]);
    }
    if (tid < G)
        atomicAdd(&w.L[u * Gp + tid], lred[tid]);
    __threadfence();
    __syncthreads();
    if (tid == 0)
        last = (atomicAdd(&w.cnt[u], 1u) == static_cast<uint32_t>(nblk - 1)) ? 1 : 0;
    __syncthreads();
    if (!last)
        return;
    __threadfence();
    if constexpr (LC) {
        // learned-coder shapes: fd applied once to the softmax-weighted latent sum, o += Wd_V
        // (sum_i p_i z_i); the latent sums staged in shared memory, one warp per output row c
        for (int x = tid; x < G * D; x += 256)
            red[0][x / D][x % D] = __ldcg(&w.Olat[static_cast<int64_t>(u) * Gp * D + x]);
        __syncthreads();
        // thread: output row c = tid % D for the heads h = tid / D, tid / D + 2, ... (the row of
        // Wd_V read once, sixteen 16-byte loads in flight)
        const int c = tid % D;
        const uint4* wrow = reinterpret_cast<const uint4*>(a.cw[7] + c * D);
        for (int h = tid / D; h < G; h += 256 / D) {
            const float* ol = red[0][h];
            float acc = 0.0f;
#pragma unroll
            for (int i0 = 0; i0 < D / 8; i0 += 8) {
                uint4 wr[8];                       // eight 16-byte loads in flight
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    wr[i] = wrow[i0 + i];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t ww[4] = {wr[i].x, wr[i].y, wr[i].z, wr[i].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc = fmaf(bf16_bits_to_f32(ww[e] & 0xffffu), ol[8 * (i0 + i) + 2 * e], acc);
                        acc = fmaf(bf16_bits_to_f32(ww[e] >> 16), ol[8 * (i0 + i) + 2 * e + 1], acc);
                    }
                }
            }
            red[1][h][c] = acc;
        }
        __syncthreads();
    }
    for (int x = tid; x < G * D; x += 256) {
        const int h = x / D, c = x % D;
        float o = __ldcg(&w.O[static_cast<int64_t>(u) * Gp * D + x]);
        if constexpr (LC)
            o += red[1][h][c];
        const float l = __ldcg(&w.L[u * Gp + h]);
        const float res = (l > 0.0f) ? o / l : 0.0f;
        const int64_t e = (static_cast<int64_t>(um.seq) * a.Hq + kvh * G + h) * D + c;
        if (a.out_dtype == RKV_DTYPE_F32)
            static_cast<float*>(out)[e] = res;
        else
            static_cast<uint16_t*>(out)[e] = f32_to_bf16_bits(res);
    }
}

// ==== host side ==============================================================================

constexpr int kTeams = 2;      // warp teams of the tokens kernel (each takes every other stage)

int heads_padded(int G) { return G <= 4 ? 4 : 8; }

// Opt-in shared memory per block on sm_100 (227 KB); a constant so that workspace sizes do
// not depend on the device present when they are computed.
constexpr int kSmemOptin = 232448;

// Pipeline depth that fits next to the unit tables (0 if fewer than four stages fit);
// table_refs = 0 when the tables stay in global memory.
int tok_stages(const CacheArgs& a, int table_refs)
{
    const int Gp = heads_padded(a.G);
    const int fixed = TokLayout(Gp, kConsWarps * kTeams, table_refs, 0).total + 1024;
    const int avail = kSmemOptin - fixed;
    const int n = avail / kStageBytes;
    return n < 4 ? 0 : (n > 8 ? 8 : n);
}

// Score tables in shared memory when they fit next to four or more stages, else in L2.
bool tables_global(const CacheArgs& a) { return tok_stages(a, a.max_refs) == 0; }

constexpr int kMaxCta = 160;   // grid cap of the tokens kernel

struct WsOffsets {
    uint64_t s_tab, W, mpart, O, L, cnt, Olat, qlat, end;
};

WsOffsets ws_offsets(const CacheArgs& a, int64_t ref_rows)
{
    const int Gp = heads_padded(a.G);
    const int n_chunk = (a.max_refs + kRefChunk - 1) / kRefChunk > 0 ? (a.max_refs + kRefChunk - 1) / kRefChunk : 1;
    uint64_t off = 0;
    auto take = [&](uint64_t bytes) {
        const uint64_t o = off;
        off = (off + bytes + 255) / 256 * 256;
        return o;
    };
    WsOffsets o;
    o.s_tab = take(4ull * ref_rows * Gp);
    o.W = take(4ull * ref_rows * Gp);
    o.mpart = take(4ull * a.n_units * n_chunk * Gp);
    o.O = take(4ull * a.n_units * Gp * 128);
    o.L = take(4ull * a.n_units * Gp);
    o.cnt = take(4ull * a.n_units);
    o.Olat = take(a.coder == 1 ? 4ull * a.n_units * Gp * 128 : 0);
    o.qlat = take(a.coder == 1 ? 2ull * a.n_units * a.G * 128 : 0);
    o.end = off;
    return o;
}

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn encoder()
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeFn>(fn);
}

// Byte-typed 2D map over the int4 code rows (64 bytes each), 128-row boxes, 64-byte swizzle.
bool code_map(EncodeFn enc, CUtensorMap* m, const void* base, int64_t rows)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kCodeRow), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kCodeRow)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kCodeRow), static_cast<cuuint32_t>(kTok)};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int Gp>
cudaError_t launch_gp(const CacheArgs& a, int64_t cmp_rows, const void* q, void* out, const MmaWs& w, int nst,
                      cudaStream_t st)
{
    EncodeFn enc = encoder();
    if (!enc)
        return cudaErrorNotSupported;
    alignas(64) CUtensorMap mK;
    alignas(64) CUtensorMap mV;
    if (!code_map(enc, &mK, a.codes_K, cmp_rows) || !code_map(enc, &mV, a.codes_V, cmp_rows))
        return cudaErrorInvalidValue;
    const dim3 rgrid(w.n_chunk, a.n_units);
    const dim3 fgrid((w.n_chunk + kRefBlock - 1) / kRefBlock, a.n_units);   // refs kernel
    if (a.coder == 1)
        mma_scores_kernel<Gp, 16, true><<<rgrid, 128, 0, st>>>(a, q, w);
    else if (a.ref_bits == 4)
        mma_scores_kernel<Gp, 4, false><<<rgrid, 128, 0, st>>>(a, q, w);
    else
        mma_scores_kernel<Gp, 16, false><<<rgrid, 128, 0, st>>>(a, q, w);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    if (w.n_tiles > 0) {
        // learned-coder shapes: the tokens kernel meets the latent codes with q' and sums the
        // latent V side into Olat (the refs kernel applies fd to it)
        MmaWs wt = w;
        const void* qt = q;
        if (a.coder == 1) {
            wt.O = w.Olat;
            qt = w.qlat;
        }
        e = launch_tokens_tc(a, wt, qt, Gp, st);
        if (e != cudaSuccess)
            return e;
    }
    if (a.coder == 1)
        return launch_pdl(mma_refs_kernel<Gp, 16, true>, fgrid, dim3(256), 0, st, a, out, w);
    if (a.ref_bits == 4)
        return launch_pdl(mma_refs_kernel<Gp, 4, false>, fgrid, dim3(256), 0, st, a, out, w);
    return launch_pdl(mma_refs_kernel<Gp, 16, false>, fgrid, dim3(256), 0, st, a, out, w);
}

}  // namespace

bool decode_mma_supported(const CacheArgs& a)
{
    return a.D == 128 && a.bits == 4 && a.group == 32 && a.in_dtype == RKV_DTYPE_BF16 && a.G >= 1 && a.G <= 8 &&
           a.k >= 1 && a.k <= 8 && tok_stages(a, 0) > 0;
}

uint64_t decode_mma_ws_bytes(const CacheArgs& a, int64_t ref_rows) { return ws_offsets(a, ref_rows).end; }

cudaError_t launch_decode_mma(const CacheArgs& a, int64_t ref_rows, int64_t cmp_rows, const void* q, void* out,
                              void* workspace, cudaStream_t st)
{
    const WsOffsets o = ws_offsets(a, ref_rows);
    char* base = static_cast<char*>(workspace);
    MmaWs w;
    w.s_tab = reinterpret_cast<float*>(base + o.s_tab);
    w.W = reinterpret_cast<float*>(base + o.W);
    w.mpart = reinterpret_cast<float*>(base + o.mpart);
    w.O = reinterpret_cast<float*>(base + o.O);
    w.L = reinterpret_cast<float*>(base + o.L);
    w.cnt = reinterpret_cast<uint32_t*>(base + o.cnt);
    w.Olat = reinterpret_cast<float*>(base + o.Olat);
    w.qlat = reinterpret_cast<uint16_t*>(base + o.qlat);
    w.n_chunk = (a.max_refs + kRefChunk - 1) / kRefChunk > 0 ? (a.max_refs + kRefChunk - 1) / kRefChunk : 1;
    w.n_tiles = static_cast<int>(cmp_rows / kTok);
    {
        int dev = 0, sms = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return e;
        w.n_cta = std::min(std::min(sms, kMaxCta), std::max(w.n_tiles, 1));
    }
    w.cK = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
    const int nst = tok_stages(a, tables_global(a) ? 0 : a.max_refs);
    if (nst < 4)
        return cudaErrorNotSupported;
    return heads_padded(a.G) == 4 ? launch_gp<4>(a, cmp_rows, q, out, w, nst, st)
                                  : launch_gp<8>(a, cmp_rows, q, out, w, nst, st);
}

}  // namespace rkv
