// Decode attention over the compressed cache: the reference-side kernels (ResidualKV paper
// summary page, "Practical Deployment via Sparse-vLLM": reconstruction fused into attention;
// news page, "How ResidualKV Works": tokens rebuilt on the fly when attention needs them).
//
// The algebra is the factorised one (reference scores s_j = q.refK_j, reference
// weights w_j = sum of p_i / k_eff over the tokens that chose j):
//   logit_i = mean_{j in S(i)} s_j + sum_g sK_ig * (q . codeK_i)_g
//   out     = (sum_i p_i sum_g sV_ig codeV_i|g + sum_j (p_j + w_j) refV_j) / (sum_i p_i + sum_j p_j)
// with every p taken against one common offset m = max_j s_j per (unit, q-head), so
// partial sums from any number of CTAs add without rescaling.  Three kernels, chained with
// programmatic dependent launch:
//   1. scores:  s_j for every reference (fp32, log2 units, m16n8k16 bf16 MMAs) and
//               per-64-reference maxima; zeroes the weight and output accumulators;
//   2. tokens:  the compressed tokens on the tcgen05 tensor cores (kernels_decode_tc.cu);
//   3. refs:    sum_j (p_j + w_j) refV_j per 64-reference chunk; the last chunk of a
//               unit to finish normalises and writes the output.

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

constexpr int kTok = 128;            // tokens per tile of the tokens kernel (= compressed-row padding)

// ---- small PTX wrappers ------------------------------------------------------------------

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

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
    float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    auto word = [](const uint4 (&v)[4], int i) {
        const uint4 x = v[i >> 2];
        return (i & 3) == 0 ? x.x : (i & 3) == 1 ? x.y : (i & 3) == 2 ? x.z : x.w;
    };
#pragma unroll
    for (int kb = 0; kb < 8; ++kb)
        mma_bf16(d, word(ar[0], 2 * kb), word(ar[1], 2 * kb), word(ar[0], 2 * kb + 1), word(ar[1], 2 * kb + 1),
                 word(bq, 2 * kb), word(bq, 2 * kb + 1));
    // everything above only reads (the cache's reference keys and the query); the writes below
    // reuse the workspace of the previous decode on this stream, which may still be running
    // (this kernel is its programmatic dependent): wait for it here
    grid_dep_wait();
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

// ==== 3. reference tokens, reference weights, output =========================================

// Chunks per CTA of the refs kernel (w.ref_blk): as few as keep the grid within one wave of
// resident CTAs.  The kernel is bound by each CTA's chain of dependent loads, so a second wave
// that starts only when the first ends costs a whole chain; the V rows of a CTA's later
// chunks are prefetched into L2 before the wait on the tokens kernel.
constexpr int kRefsPerSm = 4;   // resident CTAs of the refs kernel per SM (launch bounds)

template <int Gp, int RB, bool LC>
__global__ void __launch_bounds__(256, kRefsPerSm) mma_refs_kernel(const CacheArgs a, void* __restrict__ out, const MmaWs w)
{
    constexpr int D = 128;
    constexpr int RQ = kRefChunk / 4;      // references per thread quarter and chunk
    __shared__ float wt[kRefChunk][Gp];
    __shared__ float red[4][Gp][D];
    __shared__ float lred[Gp];
    __shared__ uint32_t key[Gp];
    __shared__ int last;
    grid_dep_launch();   // the next decode's scores kernel may start its loads
    const int u = blockIdx.y, tid = threadIdx.x;
    const UnitMeta um = a.units[u];
    const int R = um.R;
    const int nch = max(1, (R + kRefChunk - 1) / kRefChunk);
    const int nblk = (nch + w.ref_blk - 1) / w.ref_blk;
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
    {
        // the V rows of this CTA's later chunks into L2 (the first chunk's go to registers below)
        constexpr int row_bytes = (RB == 4) ? D / 2 : 2 * D;
        const int c_hi = min(nch, (static_cast<int>(blockIdx.x) + 1) * w.ref_blk);
        const int r_lo = min(R, (static_cast<int>(blockIdx.x) * w.ref_blk + 1) * kRefChunk);
        const int r_hi = min(R, c_hi * kRefChunk);
        const char* vb = reinterpret_cast<const char*>(a.ref_V) + (um.ref_row + r_lo) * row_bytes;
        for (int o = tid * 128; o < (r_hi - r_lo) * row_bytes; o += 256 * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(vb + o));
    }
    for (int sc = 0; sc < w.ref_blk; ++sc) {
        const int ch = static_cast<int>(blockIdx.x) * w.ref_blk + sc;
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

int heads_padded(int G) { return G <= 4 ? 4 : 8; }

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
cudaError_t launch_gp(const CacheArgs& a, const void* q, void* out, const MmaWs& w, cudaStream_t st)
{
    const dim3 rgrid(w.n_chunk, a.n_units);
    const dim3 fgrid((w.n_chunk + w.ref_blk - 1) / w.ref_blk, a.n_units);   // refs kernel
    // the scores kernel loads and multiplies while the previous decode on the stream finishes
    // (it waits for it before its first write)
    cudaError_t e = (a.coder == 1)      ? launch_pdl(mma_scores_kernel<Gp, 16, true>, rgrid, dim3(128), 0, st, a, q, w)
                    : (a.ref_bits == 4) ? launch_pdl(mma_scores_kernel<Gp, 4, false>, rgrid, dim3(128), 0, st, a, q, w)
                                        : launch_pdl(mma_scores_kernel<Gp, 16, false>, rgrid, dim3(128), 0, st, a, q, w);
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
           a.k >= 1 && a.k <= 8;
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
        // refs kernel: one wave of resident CTAs (at most four chunks per CTA)
        const int64_t chunks = static_cast<int64_t>(w.n_chunk) * a.n_units;
        const int64_t slots = static_cast<int64_t>(kRefsPerSm) * sms;
        w.ref_blk = static_cast<int>(std::min<int64_t>(4, std::max<int64_t>(1, (chunks + slots - 1) / slots)));
    }
    w.cK = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
    return heads_padded(a.G) == 4 ? launch_gp<4>(a, q, out, w, st) : launch_gp<8>(a, q, out, w, st);
}

}  // namespace rkv
