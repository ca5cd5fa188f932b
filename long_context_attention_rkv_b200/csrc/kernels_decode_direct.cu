// Decode attention by direct reconstruction (ResidualKV paper summary page,
// "Practical Deployment via Sparse-vLLM": a fused kernel that gathers the
// reference tokens, takes their mean and adds the residual; news page, "How
// ResidualKV Works": tokens are rebuilt on the fly when attention needs them).
//
// Literal form: for every cached token a warp gathers its k reference rows
// (L2-resident), averages them, adds the dequantised residual and feeds the row
// into an online softmax for the G query heads of the kv head.  Nothing is
// written back.  Kept as the straightforward baseline of the factorised decode.
//
// Grid: (splits, units); each CTA takes one contiguous range of the unit's
// tokens (references first, then compressed tokens) and writes one partial
// softmax state (m, l, o[D]) per query head, in log2 units.  The combine
// kernel merges the splits.  With a position list (selective decompression)
// the CTA ranges split the unit's listed positions instead, each mapped to its
// reference row or compressed slot.
#include <cfloat>
#include <cmath>

#include "device_common.cuh"
#include "launchers.h"

namespace rkv {

namespace {

constexpr int kWarps = 4;

template <int NPL, int RB>
__device__ __forceinline__ bool rebuild_compressed(const CacheArgs& a, const UnitMeta& um, int c, int lane,
                                                   float (&xk)[NPL], float (&xv)[NPL])
{
    constexpr int D = NPL * 32;
    constexpr int LPG = 32 / NPL;
    const int64_t row = um.cmp_row + c;
    const uint16_t* id = a.idx + row * a.k;
    int keff = 0;
    bool bad = false;
    float sk[NPL], sv[NPL];
#pragma unroll
    for (int j = 0; j < NPL; ++j)
        sk[j] = sv[j] = 0.0f;
    for (int l = 0; l < a.k; ++l) {
        const int o = id[l];
        if (o == RKV_IDX_UNUSED)
            break;
        bad |= o >= um.R;
        if (bad)
            break;
        float rk[NPL], rv[NPL];
        load_ref<NPL, RB>(a, 0, um.ref_row + o, lane * NPL, rk);
        load_ref<NPL, RB>(a, 1, um.ref_row + o, lane * NPL, rv);
#pragma unroll
        for (int j = 0; j < NPL; ++j) {
            sk[j] = (l == 0) ? rk[j] : __fadd_rn(sk[j], rk[j]);
            sv[j] = (l == 0) ? rv[j] : __fadd_rn(sv[j], rv[j]);
        }
        ++keff;
    }
    if (bad || keff == 0)
        return false;
    const float fk = static_cast<float>(keff);
    const uint8_t* ck = a.codes_K + row * a.code_bytes;
    const uint8_t* cv = a.codes_V + row * a.code_bytes;
    const float s_k = __half2float(__ushort_as_half(a.scale_K[row * a.n_groups + lane / LPG]));
    const float s_v = __half2float(__ushort_as_half(a.scale_V[row * a.n_groups + lane / LPG]));
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        xk[j] = __fadd_rn(__fdiv_rn(sk[j], fk), __fmul_rn(static_cast<float>(code_at(ck, a.bits, lane * NPL + j)), s_k));
        xv[j] = __fadd_rn(__fdiv_rn(sv[j], fk), __fmul_rn(static_cast<float>(code_at(cv, a.bits, lane * NPL + j)), s_v));
    }
    return true;
}

template <int NPL, int GMAX, int RB>
__global__ void __launch_bounds__(kWarps * 32) decode_direct_kernel(CacheArgs a, const void* __restrict__ q,
                                                                    float* __restrict__ part, int splits,
                                                                    float qscale, const int32_t* __restrict__ sel,
                                                                    const int32_t* __restrict__ sel_cnt,
                                                                    int sel_stride)
{
    constexpr int D = NPL * 32;
    __shared__ float s_m[kWarps][GMAX];
    __shared__ float s_l[kWarps][GMAX];
    __shared__ float s_o[kWarps][GMAX][D];

    const int u = blockIdx.y;
    const int split = blockIdx.x;
    const UnitMeta um = a.units[u];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = a.G;
    const int h = u - um.seq * a.Hkv;
    const int T = sel ? max(0, min(sel_cnt[u], sel_stride)) : um.R + um.C;
    const int per = (T + splits - 1) / splits;
    const int v0 = split * per;
    const int v1 = min(T, v0 + per);

    float qv[GMAX][NPL];
    float m[GMAX], l[GMAX], o[GMAX][NPL];
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
        m[g] = -FLT_MAX;
        l[g] = 0.0f;
#pragma unroll
        for (int j = 0; j < NPL; ++j) {
            o[g][j] = 0.0f;
            qv[g][j] = 0.0f;
        }
        if (g < G) {
            const int64_t e = (static_cast<int64_t>(um.seq) * a.Hq + h * G + g) * D + lane * NPL;
            load_row_part<NPL>(q, e, a.in_dtype, qv[g]);
#pragma unroll
            for (int j = 0; j < NPL; ++j)
                qv[g][j] *= qscale;
        }
    }

    for (int vi = v0 + warp; vi < v1; vi += kWarps) {
        int v = vi;
        if (sel) {
            // listed position -> storage index: reference ordinal, or R + compressed slot
            const int p = sel[static_cast<int64_t>(u) * sel_stride + vi];
            if (p < 0 || p >= um.n) {
                if (lane == 0)
                    report(a.err, RKV_ERR_INVALID_ARG);
                continue;
            }
            const int nr = refs_upto(a.ph, p);
            v = is_ref_pos(a.ph, p) ? nr - 1 : um.R + (p - nr);
        }
        float xk[NPL], xv[NPL];
        if (v < um.R) {
            load_ref<NPL, RB>(a, 0, um.ref_row + v, lane * NPL, xk);
            load_ref<NPL, RB>(a, 1, um.ref_row + v, lane * NPL, xv);
        } else if (!rebuild_compressed<NPL, RB>(a, um, v - um.R, lane, xk, xv)) {
            if (lane == 0)
                report(a.err, RKV_ERR_CORRUPT);
            continue;
        }
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            if (g < G) {
                float d = 0.0f;
#pragma unroll
                for (int j = 0; j < NPL; ++j)
                    d = fmaf(qv[g][j], xk[j], d);
                d = warp_sum(d);
                const float mn = fmaxf(m[g], d);
                const float corr = exp2f(m[g] - mn);
                const float p = exp2f(d - mn);
                l[g] = fmaf(l[g], corr, p);
#pragma unroll
                for (int j = 0; j < NPL; ++j)
                    o[g][j] = fmaf(o[g][j], corr, p * xv[j]);
                m[g] = mn;
            }
        }
    }

    // merge the warps of the CTA
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
        if (g < G) {
            if (lane == 0) {
                s_m[warp][g] = m[g];
                s_l[warp][g] = l[g];
            }
#pragma unroll
            for (int j = 0; j < NPL; ++j)
                s_o[warp][g][lane * NPL + j] = o[g][j];
        }
    }
    __syncthreads();
    float* out = part + (static_cast<int64_t>(u) * splits + split) * G * (D + 2);
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D;
        const int c = i % D;
        float M = -FLT_MAX;
        for (int w = 0; w < kWarps; ++w)
            M = fmaxf(M, s_m[w][g]);
        float L = 0.0f, O = 0.0f;
        for (int w = 0; w < kWarps; ++w) {
            const float f = (s_l[w][g] > 0.0f) ? exp2f(s_m[w][g] - M) : 0.0f;
            L = fmaf(s_l[w][g], f, L);
            O = fmaf(s_o[w][g][c], f, O);
        }
        if (c == 0) {
            out[g * (D + 2)] = M;
            out[g * (D + 2) + 1] = L;
        }
        out[g * (D + 2) + 2 + c] = O;
    }
}

template <int NPL>
__global__ void decode_combine_kernel(CacheArgs a, int splits, const float* __restrict__ part, void* out)
{
    constexpr int D = NPL * 32;
    const int b = blockIdx.y;
    const int hq = blockIdx.x;
    const int G = a.G;
    const int u = b * a.Hkv + hq / G;
    const int g = hq % G;
    const int c = threadIdx.x;
    const float* base = part + static_cast<int64_t>(u) * splits * G * (D + 2) + g * (D + 2);
    float M = -FLT_MAX;
    for (int s = 0; s < splits; ++s) {
        const float* p = base + static_cast<int64_t>(s) * G * (D + 2);
        if (p[1] > 0.0f)
            M = fmaxf(M, p[0]);
    }
    float L = 0.0f, O = 0.0f;
    for (int s = 0; s < splits; ++s) {
        const float* p = base + static_cast<int64_t>(s) * G * (D + 2);
        if (p[1] > 0.0f) {
            const float f = exp2f(p[0] - M);
            L = fmaf(p[1], f, L);
            O = fmaf(p[2 + c], f, O);
        }
    }
    const float r = (L > 0.0f) ? O / L : 0.0f;
    const int64_t e = (static_cast<int64_t>(b) * a.Hq + hq) * D + c;
    if (a.out_dtype == RKV_DTYPE_F32)
        static_cast<float*>(out)[e] = r;
    else
        static_cast<uint16_t*>(out)[e] = f32_to_bf16_bits(r);
}

}  // namespace

template <int NPL, int GMAX>
static void launch_dd(const CacheArgs& a, dim3 grid, const void* q, float* partials, int splits, float qscale,
                      const int32_t* sel, const int32_t* sel_cnt, int sel_stride, cudaStream_t st)
{
    if (a.ref_bits == 4)
        decode_direct_kernel<NPL, GMAX, 4><<<grid, kWarps * 32, 0, st>>>(a, q, partials, splits, qscale, sel, sel_cnt,
                                                                         sel_stride);
    else
        decode_direct_kernel<NPL, GMAX, 16><<<grid, kWarps * 32, 0, st>>>(a, q, partials, splits, qscale, sel,
                                                                          sel_cnt, sel_stride);
}

cudaError_t launch_decode_direct(const CacheArgs& a, int splits, const void* q, float* partials, cudaStream_t st,
                                 const int32_t* sel, const int32_t* sel_cnt, int sel_stride)
{
    const dim3 grid(splits, a.n_units);
    const float qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(a.D)));
    if (a.D == 128) {
        if (a.G <= 8)
            launch_dd<4, 8>(a, grid, q, partials, splits, qscale, sel, sel_cnt, sel_stride, st);
        else
            launch_dd<4, 16>(a, grid, q, partials, splits, qscale, sel, sel_cnt, sel_stride, st);
    } else {
        if (a.G <= 8)
            launch_dd<2, 8>(a, grid, q, partials, splits, qscale, sel, sel_cnt, sel_stride, st);
        else
            launch_dd<2, 16>(a, grid, q, partials, splits, qscale, sel, sel_cnt, sel_stride, st);
    }
    return cudaGetLastError();
}

cudaError_t launch_decode_combine(const CacheArgs& a, int batch, int splits, const float* partials, void* out,
                                  cudaStream_t st)
{
    const dim3 grid(a.Hq, batch);
    if (a.D == 128)
        decode_combine_kernel<4><<<grid, 128, 0, st>>>(a, splits, partials, out);
    else
        decode_combine_kernel<2><<<grid, 64, 0, st>>>(a, splits, partials, out);
    return cudaGetLastError();
}

}  // namespace rkv
