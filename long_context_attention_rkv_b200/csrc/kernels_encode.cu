// Residual encoder (ResidualKV paper summary page, "DeltaKV Framework
// Architecture": top-k nearest references, mean reference KV_R, residual
// KV - KV_R; news page "New KV Cache Compression Method Cuts Long-Context
// Inference Costs by 85%", "How ResidualKV Works": quantized residual codes).
//
// One warp per compressed token; each lane owns D/32 consecutive channels.
//  1. Final top-k.  The search handed over its kc best candidates by
//     t = k.r - |r|^2/2 computed with fp32 accumulation.  Every candidate
//     whose t is within 2*delta of the k-th (delta = 2^-13 (|k|^2 + max|r|^2),
//     far above the accumulation error of a 128-term dot product) is re-ranked
//     by its exact-order fp32 distance sum_c (k_c - r_c)^2, ties to the lower
//     ordinal.  If even the last kept candidate is that close, the list may be
//     incomplete and the warp rescans every candidate exactly.
//  2. Mean of the chosen rows in ascending ordinal order (fp32, left to right)
//     and one IEEE division by k_eff; residual = x - mean (fp32).
//  3. Per 32-channel group: a = max|residual|, scale = binary16 rounded up from
//     a / qmax, code = round-half-even(residual / scale).  All of step 2-3 use
//     correctly rounded fp32 operations with no contraction, so codes match an
//     IEEE fp32 evaluation of the same steps bit for bit.
#include <cfloat>

#include "device_common.cuh"
#include "launchers.h"

namespace rkv {

namespace {

constexpr int kWarps = 8;

template <int NPL>
__device__ __forceinline__ float partial_dist(const float (&x)[NPL], const uint16_t* r)
{
    float rv[NPL];
    load_bf16<NPL>(r, rv);
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const float d = __fsub_rn(x[i], rv[i]);
        s = __fmaf_rn(d, d, s);
    }
    return s;
}

// Exhaustive exact top-k over candidates [0, ncand) for one warp.  The key row is
// staged in xs (shared, D floats).  Afterwards lanes 0..keff-1 hold the chosen ordinals.
template <int NPL>
__device__ void exhaustive_topk(const CacheArgs& a, const UnitMeta& um, const float* xs, int ncand, int k, int lane,
                                int& my_ord)
{
    constexpr int D = NPL * 32;
    float bd[RKV_MAX_K];
    int bo[RKV_MAX_K];
#pragma unroll
    for (int s = 0; s < RKV_MAX_K; ++s) {
        bd[s] = FLT_MAX;
        bo[s] = 0x7fffffff;
    }
    for (int j = lane; j < ncand; j += 32) {
        const uint16_t* r = a.ref_K + (um.ref_row + j) * D;
        float d = 0.0f;
        for (int c = 0; c < D; c += 2) {
            float rv[2];
            load_bf16<2>(r + c, rv);
            const float e0 = __fsub_rn(xs[c], rv[0]);
            const float e1 = __fsub_rn(xs[c + 1], rv[1]);
            d = __fmaf_rn(e0, e0, d);
            d = __fmaf_rn(e1, e1, d);
        }
        // insert by (d ascending, ordinal ascending) into the first k slots
        float cv = d;
        int ci = j;
#pragma unroll
        for (int s = 0; s < RKV_MAX_K; ++s) {
            if (s < k) {
                const bool before = (cv < bd[s]) || (cv == bd[s] && ci < bo[s]);
                const float fd = bd[s];
                const int fo = bo[s];
                bd[s] = before ? cv : fd;
                bo[s] = before ? ci : fo;
                cv = before ? fd : cv;
                ci = before ? fo : ci;
            }
        }
    }
    // merge the 32 per-lane lists: k rounds of a warp-wide (d, ordinal) minimum
    int head = 0;
    my_ord = RKV_IDX_UNUSED;
    for (int r = 0; r < k && r < ncand; ++r) {
        float hd = FLT_MAX;
        int ho = 0x7fffffff;
#pragma unroll
        for (int s = 0; s < RKV_MAX_K; ++s)
            if (s == head) {
                hd = bd[s];
                ho = bo[s];
            }
        float wd = hd;
        int wo = ho;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float od = __shfl_xor_sync(0xffffffffu, wd, off);
            const int oo = __shfl_xor_sync(0xffffffffu, wo, off);
            if (od < wd || (od == wd && oo < wo)) {
                wd = od;
                wo = oo;
            }
        }
        if (ho == wo && hd == wd)
            ++head;
        if (lane == r)
            my_ord = wo;
    }
}

template <int NPL>
__device__ __forceinline__ void quantise_store(const float (&x)[NPL], const float (&m)[NPL], int bits, int lane,
                                               uint8_t* codes_row, uint16_t* scale_row, int32_t* err)
{
    constexpr int LPG = 32 / NPL;  // lanes per 32-channel group
    const int qmax = (bits == 8) ? 127 : 7;
    float d[NPL];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        d[i] = __fsub_rn(x[i], m[i]);
        amax = fmaxf(amax, fabsf(d[i]));
    }
#pragma unroll
    for (int off = 1; off < LPG; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    uint16_t sbits = 0;
    float s = 0.0f;
    if (amax > 0.0f) {
        const __half h = __float2half_ru(__fdiv_rn(amax, static_cast<float>(qmax)));
        sbits = __half_as_ushort(h);
        s = __half2float(h);
        if ((sbits & 0x7c00u) == 0x7c00u)
            report(err, RKV_ERR_UNSUPPORTED);
    }
    int q[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        int c = 0;
        if (amax > 0.0f) {
            c = static_cast<int>(rintf(__fdiv_rn(d[i], s)));
            c = max(-qmax, min(qmax, c));
        }
        q[i] = c;
    }
    if (bits == 8) {
        if constexpr (NPL == 4) {
            const uint32_t w = (q[0] & 0xff) | ((q[1] & 0xff) << 8) | ((q[2] & 0xff) << 16) | (uint32_t(q[3] & 0xff) << 24);
            reinterpret_cast<uint32_t*>(codes_row)[lane] = w;
        } else {
            const uint16_t w = static_cast<uint16_t>((q[0] & 0xff) | ((q[1] & 0xff) << 8));
            reinterpret_cast<uint16_t*>(codes_row)[lane] = w;
        }
    } else {
        if constexpr (NPL == 4) {
            const uint16_t w = static_cast<uint16_t>((q[0] & 0xf) | ((q[1] & 0xf) << 4) | ((q[2] & 0xf) << 8) | ((q[3] & 0xf) << 12));
            reinterpret_cast<uint16_t*>(codes_row)[lane] = w;
        } else {
            codes_row[lane] = static_cast<uint8_t>((q[0] & 0xf) | ((q[1] & 0xf) << 4));
        }
    }
    if ((lane % LPG) == 0)
        scale_row[lane / LPG] = sbits;
}

template <int NPL, int KC>
__global__ void __launch_bounds__(kWarps * 32) encode_kernel(CacheArgs a, const void* __restrict__ K,
                                                             const void* __restrict__ V,
                                                             const uint16_t* __restrict__ cand_idx,
                                                             const float* __restrict__ cand_t)
{
    constexpr int D = NPL * 32;
    __shared__ float xs[kWarps][D];
    __shared__ int sorted[kWarps][RKV_MAX_K];

    const int u = blockIdx.y;
    const UnitMeta um = a.units[u];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int c = blockIdx.x * kWarps + warp;
    if (c >= um.C)
        return;
    const int k = a.k;
    const int p = slot_pos(a.ph, c);
    const int ncand = min(refs_upto(a.ph, p), um.R);
    const int64_t row = um.cmp_row + c;
    const int64_t e = (static_cast<int64_t>(u) * a.max_len + p) * D + lane * NPL;
    float xk[NPL], xv[NPL];
    load_row_part<NPL>(K, e, a.in_dtype, xk);
    load_row_part<NPL>(V, e, a.in_dtype, xv);

    // ---- 1. final top-k -------------------------------------------------------------
    const int nvalid = min(KC, ncand);
    int my_ord = RKV_IDX_UNUSED;
    float my_t = -FLT_MAX;
    if (lane < nvalid) {
        my_ord = cand_idx[row * KC + lane];
        my_t = cand_t[row * KC + lane];
    }
    const bool bad = (lane < nvalid) && (my_ord >= ncand);
    if (__any_sync(0xffffffffu, bad)) {
        if (lane == 0)
            report(a.err, RKV_ERR_CORRUPT);
        return;
    }
    bool chosen = false;
    int keff = min(k, nvalid);
    if (nvalid <= k) {
        chosen = lane < nvalid;
    } else {
        float xx = 0.0f;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            xx = fmaf(xk[i], xk[i], xx);
        xx = warp_sum(xx);
        const float hmax = warp_max(lane < nvalid ? a.ref_hn[um.ref_row + my_ord] : 0.0f);
        const float delta = ldexpf(xx + 2.0f * hmax, -13);
        const float tk = __shfl_sync(0xffffffffu, my_t, k - 1);
        const float tlast = __shfl_sync(0xffffffffu, my_t, KC - 1);
        const bool incomplete = (nvalid == KC) && (ncand > KC) && (tlast >= tk - 2.0f * delta);
        if (incomplete) {
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                xs[warp][lane * NPL + i] = xk[i];
            __syncwarp();
            exhaustive_topk<NPL>(a, um, xs[warp], ncand, k, lane, my_ord);
            chosen = lane < keff;
        } else {
            const bool inset = (lane < nvalid) && (lane < k || my_t >= tk - 2.0f * delta);
            const unsigned set = __ballot_sync(0xffffffffu, inset);
            float my_d = FLT_MAX;
            for (unsigned m = set; m; m &= m - 1) {
                const int l = __ffs(m) - 1;
                const int o = __shfl_sync(0xffffffffu, my_ord, l);
                const float d = warp_sum(partial_dist<NPL>(xk, a.ref_K + (um.ref_row + o) * D + lane * NPL));
                if (lane == l)
                    my_d = d;
            }
            int rank = 0;
            for (unsigned m = set; m; m &= m - 1) {
                const int l = __ffs(m) - 1;
                const float d = __shfl_sync(0xffffffffu, my_d, l);
                const int o = __shfl_sync(0xffffffffu, my_ord, l);
                rank += (d < my_d || (d == my_d && o < my_ord)) ? 1 : 0;
            }
            chosen = inset && rank < k;
        }
    }
    // ascending ordinal order of the chosen set
    const unsigned cm = __ballot_sync(0xffffffffu, chosen);
    int pos = 0;
    for (unsigned m = cm; m; m &= m - 1) {
        const int l = __ffs(m) - 1;
        const int o = __shfl_sync(0xffffffffu, my_ord, l);
        pos += (o < my_ord) ? 1 : 0;
    }
    if (chosen)
        sorted[warp][pos] = my_ord;
    __syncwarp();
    if (lane < k)
        a.idx[row * k + lane] = (lane < keff) ? static_cast<uint16_t>(sorted[warp][lane])
                                              : static_cast<uint16_t>(RKV_IDX_UNUSED);

    // ---- 2. mean reference (fp32, ascending ordinals, one division) -------------------
    float mk[NPL], mv[NPL];
    {
        const int o = sorted[warp][0];
        load_bf16<NPL>(a.ref_K + (um.ref_row + o) * D + lane * NPL, mk);
        load_bf16<NPL>(a.ref_V + (um.ref_row + o) * D + lane * NPL, mv);
    }
    for (int i = 1; i < keff; ++i) {
        const int o = sorted[warp][i];
        float rk[NPL], rv[NPL];
        load_bf16<NPL>(a.ref_K + (um.ref_row + o) * D + lane * NPL, rk);
        load_bf16<NPL>(a.ref_V + (um.ref_row + o) * D + lane * NPL, rv);
#pragma unroll
        for (int j = 0; j < NPL; ++j) {
            mk[j] = __fadd_rn(mk[j], rk[j]);
            mv[j] = __fadd_rn(mv[j], rv[j]);
        }
    }
    const float fk = static_cast<float>(keff);
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        mk[j] = __fdiv_rn(mk[j], fk);
        mv[j] = __fdiv_rn(mv[j], fk);
    }

    // ---- 3. residual and group quantiser ---------------------------------------------
    quantise_store<NPL>(xk, mk, a.bits, lane, a.codes_K + row * a.code_bytes, a.scale_K + row * a.n_groups, a.err);
    quantise_store<NPL>(xv, mv, a.bits, lane, a.codes_V + row * a.code_bytes, a.scale_V + row * a.n_groups, a.err);
}

template <int NPL>
cudaError_t launch_npl(const CacheArgs& a, int max_C, const void* K, const void* V, const uint16_t* ci,
                       const float* ct, cudaStream_t st)
{
    const dim3 grid((max_C + kWarps - 1) / kWarps, a.n_units);
    switch (a.kc) {
    case 8: encode_kernel<NPL, 8><<<grid, kWarps * 32, 0, st>>>(a, K, V, ci, ct); break;
    case 12: encode_kernel<NPL, 12><<<grid, kWarps * 32, 0, st>>>(a, K, V, ci, ct); break;
    default: encode_kernel<NPL, 20><<<grid, kWarps * 32, 0, st>>>(a, K, V, ci, ct); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode(const CacheArgs& a, int max_C, const void* K, const void* V, const uint16_t* cand_idx,
                          const float* cand_t, cudaStream_t st)
{
    if (max_C <= 0)
        return cudaSuccess;
    return (a.D == 128) ? launch_npl<4>(a, max_C, K, V, cand_idx, cand_t, st)
                        : launch_npl<2>(a, max_C, K, V, cand_idx, cand_t, st);
}

}  // namespace rkv
