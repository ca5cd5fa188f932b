// Decode attention over the compressed cache, with the reconstruction folded
// into the attention algebra (ResidualKV paper summary page, "Practical
// Deployment via Sparse-vLLM": fused gather + mean + residual add; news page,
// "How ResidualKV Works": tokens rebuilt on the fly when attention needs them).
//
// A compressed token i has K_i = mean_{j in S(i)} r_j + dK_i and V_i likewise,
// with |S(i)| = k_eff.  Attention over the rebuilt cache is, exactly,
//   logit_i = mean_{j in S(i)} s_j + q . dK_i           with s_j = q . refK_j
//   sum_i p_i V_i = sum_i p_i dV_i + sum_j w_j refV_j    with w_j = sum_{i: j in S(i)} p_i / k_eff
// (reference tokens contribute p_j to w_j).  So a step reads every reference row
// once (for s and for w.refV) and per compressed token only its codes, scales
// and reference ordinals, never the k reference rows of each token.
//
// One thread-block cluster of S CTAs per (sequence, kv-head) unit:
//   1. each CTA computes s for its slice of the references (in log2 units,
//      softmax scale folded in) and their maximum; the cluster agrees on
//      m = max_j s_j over distributed shared memory;
//   2. each CTA streams its share of the compressed tokens: eight lanes per
//      token, a lane owns D/8 channels; logits use the s of the token's
//      references read from the owning CTAs' shared memory; p = 2^(logit - m);
//      the lane accumulates p * scale * code into o, and w_j += p / k_eff goes
//      to the CTA's own w array with shared-memory atomics;
//   3. after a cluster barrier every CTA sums w over the cluster for its
//      reference slice, adds (p_j + w_j) refV_j for those references, and the
//      cluster sums the partial outputs; rank 0 normalises and writes them.
// All CTAs use the same m, so partial sums add without rescaling.  A logit more
// than 100 (log2 units) above m would overflow that scheme; it is reported as
// RKV_ERR_UNSUPPORTED instead of producing a wrong result.
#include <cooperative_groups.h>

#include <cfloat>
#include <cmath>

#include "device_common.cuh"
#include "launchers.h"

namespace cg = cooperative_groups;

namespace rkv {

namespace {

constexpr int kThreads = 256;
constexpr int kLPT = 8;                  // lanes per token
constexpr int kTokPerBlock = kThreads / kLPT;

// dynamic shared memory layout (floats): w [R][G] | s slice [slice][G] | q [G][D] | o [G][D] | l [G] | misc
struct FactLayout {
    int G, D, slice;
    int w_off, s_off, q_off, o_off, l_off, misc_off, total;
    // every region starts on a 16-byte boundary (float4 accesses)
    __host__ __device__ static int up4(int x) { return (x + 3) & ~3; }
    __host__ __device__ FactLayout(int G_, int D_, int R, int slice_) : G(G_), D(D_), slice(slice_)
    {
        w_off = 0;
        s_off = up4(w_off + R * G);
        q_off = up4(s_off + slice * G);
        o_off = up4(q_off + G * D);
        l_off = up4(o_off + G * D);
        misc_off = l_off + 16;
        total = misc_off + 16;
    }
};

__device__ __forceinline__ float tsum8(float v)
{
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    return v;
}

// Eight int4 codes (two's complement nibbles, lowest nibble first) to floats: the nibble
// with its sign bit flipped is the offset-binary value n + 8; placed in the low mantissa
// bits of 2^23 it reads as 2^23 + n + 8, and subtracting 2^23 + 8 leaves n exactly.
__device__ __forceinline__ void dequant8(uint32_t w, float* out)
{
    const uint32_t x = w ^ 0x88888888u;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        out[i] = __uint_as_float(0x4b000000u | ((x >> (4 * i)) & 0xfu)) - 8388616.0f;
}

// Dequantised codes of this lane's CPL channels (int4 two per byte, even channel low; int8).
template <int CPL>
__device__ __forceinline__ void load_codes(const uint8_t* row, int bits, int sub, float (&c)[CPL])
{
    if (bits == 8) {
        const uint8_t* p = row + sub * CPL;
#pragma unroll
        for (int h = 0; h < CPL / 8; ++h) {
            const uint2 w = *reinterpret_cast<const uint2*>(p + 8 * h);
            const uint32_t ww[2] = {w.x, w.y};
#pragma unroll
            for (int i = 0; i < 8; ++i)
                c[8 * h + i] = static_cast<float>(static_cast<int8_t>((ww[i / 4] >> (8 * (i % 4))) & 0xff));
        }
    } else {
        const uint8_t* p = row + sub * (CPL / 2);
#pragma unroll
        for (int h = 0; h < CPL / 8; ++h)
            dequant8(*reinterpret_cast<const uint32_t*>(p + 4 * h), &c[8 * h]);
    }
}

template <int CPL, int G>
__global__ void __launch_bounds__(kThreads, 2)
    decode_fact_kernel(const CacheArgs a, const void* __restrict__ q, void* __restrict__ out, float qscale)
{
    constexpr int D = CPL * kLPT;
    extern __shared__ float sm[];
    cg::cluster_group cluster = cg::this_cluster();
    const int S = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int u = blockIdx.y;
    const UnitMeta um = a.units[u];
    const int h = u - um.seq * a.Hkv;
    const int R = um.R;
    const int slice = (R + S - 1) / S;
    const FactLayout L(G, D, a.max_refs, slice);
    float* w = sm + L.w_off;
    float* s_sl = sm + L.s_off;
    float* qs = sm + L.q_off;
    float* osum = sm + L.o_off;
    float* lsum = sm + L.l_off;
    float* misc = sm + L.misc_off;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- prologue: q (log2-scaled), zero w / o / l -----------------------------------------
    for (int i = tid; i < G * D; i += kThreads) {
        const int g = i / D, c = i % D;
        const int64_t e = (static_cast<int64_t>(um.seq) * a.Hq + h * G + g) * D + c;
        qs[i] = (a.in_dtype == RKV_DTYPE_F32 ? static_cast<const float*>(q)[e]
                                             : bf16_bits_to_f32(static_cast<const uint16_t*>(q)[e])) * qscale;
        osum[i] = 0.0f;
    }
    for (int i = tid; i < R * G; i += kThreads)
        w[i] = 0.0f;
    if (tid < 16)
        lsum[tid] = 0.0f;
    __syncthreads();

    // ---- 1. reference scores of this CTA's slice, and their maximum ----------------------
    const int j_lo = rank * slice;
    const int j_hi = min(R, j_lo + slice);
    float mloc[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
        mloc[g] = -FLT_MAX;
    {
        // eight lanes per reference row
        const int grp = tid / kLPT, sub = tid % kLPT;
        for (int j = j_lo + grp; j - grp < j_hi; j += kTokPerBlock) {
            const bool ok = j < j_hi;
            float r[CPL];
            if (ok) {
                load_ref<CPL>(a, 0, um.ref_row + j, sub * CPL, r);
            } else {
#pragma unroll
                for (int i = 0; i < CPL; ++i)
                    r[i] = 0.0f;
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float d = 0.0f;
#pragma unroll
                for (int i = 0; i < CPL; ++i)
                    d = fmaf(qs[g * D + sub * CPL + i], r[i], d);
                d = tsum8(d);
                if (ok) {
                    if (sub == 0)
                        s_sl[(j - j_lo) * G + g] = d;
                    mloc[g] = fmaxf(mloc[g], d);
                }
            }
        }
    }
    // block max, then cluster max
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float v = mloc[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        mloc[g] = v;
    }
    __shared__ float wmax[kThreads / 32][G];
    if (lane == 0)
#pragma unroll
        for (int g = 0; g < G; ++g)
            wmax[warp][g] = mloc[g];
    __syncthreads();
    if (tid < G) {
        float v = -FLT_MAX;
        for (int i = 0; i < kThreads / 32; ++i)
            v = fmaxf(v, wmax[i][tid]);
        misc[tid] = v;                          // this CTA's slice maximum
    }
    cluster.sync();
    __shared__ float peer_max[16][G];
    if (tid < S * G)
        peer_max[tid / G][tid % G] = cluster.map_shared_rank(misc, tid / G)[tid % G];
    __syncthreads();
    float m[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float v = -FLT_MAX;
        for (int r2 = 0; r2 < S; ++r2)
            v = fmaxf(v, peer_max[r2][g]);
        m[g] = (v == -FLT_MAX) ? 0.0f : v;      // empty unit: any finite reference
    }

    // ---- 2. compressed tokens of this CTA ---------------------------------------------
    const int C = um.C;
    const int per = (C + S - 1) / S;
    const int c_lo = rank * per;
    const int c_hi = min(C, c_lo + per);
    const int tg = tid / kLPT;
    const int sub = tid % kLPT;
    const int k = a.k;
    float o[G][CPL];
    float l_acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        l_acc[g] = 0.0f;
#pragma unroll
        for (int i = 0; i < CPL; ++i)
            o[g][i] = 0.0f;
    }
    bool overflow = false;
    bool corrupt = false;
    constexpr int LPG = 32 / CPL;   // lanes per 32-channel scale group
    const float* qlane = qs + sub * CPL;
    // the next token's ordinal, codes and scales are fetched one iteration ahead
    auto fetch = [&](int cc, int& oi, uint4& ck, uint4& cv, uint16_t& sk, uint16_t& sv) {
        const bool act = cc < c_hi;
        const int64_t row = um.cmp_row + (act ? cc : c_lo);
        oi = (act && sub < k) ? a.idx[row * k + sub] : RKV_IDX_UNUSED;
        const int cb = CPL * a.bits / 8;   // code bytes of this lane: 8 (int4) or 16 (int8) at D = 128
        const uint8_t* pk = a.codes_K + row * a.code_bytes + sub * cb;
        const uint8_t* pv = a.codes_V + row * a.code_bytes + sub * cb;
        if (cb == 16) {
            ck = *reinterpret_cast<const uint4*>(pk);
            cv = *reinterpret_cast<const uint4*>(pv);
        } else if (cb == 8) {
            const uint2 x = *reinterpret_cast<const uint2*>(pk), y = *reinterpret_cast<const uint2*>(pv);
            ck = make_uint4(x.x, x.y, 0u, 0u);
            cv = make_uint4(y.x, y.y, 0u, 0u);
        } else {
            const uint32_t x = *reinterpret_cast<const uint32_t*>(pk), y = *reinterpret_cast<const uint32_t*>(pv);
            ck = make_uint4(x, 0u, 0u, 0u);
            cv = make_uint4(y, 0u, 0u, 0u);
        }
        sk = a.scale_K[row * a.n_groups + sub / LPG];
        sv = a.scale_V[row * a.n_groups + sub / LPG];
    };
    auto unpack = [&](const uint4& w4, float (&cf)[CPL]) {
        const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
        if (a.bits == 8) {
#pragma unroll
            for (int i = 0; i < CPL; ++i)
                cf[i] = static_cast<float>(static_cast<int8_t>((ww[i / 4] >> (8 * (i % 4))) & 0xff));
        } else {
#pragma unroll
            for (int h2 = 0; h2 < CPL / 8; ++h2)
                dequant8(ww[h2], &cf[8 * h2]);
        }
    };
    int n_oi = RKV_IDX_UNUSED;
    uint4 n_ck = make_uint4(0u, 0u, 0u, 0u), n_cv = n_ck;
    uint16_t n_sk = 0, n_sv = 0;
    if (c_lo < c_hi)   // (fetch reads row c_lo for slots past the range: it must exist)
        fetch(c_lo + tg, n_oi, n_ck, n_cv, n_sk, n_sv);
    for (int c0 = c_lo; c0 < c_hi; c0 += kTokPerBlock) {
        const int c = c0 + tg;
        const bool act = c < c_hi;
        const int o_idx = n_oi;
        const uint4 ckw = n_ck, cvw = n_cv;
        const float sk = __half2float(__ushort_as_half(n_sk));
        const float sv = __half2float(__ushort_as_half(n_sv));
        fetch(c + kTokPerBlock, n_oi, n_ck, n_cv, n_sk, n_sv);
        const bool has = act && o_idx != RKV_IDX_UNUSED;
        corrupt |= has && o_idx >= R;
        const bool use = has && o_idx < R;
        float sref[G];
        if (use) {
            const int owner = o_idx / slice;
            const float* sp = cluster.map_shared_rank(s_sl, owner) + (o_idx - owner * slice) * G;
            if constexpr (G == 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(sp);
                sref[0] = v4.x; sref[1] = v4.y; sref[2] = v4.z; sref[3] = v4.w;
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g)
                    sref[g] = sp[g];
            }
        } else {
#pragma unroll
            for (int g = 0; g < G; ++g)
                sref[g] = 0.0f;
        }
        const float keff = tsum8(use ? 1.0f : 0.0f);
        const float rk = 1.0f / fmaxf(keff, 1.0f);
        float cf[CPL];
        unpack(ckw, cf);
        float p[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float d = 0.0f;
#pragma unroll
            for (int i = 0; i < CPL; i += 4) {
                const float4 qv = *reinterpret_cast<const float4*>(qlane + g * D + i);
                d = fmaf(qv.x, cf[i], d);
                d = fmaf(qv.y, cf[i + 1], d);
                d = fmaf(qv.z, cf[i + 2], d);
                d = fmaf(qv.w, cf[i + 3], d);
            }
            const float logit = tsum8(fmaf(d, sk, sref[g] * rk));
            const float e = logit - m[g];
            overflow |= act && e > 100.0f;
            p[g] = (act && keff > 0.0f) ? exp2f(fminf(e, 100.0f)) : 0.0f;
            l_acc[g] += (sub == 0) ? p[g] : 0.0f;
        }
        unpack(cvw, cf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float ps = p[g] * sv;
#pragma unroll
            for (int i = 0; i < CPL; ++i)
                o[g][i] = fmaf(ps, cf[i], o[g][i]);
        }
        if (use) {
#pragma unroll
            for (int g = 0; g < G; ++g)
                atomicAdd(&w[o_idx * G + g], p[g] * rk);
        }
    }
    // reference tokens of this CTA's slice: p_j joins w_j
    for (int i = tid; i < (j_hi - j_lo) * G; i += kThreads) {
        const int g = i % G;
        const float pj = exp2f(s_sl[i] - m[g]);
        atomicAdd(&w[(j_lo + i / G) * G + g], pj);
        atomicAdd(&lsum[g], pj);
    }
    if (__any_sync(0xffffffffu, overflow))
        if (lane == 0)
            report(a.err, RKV_ERR_UNSUPPORTED);
    if (__any_sync(0xffffffffu, corrupt))
        if (lane == 0)
            report(a.err, RKV_ERR_CORRUPT);
    // block partial of o (sum over the token groups: first the four of a warp, then
    // shared-memory atomics from one group per warp) and l
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            float v = o[g][i];
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            if (lane < kLPT)
                atomicAdd(&osum[g * D + sub * CPL + i], v);
        }
        float lv = l_acc[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            lv += __shfl_xor_sync(0xffffffffu, lv, off);
        if (lane == 0)
            atomicAdd(&lsum[g], lv);
    }
    cluster.sync();

    // ---- 3. w over the cluster for this CTA's reference slice, times refV ----------------
    // (the slice's scores are no longer needed: its buffer takes the cluster-summed w)
    float* wt = s_sl;
    for (int i = tid; i < (j_hi - j_lo) * G; i += kThreads) {
        float part[16];
#pragma unroll
        for (int r2 = 0; r2 < 16; ++r2)
            part[r2] = (r2 < S) ? cluster.map_shared_rank(w, r2)[j_lo * G + i] : 0.0f;
        float v = 0.0f;
#pragma unroll
        for (int r2 = 0; r2 < 16; ++r2)
            v += part[r2];
        wt[i] = v;
    }
    __syncthreads();
    // sum_j w_j refV_j over the slice: thread (g, channel pair), eight rows in flight
    for (int i = tid; i < G * (D / 2); i += kThreads) {
        const int g = i / (D / 2), cp = (i % (D / 2)) * 2;
        float acc0 = 0.0f, acc1 = 0.0f;
        for (int j = j_lo; j < j_hi; j += 8) {
            float rv[8][2];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                rv[t][0] = rv[t][1] = 0.0f;
                if (j + t < j_hi)
                    load_ref<2>(a, 1, um.ref_row + j + t, cp, rv[t]);
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const float wj = (j + t < j_hi) ? wt[(j + t - j_lo) * G + g] : 0.0f;
                acc0 = fmaf(wj, rv[t][0], acc0);
                acc1 = fmaf(wj, rv[t][1], acc1);
            }
        }
        osum[g * D + cp] += acc0;
        osum[g * D + cp + 1] += acc1;
    }
    cluster.sync();
    // ---- combine the cluster's partial outputs (rank 0 writes) ---------------------------
    if (rank == 0) {
        for (int i = tid; i < G * D; i += kThreads) {
            const int g = i / D;
            float po[16], pl[16];
#pragma unroll
            for (int r2 = 0; r2 < 16; ++r2) {
                po[r2] = (r2 < S) ? cluster.map_shared_rank(osum, r2)[i] : 0.0f;
                pl[r2] = (r2 < S) ? cluster.map_shared_rank(lsum, r2)[g] : 0.0f;
            }
            float ov = 0.0f, lv = 0.0f;
#pragma unroll
            for (int r2 = 0; r2 < 16; ++r2) {
                ov += po[r2];
                lv += pl[r2];
            }
            const float res = (lv > 0.0f) ? ov / lv : 0.0f;
            const int64_t e = (static_cast<int64_t>(um.seq) * a.Hq + h * G + g) * D + (i % D);
            if (a.out_dtype == RKV_DTYPE_F32)
                static_cast<float*>(out)[e] = res;
            else
                static_cast<uint16_t*>(out)[e] = f32_to_bf16_bits(res);
        }
    }
    cluster.sync();   // peers' shared memory stays alive until rank 0 has read it
}

size_t fact_smem(const CacheArgs& a, int cluster)
{
    const int slice = (a.max_refs + cluster - 1) / cluster;
    const FactLayout L(a.G, a.D, a.max_refs, slice);
    return static_cast<size_t>(L.total) * sizeof(float);
}

template <int CPL, int G>
cudaError_t launch_g(const CacheArgs& a, int cluster, const void* q, void* out, float qscale, cudaStream_t st)
{
    auto kern = decode_fact_kernel<CPL, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess)
        return e;
    // the largest cluster size <= the requested one that fits shared memory and that the
    // device can place
    for (int cs = cluster; cs >= 1; cs /= 2) {
        const size_t smem = fact_smem(a, cs);
        if (smem > 220 * 1024)
            continue;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess)
            return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cs, a.n_units, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n_clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&n_clusters, kern, &cfg) != cudaSuccess || n_clusters < 1) {
            cudaGetLastError();
            continue;
        }
        return cudaLaunchKernelEx(&cfg, kern, a, q, out, qscale);
    }
    return cudaErrorNotSupported;
}

template <int CPL>
cudaError_t launch_cpl(const CacheArgs& a, int cluster, const void* q, void* out, float qscale, cudaStream_t st)
{
    switch (a.G) {
    case 1: return launch_g<CPL, 1>(a, cluster, q, out, qscale, st);
    case 2: return launch_g<CPL, 2>(a, cluster, q, out, qscale, st);
    case 4: return launch_g<CPL, 4>(a, cluster, q, out, qscale, st);
    case 7: return launch_g<CPL, 7>(a, cluster, q, out, qscale, st);
    case 8: return launch_g<CPL, 8>(a, cluster, q, out, qscale, st);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace

bool decode_fact_supported(const CacheArgs& a)
{
    if (!(a.G == 1 || a.G == 2 || a.G == 4 || a.G == 7 || a.G == 8))
        return false;
    return fact_smem(a, 16) <= 220 * 1024;
}

// Largest cluster size (power of two, <= 16) that the device can place, aimed at about one CTA
// per SM over all units.
int decode_fact_cluster(const CacheArgs& a, int sms)
{
    int want = 1;
    while (want < 16 && (want * 2) * a.n_units <= sms)
        want *= 2;
    return want;
}

cudaError_t launch_decode_fact(const CacheArgs& a, int cluster, const void* q, void* out, cudaStream_t st)
{
    const float qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(a.D)));
    return (a.D == 128) ? launch_cpl<16>(a, cluster, q, out, qscale, st)
                        : launch_cpl<8>(a, cluster, q, out, qscale, st);
}

}  // namespace rkv
