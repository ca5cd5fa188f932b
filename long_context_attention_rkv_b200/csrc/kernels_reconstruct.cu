// Reconstruction of selected rows (ResidualKV paper summary page, "DeltaKV
// Framework Architecture": KV = KV_delta + KV_R; "Training and Inference
// Integration": only the rows a step needs are decompressed).
//
// One warp per requested position; lanes own D/32 consecutive channels.
// Reference positions return the stored bf16 row.  Compressed positions return
// mean(references) + code * scale with the mean formed exactly as the encoder
// formed it (fp32, ascending ordinals, one division); with the learned-coder
// shapes, mean + Wd (code * scale) (the decompressor fd applied to the latent).
#include "device_common.cuh"
#include "launchers.h"

namespace rkv {

namespace {

constexpr int kWarps = 8;

template <int NPL>
__device__ __forceinline__ void store_row(void* out, int64_t elem, int dtype, const float (&v)[NPL])
{
    if (dtype == RKV_DTYPE_F32) {
        float* p = static_cast<float*>(out) + elem;
        if constexpr (NPL == 4)
            *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
        else
            *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
        uint16_t* p = static_cast<uint16_t*>(out) + elem;
        if constexpr (NPL == 4)
            *reinterpret_cast<uint2*>(p) = make_uint2(f32_to_bf16_bits(v[0]) | (uint32_t(f32_to_bf16_bits(v[1])) << 16),
                                                      f32_to_bf16_bits(v[2]) | (uint32_t(f32_to_bf16_bits(v[3])) << 16));
        else
            *reinterpret_cast<uint32_t*>(p) = f32_to_bf16_bits(v[0]) | (uint32_t(f32_to_bf16_bits(v[1])) << 16);
    }
}

template <int NPL>
__device__ __forceinline__ void dequant_add(const uint8_t* codes_row, const uint16_t* scale_row, int bits, int lane,
                                            float (&x)[NPL])
{
    constexpr int LPG = 32 / NPL;
    const float s = __half2float(__ushort_as_half(scale_row[lane / LPG]));
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int q = code_at(codes_row, bits, lane * NPL + i);
        x[i] = __fadd_rn(x[i], __fmul_rn(static_cast<float>(q), s));
    }
}

// Learned-coder shapes: x += Wd z_hat for this lane's channels, z_hat the dequantised latent
// codes (the lanes' parts exchanged by shuffles); Wd bf16 [D][D].
template <int NPL>
__device__ __forceinline__ void fd_add(const uint8_t* codes_row, const uint16_t* scale_row, int bits, int lane,
                                       const uint16_t* Wd, float (&x)[NPL])
{
    constexpr int D = NPL * 32;
    constexpr int LPG = 32 / NPL;
    const float s = __half2float(__ushort_as_half(scale_row[lane / LPG]));
    float z[NPL], acc[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        z[i] = __fmul_rn(static_cast<float>(code_at(codes_row, bits, lane * NPL + i)), s);
        acc[i] = 0.0f;
    }
    for (int src = 0; src < 32; ++src) {
#pragma unroll
        for (int e = 0; e < NPL; ++e) {
            const float zl = __shfl_sync(0xffffffffu, z[e], src);
            const int l = src * NPL + e;
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                acc[i] = fmaf(bf16_bits_to_f32(Wd[(lane * NPL + i) * D + l]), zl, acc[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        x[i] = __fadd_rn(x[i], acc[i]);
}

template <int NPL>
__global__ void __launch_bounds__(kWarps * 32) reconstruct_kernel(CacheArgs a, int unit,
                                                                  const int32_t* __restrict__ positions, int64_t n_pos,
                                                                  void* K_out, void* V_out, int out_dtype)
{
    constexpr int D = NPL * 32;
    const int lane = threadIdx.x & 31;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    if (i >= n_pos)
        return;
    const UnitMeta um = a.units[unit];
    const int p = positions ? positions[i] : static_cast<int>(i);
    if (p < 0 || p >= um.n) {
        if (lane == 0)
            report(a.err, RKV_ERR_INVALID_ARG);
        return;
    }
    const int nle = refs_upto(a.ph, p);
    float xk[NPL], xv[NPL];
    if (is_ref_pos(a.ph, p)) {
        load_ref<NPL>(a, 0, um.ref_row + nle - 1, lane * NPL, xk);
        load_ref<NPL>(a, 1, um.ref_row + nle - 1, lane * NPL, xv);
    } else {
        const int64_t row = um.cmp_row + (p - nle);
        const uint16_t* id = a.idx + row * a.k;
        int keff = 0;
        bool bad = false;
        for (int l = 0; l < a.k; ++l) {
            const int o = id[l];
            if (o == RKV_IDX_UNUSED)
                break;
            bad |= (o >= nle) || (l > 0 && o <= id[l - 1]);
            ++keff;
        }
        if (bad || keff == 0) {
            if (lane == 0)
                report(a.err, RKV_ERR_CORRUPT);
            return;
        }
        load_ref<NPL>(a, 0, um.ref_row + id[0], lane * NPL, xk);
        load_ref<NPL>(a, 1, um.ref_row + id[0], lane * NPL, xv);
        for (int l = 1; l < keff; ++l) {
            float rk[NPL], rv[NPL];
            load_ref<NPL>(a, 0, um.ref_row + id[l], lane * NPL, rk);
            load_ref<NPL>(a, 1, um.ref_row + id[l], lane * NPL, rv);
#pragma unroll
            for (int j = 0; j < NPL; ++j) {
                xk[j] = __fadd_rn(xk[j], rk[j]);
                xv[j] = __fadd_rn(xv[j], rv[j]);
            }
        }
        const float fk = static_cast<float>(keff);
#pragma unroll
        for (int j = 0; j < NPL; ++j) {
            xk[j] = __fdiv_rn(xk[j], fk);
            xv[j] = __fdiv_rn(xv[j], fk);
        }
        if (a.coder == 1) {
            fd_add<NPL>(a.codes_K + row * a.code_bytes, a.scale_K + row * a.n_groups, a.bits, lane, a.cw[3], xk);
            fd_add<NPL>(a.codes_V + row * a.code_bytes, a.scale_V + row * a.n_groups, a.bits, lane, a.cw[7], xv);
        } else {
            dequant_add<NPL>(a.codes_K + row * a.code_bytes, a.scale_K + row * a.n_groups, a.bits, lane, xk);
            dequant_add<NPL>(a.codes_V + row * a.code_bytes, a.scale_V + row * a.n_groups, a.bits, lane, xv);
        }
    }
    const int64_t o = i * D + lane * NPL;
    if (K_out)
        store_row<NPL>(K_out, o, out_dtype, xk);
    if (V_out)
        store_row<NPL>(V_out, o, out_dtype, xv);
}

}  // namespace

cudaError_t launch_reconstruct(const CacheArgs& a, int unit, const int32_t* positions, int64_t n_pos, void* K_out,
                               void* V_out, int out_dtype, cudaStream_t st)
{
    if (n_pos <= 0)
        return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((n_pos + kWarps - 1) / kWarps);
    if (a.D == 128)
        reconstruct_kernel<4><<<grid, kWarps * 32, 0, st>>>(a, unit, positions, n_pos, K_out, V_out, out_dtype);
    else
        reconstruct_kernel<2><<<grid, kWarps * 32, 0, st>>>(a, unit, positions, n_pos, K_out, V_out, out_dtype);
    return cudaGetLastError();
}

}  // namespace rkv
