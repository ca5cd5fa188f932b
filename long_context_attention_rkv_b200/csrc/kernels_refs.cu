// Reference store: copies the key/value rows at the reference positions of every
// unit into the cache as bf16 and records 0.5*|r|^2 of each key reference
// (ResidualKV paper summary page, "DeltaKV Framework Architecture": the
// reference set T is kept uncompressed), plus -|r|^2/2 as three bf16 terms for
// the augmented column of the tensor-core search.
//
// One warp per reference row; each lane moves D/32 consecutive channels, so a
// warp reads and writes one contiguous row (256 B for bf16, D = 128).
#include "device_common.cuh"
#include "launchers.h"

namespace rkv {

template <int NPL>
__global__ void __launch_bounds__(256) refs_copy_kernel(CacheArgs a, const void* __restrict__ K,
                                                        const void* __restrict__ V)
{
    const int u = blockIdx.y;
    const UnitMeta um = a.units[u];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.x * (blockDim.x >> 5) + warp;
    if (j >= um.R)
        return;
    const int p = ref_pos_of(a.ph, j);
    const int64_t e = (static_cast<int64_t>(u) * a.max_len + p) * a.D + lane * NPL;
    float kx[NPL], vx[NPL];
    load_row_part<NPL>(K, e, a.in_dtype, kx);
    load_row_part<NPL>(V, e, a.in_dtype, vx);
    uint16_t kb[NPL], vb[NPL];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        kb[i] = f32_to_bf16_bits(kx[i]);
        vb[i] = f32_to_bf16_bits(vx[i]);
        const float r = bf16_bits_to_f32(kb[i]);
        ss = fmaf(r, r, ss);
    }
    const int64_t o = (um.ref_row + j) * a.D + lane * NPL;
    if constexpr (NPL == 4) {
        *reinterpret_cast<uint2*>(a.ref_K + o) = make_uint2(kb[0] | (uint32_t(kb[1]) << 16), kb[2] | (uint32_t(kb[3]) << 16));
        *reinterpret_cast<uint2*>(a.ref_V + o) = make_uint2(vb[0] | (uint32_t(vb[1]) << 16), vb[2] | (uint32_t(vb[3]) << 16));
    } else {
        *reinterpret_cast<uint32_t*>(a.ref_K + o) = kb[0] | (uint32_t(kb[1]) << 16);
        *reinterpret_cast<uint32_t*>(a.ref_V + o) = vb[0] | (uint32_t(vb[1]) << 16);
    }
    ss = warp_sum(ss);
    if (lane == 0) {
        const float hn = 0.5f * ss;
        a.ref_hn[um.ref_row + j] = hn;
        a.ref_pos[um.ref_row + j] = p;
        // -hn split into three bf16 terms (hi + mid + lo = hn to ~2^-24 relative): a 16-wide
        // extra K block of the search GEMM adds them to every dot product
        const uint16_t hi = f32_to_bf16_bits(hn);
        const float r1 = hn - bf16_bits_to_f32(hi);
        const uint16_t mid = f32_to_bf16_bits(r1);
        const uint16_t lo = f32_to_bf16_bits(r1 - bf16_bits_to_f32(mid));
        uint4* aug = reinterpret_cast<uint4*>(a.ref_aug + (um.ref_row + j) * 16);
        aug[0] = make_uint4((hi ^ 0x8000u) | ((mid ^ 0x8000u) << 16), lo ^ 0x8000u, 0u, 0u);
        aug[1] = make_uint4(0u, 0u, 0u, 0u);
    }
}

cudaError_t launch_refs_copy(const CacheArgs& a, int max_R, const void* K, const void* V, cudaStream_t st)
{
    if (max_R <= 0)
        return cudaSuccess;
    const dim3 grid((max_R + 7) / 8, a.n_units);
    if (a.D == 128)
        refs_copy_kernel<4><<<grid, 256, 0, st>>>(a, K, V);
    else
        refs_copy_kernel<2><<<grid, 256, 0, st>>>(a, K, V);
    return cudaGetLastError();
}

}  // namespace rkv
