// Reference store: copies the key/value rows at the reference positions of every
// unit into the cache as bf16 and records 0.5*|r|^2 of each key reference
// (ResidualKV paper summary page, "DeltaKV Framework Architecture": the
// reference set T is kept uncompressed), plus -|r|^2/2 as three bf16 terms for
// the augmented column of the tensor-core search.  With the int4 reference store
// (paper summary page, "Improvements for AI systems": 4-bit quantization of the
// uncompressed components too) the rows are stored as int4 codes with one binary16
// scale per 32 channels instead, and the half norm is that of the stored values.
//
// One warp per reference row; each lane moves D/32 consecutive channels, so a
// warp reads and writes one contiguous row (256 B for bf16, D = 128).
#include "device_common.cuh"
#include "launchers.h"

namespace rkv {

// Stores reference row j of unit u (this warp; lane owns D/32 channels) and returns its half
// norm (the same value in every lane).
template <int NPL, int RB>
__device__ __forceinline__ float copy_ref_row(const CacheArgs& a, const UnitMeta& um, int u, int j, int lane,
                                              const void* __restrict__ K, const void* __restrict__ V)
{
    const int p = ref_pos_of(a.ph, j);
    const int64_t e = (static_cast<int64_t>(u) * a.max_len + p) * a.D + lane * NPL;
    float kx[NPL], vx[NPL];
    load_row_part<NPL>(K, e, a.in_dtype, kx);
    load_row_part<NPL>(V, e, a.in_dtype, vx);
    float ss = 0.0f;
    const int64_t row = um.ref_row + j;
    if constexpr (RB == 4) {
        // int4 reference store: codes and scales; the half norm is of the stored values
        float rk[NPL], rv[NPL];
        uint8_t* cK = reinterpret_cast<uint8_t*>(a.ref_K) + row * (a.D / 2);
        uint8_t* cV = reinterpret_cast<uint8_t*>(a.ref_V) + row * (a.D / 2);
        ref_quantise_store<NPL>(kx, lane, cK, a.ref_sK + row * (a.D / 32), rk, a.err);
        ref_quantise_store<NPL>(vx, lane, cV, a.ref_sV + row * (a.D / 32), rv, a.err);
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            ss = fmaf(rk[i], rk[i], ss);
    } else {
        uint16_t kb[NPL], vb[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            kb[i] = f32_to_bf16_bits(kx[i]);
            vb[i] = f32_to_bf16_bits(vx[i]);
            const float r = bf16_bits_to_f32(kb[i]);
            ss = fmaf(r, r, ss);
        }
        const int64_t o = row * a.D + lane * NPL;
        if constexpr (NPL == 4) {
            *reinterpret_cast<uint2*>(a.ref_K + o) = make_uint2(kb[0] | (uint32_t(kb[1]) << 16), kb[2] | (uint32_t(kb[3]) << 16));
            *reinterpret_cast<uint2*>(a.ref_V + o) = make_uint2(vb[0] | (uint32_t(vb[1]) << 16), vb[2] | (uint32_t(vb[3]) << 16));
        } else {
            *reinterpret_cast<uint32_t*>(a.ref_K + o) = kb[0] | (uint32_t(kb[1]) << 16);
            *reinterpret_cast<uint32_t*>(a.ref_V + o) = vb[0] | (uint32_t(vb[1]) << 16);
        }
    }
    ss = warp_sum(ss);
    const float hn = 0.5f * ss;
    if (lane == 0) {
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
    return hn;
}

template <int NPL, int RB>
__global__ void __launch_bounds__(256) refs_copy_kernel(CacheArgs a, const void* __restrict__ K,
                                                        const void* __restrict__ V)
{
    const int u = blockIdx.y;
    const UnitMeta um = a.units[u];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.x * (blockDim.x >> 5) + warp;
    __shared__ int hmax[8];   // the warps' half norms (non-negative floats order as ints)
    hmax[warp] = 0;
    if (j < um.R) {
        const float hn = copy_ref_row<NPL, RB>(a, um, u, j, lane, K, V);
        if (lane == 0)
            hmax[warp] = __float_as_int(hn);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int m = 0;
        for (int i = 0; i < 8; ++i)
            m = max(m, hmax[i]);
        if (m > 0)
            atomicMax(reinterpret_cast<int*>(a.ref_hn_max + u), m);
    }
}

// The tensor-core search's B operand with the int4 reference store: the stored key values as
// bf16 rows (exact: a 4-bit code times a power-of-two scale).  One thread per 8 channels.
__global__ void __launch_bounds__(256) refs_bf16_kernel(CacheArgs a, int64_t rows, uint16_t* __restrict__ out)
{
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int per_row = a.D / 8;
    if (i >= rows * per_row)
        return;
    const int64_t row = i / per_row;
    const int c0 = static_cast<int>(i % per_row) * 8;
    float v[8];
    load_ref<8>(a, 0, row, c0, v);
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h)
        w[h] = f32_to_bf16_bits(v[2 * h]) | (static_cast<uint32_t>(f32_to_bf16_bits(v[2 * h + 1])) << 16);
    *reinterpret_cast<uint4*>(out + row * a.D + c0) = make_uint4(w[0], w[1], w[2], w[3]);
}

cudaError_t launch_refs_bf16(const CacheArgs& a, int64_t rows, uint16_t* out, cudaStream_t st)
{
    const int64_t n = rows * (a.D / 8);
    if (n <= 0)
        return cudaSuccess;
    refs_bf16_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(a, rows, out);
    return cudaGetLastError();
}

cudaError_t launch_refs_copy(const CacheArgs& a, int max_R, const void* K, const void* V, cudaStream_t st)
{
    if (max_R <= 0)
        return cudaSuccess;
    const dim3 grid((max_R + 7) / 8, a.n_units);
    const bool r4 = a.ref_bits == 4;
    if (a.D == 128)
        r4 ? refs_copy_kernel<4, 4><<<grid, 256, 0, st>>>(a, K, V) : refs_copy_kernel<4, 16><<<grid, 256, 0, st>>>(a, K, V);
    else
        r4 ? refs_copy_kernel<2, 4><<<grid, 256, 0, st>>>(a, K, V) : refs_copy_kernel<2, 16><<<grid, 256, 0, st>>>(a, K, V);
    return cudaGetLastError();
}

}  // namespace rkv
