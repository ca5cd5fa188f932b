// Device helpers shared by the librkv kernels: reference schedule arithmetic,
// element conversions, warp reductions and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rkv_internal.h"

namespace rkv {

// ---- reference schedule --------------------------------------------------------------
// The reference set T of a sequence (strided, or with a stride that doubles every
// refs_per_phase references) expressed by the phase table.

__device__ __forceinline__ int phase_of_pos(const Phases& ph, int p)
{
    int q = 0;
    for (int i = 1; i < ph.n; ++i)
        q = (p >= ph.start[i]) ? i : q;
    return q;
}

// Number of references at positions <= p.
__device__ __forceinline__ int refs_upto(const Phases& ph, int p)
{
    const int q = phase_of_pos(ph, p);
    return ph.first_ord[q] + (p - ph.start[q]) / ph.stride[q] + 1;
}

__device__ __forceinline__ bool is_ref_pos(const Phases& ph, int p)
{
    const int q = phase_of_pos(ph, p);
    return (p - ph.start[q]) % ph.stride[q] == 0;
}

// Position of the reference with ordinal j.
__device__ __forceinline__ int ref_pos_of(const Phases& ph, int j)
{
    int q = 0;
    for (int i = 1; i < ph.n; ++i)
        q = (j >= ph.first_ord[i]) ? i : q;
    return ph.start[q] + (j - ph.first_ord[q]) * ph.stride[q];
}

// Position of the c-th non-reference token (compressed slot c).
__device__ __forceinline__ int slot_pos(const Phases& ph, int c)
{
    int q = 0;
    for (int i = 1; i < ph.n; ++i)
        q = (c >= ph.first_slot[i]) ? i : q;
    const int local = c - ph.first_slot[q];
    const int per = ph.stride[q] - 1;
    return ph.start[q] + (local / per) * ph.stride[q] + local % per + 1;
}

// ---- conversions ---------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Loads n consecutive elements (n = 2 or 4) of a bf16 or fp32 row as floats.
template <int N>
__device__ __forceinline__ void load_row_part(const void* base, int64_t elem, int in_dtype, float* out)
{
    if (in_dtype == RKV_DTYPE_F32) {
        const float* p = static_cast<const float*>(base) + elem;
        if constexpr (N == 4) {
            const float4 v = *reinterpret_cast<const float4*>(p);
            out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2*>(p);
            out[0] = v.x; out[1] = v.y;
        }
    } else {
        const uint16_t* p = static_cast<const uint16_t*>(base) + elem;
        if constexpr (N == 4) {
            const uint2 v = *reinterpret_cast<const uint2*>(p);
            out[0] = bf16_bits_to_f32(v.x & 0xffffu); out[1] = bf16_bits_to_f32(v.x >> 16);
            out[2] = bf16_bits_to_f32(v.y & 0xffffu); out[3] = bf16_bits_to_f32(v.y >> 16);
        } else {
            const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
            out[0] = bf16_bits_to_f32(v & 0xffffu); out[1] = bf16_bits_to_f32(v >> 16);
        }
    }
}

// N consecutive bf16 values from a bf16 array.
template <int N>
__device__ __forceinline__ void load_bf16(const uint16_t* p, float* out)
{
    if constexpr (N == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        out[0] = bf16_bits_to_f32(v.x & 0xffffu); out[1] = bf16_bits_to_f32(v.x >> 16);
        out[2] = bf16_bits_to_f32(v.y & 0xffffu); out[3] = bf16_bits_to_f32(v.y >> 16);
    } else {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
        out[0] = bf16_bits_to_f32(v & 0xffffu); out[1] = bf16_bits_to_f32(v >> 16);
    }
}

// Signed code of channel c from a packed row (int8: byte c; int4: nibble c, even channel low).
__device__ __forceinline__ int code_at(const uint8_t* row, int bits, int c)
{
    if (bits == 8)
        return static_cast<int8_t>(row[c]);
    const int b = row[c >> 1];
    const int nib = (c & 1) ? (b >> 4) : (b & 0xf);
    return (nib ^ 8) - 8;
}

// ---- warp reductions -----------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ---- device error word ---------------------------------------------------------------

__device__ __forceinline__ void report(int32_t* err, int code)
{
    atomicCAS(err, 0, code);
}

}  // namespace rkv
