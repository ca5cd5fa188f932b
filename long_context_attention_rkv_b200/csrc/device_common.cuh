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

// n / d with the multiplier and shift the host prepared (div_magic); 0 <= n < 2^31.
__device__ __forceinline__ int div_by(int n, uint64_t m, int sh)
{
    return static_cast<int>((static_cast<uint64_t>(static_cast<uint32_t>(n)) * m) >> sh);
}

// Number of references at positions <= p.
__device__ __forceinline__ int refs_upto(const Phases& ph, int p)
{
    const int q = phase_of_pos(ph, p);
    return ph.first_ord[q] + div_by(p - ph.start[q], ph.m_stride[q], ph.sh_stride[q]) + 1;
}

__device__ __forceinline__ bool is_ref_pos(const Phases& ph, int p)
{
    const int q = phase_of_pos(ph, p);
    const int o = p - ph.start[q];
    return o - div_by(o, ph.m_stride[q], ph.sh_stride[q]) * ph.stride[q] == 0;
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
    const int blk = div_by(local, ph.m_per[q], ph.sh_per[q]);
    return ph.start[q] + blk * ph.stride[q] + (local - blk * per) + 1;
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

// ---- reference rows ---------------------------------------------------------------------
// Stored values of N consecutive channels c0 .. c0 + N - 1 (c0 a multiple of N, N in {2, 4,
// 8, 16}) of reference row `row`: bf16 rows widened, or with the int4 reference store
// code * scale (exact in fp32: a 4-bit code times a binary16 value).  Side 0 = K, 1 = V.
// RB: the store's width when known at compile time (16 or 4), 0 to read it from a.
template <int N, int RB = 0>
__device__ __forceinline__ void load_ref(const CacheArgs& a, int side, int64_t row, int c0, float* out)
{
    const uint16_t* base = side ? a.ref_V : a.ref_K;
    if (RB == 4 || (RB == 0 && a.ref_bits == 4)) {
        const uint8_t* p = reinterpret_cast<const uint8_t*>(base) + row * (a.D / 2) + c0 / 2;
        const uint16_t sb = (side ? a.ref_sV : a.ref_sK)[row * (a.D / 32) + c0 / 32];
        const float s = __half2float(__ushort_as_half(sb));
        uint32_t w[(N + 7) / 8];
        if constexpr (N == 16) {
            const uint2 v = *reinterpret_cast<const uint2*>(p);
            w[0] = v.x;
            w[1] = v.y;
        } else if constexpr (N == 8) {
            w[0] = *reinterpret_cast<const uint32_t*>(p);
        } else if constexpr (N == 4) {
            w[0] = *reinterpret_cast<const uint16_t*>(p);
        } else {
            w[0] = *p;
        }
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int q = static_cast<int>(((w[i >> 3] >> (4 * (i & 7))) & 0xfu) ^ 8u) - 8;
            out[i] = __fmul_rn(static_cast<float>(q), s);
        }
    } else {
        const uint16_t* p = base + row * a.D + c0;
        if constexpr (N >= 8) {
#pragma unroll
            for (int h = 0; h < N; h += 8) {
                const uint4 v = *reinterpret_cast<const uint4*>(p + h);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    out[h + 2 * i] = bf16_bits_to_f32(w[i] & 0xffffu);
                    out[h + 2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
                }
            }
        } else {
            load_bf16<N>(p, out);
        }
    }
}

// The int4 reference store's quantiser (the residuals' group quantiser applied to the row
// itself, with the scale rounded up to a power of two so that every stored value is an
// exact bf16 number): this lane holds channels lane * NPL .. lane * NPL + NPL - 1 of a row
// (NPL = D / 32, so 32 / NPL lanes share a 32-channel group).  Per group a = max|x|; scale =
// the smallest power of two >= fl(a / 7) within binary16's 2^-24 .. 2^15 (0 when a == 0),
// code = clamp(rint(x / scale), -7, 7).  Stores the lane's codes (two per byte, even channel
// low) and, from the group's first lane, the scale as binary16; r gets code * scale.
template <int NPL>
__device__ __forceinline__ void ref_quantise_store(const float (&x)[NPL], int lane, uint8_t* codes_row,
                                                   uint16_t* scale_row, float (&r)[NPL], int32_t* err)
{
    constexpr int LPG = 32 / NPL;
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    uint16_t sbits = 0;
    float s = 0.0f;
    if (amax > 0.0f) {
        const float v = __fdiv_rn(amax, 7.0f);
        float p2 = __uint_as_float(__float_as_uint(v) & 0x7f800000u);   // 2^floor(log2 v); 0 if subnormal
        p2 = (p2 < v) ? 2.0f * p2 : p2;
        s = fmaxf(p2, 0x1p-24f);
        sbits = __half_as_ushort(__float2half_rn(s));                    // exact up to 2^15
        if (s > 0x1p15f) {
            sbits = 0x7c00u;
            report(err, RKV_ERR_UNSUPPORTED);
        }
    }
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int c = (amax > 0.0f) ? max(-7, min(7, static_cast<int>(rintf(__fdiv_rn(x[i], s))))) : 0;
        r[i] = __fmul_rn(static_cast<float>(c), s);
        packed |= static_cast<uint32_t>(c & 0xf) << (4 * i);
    }
    if constexpr (NPL == 4)
        *reinterpret_cast<uint16_t*>(codes_row + lane * 2) = static_cast<uint16_t>(packed);
    else
        codes_row[lane] = static_cast<uint8_t>(packed);
    if (lane % LPG == 0)
        scale_row[lane / LPG] = sbits;
}

}  // namespace rkv
