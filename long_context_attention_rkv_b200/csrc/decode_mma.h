// Shared pieces of the tensor-core decode (kernels_decode_mma.cu: reference scores,
// references and output; kernels_decode_tc.cu: the compressed tokens on tcgen05).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "rkv_internal.h"

namespace rkv {

constexpr int kRefChunk = 64;        // references per CTA of the scores and refs kernels

// Workspace carve-up of this decode (device pointers); see decode_mma_ws_bytes.
struct MmaWs {
    float* s_tab;     // [ref rows][Gp]  reference scores, log2 units
    float* W;         // [ref rows][Gp]  reference weights sum_i p_i / k_eff
    float* mpart;     // [units][n_chunk][Gp]  maxima of 64-reference chunks
    float* O;         // [units][Gp][D]  output numerators
    float* L;         // [units][Gp]     softmax denominators
    uint32_t* cnt;    // [units]         finished chunks of the refs kernel
    float* Olat;      // [units][Gp][D]  learned-coder shapes: latent output numerators
    uint16_t* qlat;   // [batch][Hq][D]  learned-coder shapes: Wd_K^T q (bf16)
    int n_chunk;
    int n_tiles;
    int n_cta;        // CTAs of the tokens kernel
    int ref_blk;      // 64-reference chunks per CTA of the refs kernel
    float cK;         // log2(e) / sqrt(D)
};

namespace decode_detail {

// Order-preserving map of floats to unsigned keys (0 is below every float) and back.
__device__ __forceinline__ uint32_t fkey(float f)
{
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float fkey_inv(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Common offset m of a unit's q-heads: the maximum reference score (0 for a unit without
// references).  All threads of the group load the chunk maxima in parallel and fold them
// into key[Gp] (shared, zeroed beforehand) with atomic maxima; read back with unit_m.
template <int Gp>
__device__ __forceinline__ void unit_max_fold(const MmaWs& w, int u, int R, int tid, int nthreads, uint32_t* key)
{
    // entry x holds head x % Gp: lanes 0 .. Gp-1 of each warp fold their lane classes
    const int n = ((R + kRefChunk - 1) / kRefChunk) * Gp;
    const float* src = w.mpart + static_cast<int64_t>(u) * w.n_chunk * Gp;
    for (int base = 0; base < n; base += nthreads) {
        const int x = base + tid;
        uint32_t k = (x < n) ? fkey(__ldcg(src + x)) : 0u;
#pragma unroll
        for (int o = Gp; o < 32; o <<= 1)
            k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
        if ((tid & 31) < Gp && k != 0u)
            atomicMax(&key[tid % Gp], k);
    }
}

__device__ __forceinline__ float unit_m(const uint32_t* key, int h)
{
    const uint32_t k = key[h];
    const float v = fkey_inv(k);
    return (k == 0u || v == -FLT_MAX) ? 0.0f : v;
}

}  // namespace decode_detail

// The compressed tokens of one decode step on the 5th-generation tensor cores (one thread per
// token, accumulators in TMEM).  q: the query (or q' for the learned-coder shapes) of the unit's
// heads; w.O receives the partial output sums (w.Olat for the learned-coder shapes: the caller
// passes the MmaWs with O pointing there).  Launched as a programmatic dependent of the scores
// kernel; its own dependents (the refs kernel) may start once every CTA has passed its wait.
cudaError_t launch_tokens_tc(const CacheArgs& a, const MmaWs& w, const void* q, int Gp, cudaStream_t st);

}  // namespace rkv
