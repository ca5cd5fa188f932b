// Host-side launchers of the librkv kernels (one translation unit each).
#pragma once

#include <cuda_runtime.h>

#include "rkv_internal.h"

namespace rkv {

cudaError_t launch_refs_bf16(const CacheArgs& a, int64_t rows, uint16_t* out, cudaStream_t st);
cudaError_t launch_refs_copy(const CacheArgs& a, int max_R, const void* K, const void* V, cudaStream_t st);

cudaError_t launch_select_simt(const CacheArgs& a, const Tile* tiles, int n_tiles, const void* K, uint16_t* cand_idx,
                               float* cand_t, cudaStream_t st);

// Tensor-core search (bf16 inputs, head_dim 64 or 128).
bool select_tc_supported(const CacheArgs& a);
cudaError_t launch_select_tc(const CacheArgs& a, const Tile* items, int n_items, const void* K, const uint16_t* refB,
                             int64_t in_rows, int64_t ref_rows, uint16_t* cand_idx, float* cand_t, cudaStream_t st);

// Final top-k, mean and quantiser of every compressed token.  fix: device scratch of
// 2 + 2 * fix_cap ints (fix_cap >= the compressed tokens of the layer) for the tokens the main
// pass defers to the exact passes.  The rescan of the tokens whose candidate list may be
// incomplete rewrites their lists in cand_idx / cand_t.
cudaError_t launch_encode(const CacheArgs& a, int max_C, const void* K, const void* V, uint16_t* cand_idx,
                          float* cand_t, int* fix, int fix_cap, cudaStream_t st);

// Incremental compression: one new token ([unit][D] rows) for every unit of the sequences whose
// bit is set in active (256 bits).
// Scratch that rkv_append needs inside the cache buffer (per-unit candidate lists).
uint64_t append_scratch_bytes(int n_units);
// Learned-coder shapes: latent residual codes z = fc(x) - fc(mean) of every compressed token
// (after launch_encode has chosen the references), both sides, on the tcgen05 tensor cores in
// 128-token tiles: total_tiles = the sum over units of encode_latent_tiles(compressed tokens).
// flist: device scratch of encode_latent_list_bytes(compressed rows of the layer): the groups
// the fast pass leaves to the exact pass (at most 8 per compressed row).
int encode_latent_tiles(int C);
uint64_t encode_latent_list_bytes(int64_t cmp_rows);
cudaError_t launch_encode_latent(const CacheArgs& a, const void* K, const void* V, int total_tiles, int* flist,
                                 cudaStream_t st);
cudaError_t launch_append(const CacheArgs& a, const void* K_new, const void* V_new, const uint32_t (&active)[8],
                          void* scratch, cudaStream_t st);

cudaError_t launch_reconstruct(const CacheArgs& a, int unit, const int32_t* positions, int64_t n_pos, void* K_out,
                               void* V_out, int out_dtype, cudaStream_t st);

// Literal decode: per token gather + mean of the reference rows, dequantise, add, attend.
// With sel (device [n_units][sel_stride] positions, sel_cnt [n_units] counts) only the listed
// positions are attended to.
cudaError_t launch_decode_direct(const CacheArgs& a, int splits, const void* q, float* partials, cudaStream_t st,
                                 const int32_t* sel = nullptr, const int32_t* sel_cnt = nullptr,
                                 int sel_stride = 0);

// Factorised decode (reference scores + scattered reference weights), one cluster per unit.
bool decode_fact_supported(const CacheArgs& a);
int decode_fact_cluster(const CacheArgs& a, int sms);
cudaError_t launch_decode_fact(const CacheArgs& a, int cluster, const void* q, void* out, cudaStream_t st);

// Factorised decode with the per-token contractions on the tensor cores (bf16 inputs,
// head_dim 128, int4 codes): scores, tokens and references kernels.
bool decode_mma_supported(const CacheArgs& a);
uint64_t decode_mma_ws_bytes(const CacheArgs& a, int64_t ref_rows);
cudaError_t launch_decode_mma(const CacheArgs& a, int64_t ref_rows, int64_t cmp_rows, const void* q, void* out,
                              void* workspace, cudaStream_t st);

// Merge of per-split partial softmax states into the output.
cudaError_t launch_decode_combine(const CacheArgs& a, int batch, int splits, const float* partials, void* out,
                                  cudaStream_t st);

// Self-test of the bounded waits: records RKV_ERR_TIMEOUT in *err after one wait gives up.
cudaError_t launch_wait_timeout_selftest(int32_t* err, cudaStream_t st);

}  // namespace rkv
