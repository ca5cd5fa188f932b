/*
 * rkv.h — C ABI of the residual KV-cache compression library (librkv.so).
 *
 * The method (ResidualKV / DeltaKV) keeps a strided set of tokens as
 * uncompressed references and stores every other token as a quantised
 * residual against the mean of its k nearest earlier references:
 *   - paper summary page "ResidualKV: Residual-Based KV Cache Compression for
 *     Efficient Long-Context Inference", section "DeltaKV Framework
 *     Architecture": strided reference selection (reference set T, top-k
 *     nearest by L2 distance, mean reference KV_R), residual computation, and
 *     reconstruction KV = KV_delta + KV_R;
 *   - same page, section "Practical Deployment via Sparse-vLLM": a batched L2
 *     distance kernel for the reference search and a fused reconstruction
 *     kernel (gather, mean, residual add in one launch);
 *   - news page "New KV Cache Compression Method Cuts Long-Context Inference
 *     Costs by 85%", section "How ResidualKV Works": quantized residual codes,
 *     on-the-fly reconstruction when attention needs a token, and
 *     dynamic-stride scheduling (roughly logarithmic reference growth).
 * The learned compressor/decompressor of the pages is replaced by a stated
 * stand-in: the identity plus a symmetric group quantiser (int8 or int4 codes,
 * one binary16 scale per 32 channels).
 *
 * Conventions for every call
 *   - Memory: the caller allocates every buffer (inputs, the cache, the
 *     workspace, outputs) and keeps ownership.  The library allocates no
 *     device memory and never frees caller memory.  It keeps no global state,
 *     with one exception: rkv_compress_noalloc's fixed scratch array (a
 *     file-scope device array, see that call).
 *   - Streams: `stream` is a cudaStream_t (NULL = legacy default stream).
 *     Device work is enqueued asynchronously on it; calls that only touch
 *     host memory ignore it.  Calls on distinct buffers may run concurrently.
 *   - Errors: every call returns an rkv_status.  Invalid arguments are
 *     rejected before anything is enqueued.  A failed launch returns
 *     RKV_ERR_CUDA.  Kernels that meet a corrupted cache (an out-of-range
 *     reference index, an impossible scale) or a bounded wait that ran out
 *     record RKV_ERR_CORRUPT / RKV_ERR_TIMEOUT in the cache's device error
 *     word and skip the affected work; rkv_read_device_error() returns it.
 *     Nothing aborts, traps or throws across this boundary.
 *   - Tensor layouts (row-major, contiguous, device memory unless stated):
 *       K, V   [batch][n_kv_heads][max_len][head_dim]  in_dtype  (one layer)
 *       q      [batch][n_q_heads][head_dim]            in_dtype
 *       out    [batch][n_q_heads][head_dim]            out_dtype
 *     Rows of sequence b past lengths[b] are never read.  Query head g
 *     attends with kv head g / (n_q_heads / n_kv_heads).
 *   - One cache describes one layer: bind one buffer per layer.
 */
#ifndef RKV_H
#define RKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RKV_ABI_VERSION 1

#if defined(__GNUC__)
#define RKV_API __attribute__((visibility("default")))
#else
#define RKV_API
#endif

#define RKV_DTYPE_BF16 0
#define RKV_DTYPE_F32 1

#define RKV_MAX_BATCH 256         /* sequences per cache */
#define RKV_MAX_K 16              /* neighbours per token */
#define RKV_MAX_REFS 65535        /* references per (sequence, kv-head): 16-bit ordinals, 0xFFFF = unused */
#define RKV_IDX_UNUSED 0xFFFFu

/* Optional algorithm choices (rkv_config.flags).  Results agree within the
 * library's tolerances whichever is chosen; the defaults are the fast paths. */
#define RKV_FLAG_SELECT_SIMT 0x1u    /* reference search on CUDA cores even for bf16 inputs */
#define RKV_FLAG_DECODE_DIRECT 0x2u  /* decode by gathering and averaging reference rows per token */
#define RKV_FLAG_DECODE_SIMT 0x4u    /* factorised decode on CUDA cores even where the tensor-core form applies */

typedef enum rkv_status {
    RKV_OK = 0,
    RKV_ERR_INVALID_ARG = 1, /* NULL pointer, bad size, inconsistent shape */
    RKV_ERR_UNSUPPORTED = 2, /* valid but not implemented: head_dim not 64/128, k > 16, > 65535 refs,
                                not an sm_100 device, binary16 scale overflow */
    RKV_ERR_WORKSPACE = 3,   /* cache or workspace buffer smaller than required */
    RKV_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    RKV_ERR_CORRUPT = 5,     /* device-side: cache contents out of range */
    RKV_ERR_TIMEOUT = 6      /* device-side: a bounded wait ran out */
} rkv_status;

/*
 * Static description of one layer's cache.
 *   head_dim        D, 64 or 128
 *   n_kv_heads      key/value heads (Hkv)
 *   n_q_heads       query heads, a multiple of n_kv_heads
 *   k               neighbours per compressed token, 1..16
 *   bits            residual code width, 4 or 8
 *   group           channels per binary16 scale; must be 32
 *   stride0         reference stride s (>= 2): positions 0, s, 2s, ... are references
 *   refs_per_phase  0: fixed stride.  > 0: dynamic stride — the stride doubles
 *                   after every refs_per_phase references (phase p has stride
 *                   stride0 * 2^p and starts where phase p-1's references end)
 *   in_dtype        RKV_DTYPE_BF16 or RKV_DTYPE_F32, for K, V and q
 *   out_dtype       decode output dtype, RKV_DTYPE_BF16 or RKV_DTYPE_F32
 *   batch           sequences, 1..RKV_MAX_BATCH
 *   max_len         row pitch (tokens) of K and V, >= every length
 *   flags           RKV_FLAG_* bits
 *   ref_bits        0 or 16: references stored as bf16 rows.  4: the int4 reference
 *                   store (paper summary page, "Improvements for AI systems" and "Impact
 *                   and Future Directions": full-pipeline 4-bit quantization, applied to
 *                   the uncompressed components too): each reference row of K and V is
 *                   quantised by itself with the residuals' group quantiser (int4 codes,
 *                   one scale per 32 channels stored as binary16), except that the scale
 *                   is rounded up to a power of two, so every stored value code * scale
 *                   is an exact bf16 number; every stage (selection, mean, residual,
 *                   reconstruction, attention) uses that stored value.  Decode then reads
 *                   72 instead of 256 bytes per reference row and side at D = 128.
 *   coder           0: the stored residual is x - mean of the k references.  1: the
 *                   learned-coder shapes (paper summary page, "DeltaKV Framework
 *                   Architecture": z = fc(KV) - fc(KV_R), KV = fd(z) + KV_R;
 *                   "Improvements for AI systems": fc a SwiGLU block, fd a bias-free
 *                   linear projection), with weights the caller binds by rkv_set_coder:
 *                   fc(x) = Wo (silu(Wg x) * (Wu x)), fd(z) = Wd z, hidden and latent
 *                   widths equal to head_dim.  The latent residual z is stored in the
 *                   identity coder's layout with its group quantiser, except that each
 *                   group's scale is the smallest power of two >= max|z| / qmax (so the
 *                   stored codes do not depend on the last bits of how z is evaluated);
 *                   groups whose scale the tensor-core evaluation cannot settle are
 *                   recomputed in double by an extra pass.  Decode
 *                   applies fd by linearity: the codes meet Wd^T q, and Wd is applied once
 *                   to the softmax-weighted latent sum.  Requires head_dim 128, bits 4,
 *                   bf16 inputs, ref_bits 16, n_q_heads / n_kv_heads <= 8 and k <= 8; the
 *                   RKV_FLAG_DECODE_* flags, rkv_decode_attn_sparse and rkv_append answer
 *                   RKV_ERR_UNSUPPORTED for it.
 */
typedef struct rkv_config {
    int32_t head_dim;
    int32_t n_kv_heads;
    int32_t n_q_heads;
    int32_t k;
    int32_t bits;
    int32_t group;
    int32_t stride0;
    int32_t refs_per_phase;
    int32_t in_dtype;
    int32_t out_dtype;
    int32_t batch;
    int32_t max_len;
    uint32_t flags;
    int32_t ref_bits;    /* reference store: 0 or 16 = bf16 rows; 4 = int4 codes, one binary16
                            scale per 32 channels (see below) */
    int32_t coder;       /* 0: identity coder (residual = x - mean); 1: learned-coder shapes */
    int32_t reserved;
} rkv_config;

/* Host-side handle of a bound cache.  Caller-allocated, opaque, plain data:
 * copying it with memcpy gives an equivalent handle. */
#define RKV_CACHE_DESC_BYTES 32768
typedef struct rkv_cache_desc {
    uint64_t opaque[RKV_CACHE_DESC_BYTES / 8];
} rkv_cache_desc;

/* Device pointers and sizes of one (sequence, kv-head) unit of a bound cache.
 * Layout of each array (rows contiguous):
 *   ref_K, ref_V     [n_ref][head_dim] bf16   reference rows, reference ordinal order
 *                    (int4 reference store: [n_ref][head_dim/2] codes packed like the
 *                    residual codes, with ref_scale_K/V [n_ref][head_dim/32] binary16)
 *   ref_half_norm    [n_ref] float            0.5 * |ref_K row|^2 (fp32)
 *   ref_pos          [n_ref] int32            position of each reference
 *   codes_K, codes_V [n_cmp][code_bytes]      residual codes of the compressed tokens in
 *                                             position order; int8: one byte per channel;
 *                                             int4: two channels per byte, even channel in
 *                                             the low nibble; two's complement
 *   scale_K, scale_V [n_cmp][n_groups] binary16 bits
 *   idx              [n_cmp][k] uint16        reference ordinals, ascending, 0xFFFF padding */
typedef struct rkv_unit_view {
    int32_t n;
    int32_t n_ref;
    int32_t n_cmp;
    int32_t k;
    int32_t code_bytes;
    int32_t n_groups;
    int32_t ref_bits;    /* 16: ref_K/ref_V are bf16 rows; 4: int4 codes [n_ref][head_dim/2] */
    int32_t reserved;
    void* ref_K;
    void* ref_V;
    float* ref_half_norm;
    int32_t* ref_pos;
    uint8_t* codes_K;
    uint8_t* codes_V;
    uint16_t* scale_K;
    uint16_t* scale_V;
    uint16_t* idx;
    uint16_t* ref_scale_K;   /* ref_bits 4: binary16 scales [n_ref][head_dim/32]; else NULL */
    uint16_t* ref_scale_V;
} rkv_unit_view;

/* ABI version of the loaded library (RKV_ABI_VERSION). */
RKV_API int32_t rkv_abi_version(void);

/* Static text for a status code. */
RKV_API const char* rkv_status_string(rkv_status s);

/*
 * Reference positions of one sequence of length n under cfg's schedule
 * (paper summary page, "DeltaKV Framework Architecture", strided reference
 * set; news page, "How ResidualKV Works", dynamic stride).  Host only.
 * Writes min(count, cap) ascending positions to pos (host memory; may be NULL)
 * and the count to *n_ref.
 */
RKV_API rkv_status rkv_schedule(const rkv_config* cfg, int32_t n, int32_t* pos, int64_t cap, int32_t* n_ref);

/*
 * Bytes of the cache buffer and of the workspace that rkv_compress and
 * rkv_decode_attn need for one layer with these sequence lengths
 * (lengths: host array of cfg->batch entries, 0 <= length <= max_len).
 * Host only.
 */
RKV_API rkv_status rkv_cache_size(const rkv_config* cfg, const int32_t* lengths, uint64_t* cache_bytes,
                          uint64_t* workspace_bytes);

/*
 * Lays a cache out in dev_buf (device memory, >= rkv_cache_size bytes,
 * 256-byte aligned) and fills *desc.  Writes the per-unit tables and clears
 * the device error word with synchronous copies (returns after they finish);
 * the rest of the buffer is left as is until rkv_build_refs/rkv_compress.
 * Fails with RKV_ERR_UNSUPPORTED on a device other than sm_100.
 */
RKV_API rkv_status rkv_cache_bind(const rkv_config* cfg, const int32_t* lengths, void* dev_buf, uint64_t bytes,
                          rkv_cache_desc* desc);

/* Device pointers of one unit (host only; no device access). */
RKV_API rkv_status rkv_unit_view_get(const rkv_cache_desc* desc, int32_t seq, int32_t kv_head, rkv_unit_view* out);

/*
 * Reference store (paper summary page, "DeltaKV Framework Architecture",
 * strided reference selection: the reference set T is kept uncompressed).
 * For every unit copies the K and V rows at the reference positions into
 * ref_K / ref_V as bf16 (fp32 inputs rounded to nearest even), and writes
 * ref_half_norm and ref_pos.  K, V: one layer, layout above.
 */
RKV_API rkv_status rkv_build_refs(const rkv_cache_desc* desc, const void* K, const void* V, void* stream);

/*
 * Compression of every non-reference token (paper summary page, "DeltaKV
 * Framework Architecture": top-k nearest references by L2 distance on the key,
 * mean reference, residual; news page, "How ResidualKV Works": quantized
 * residual codes).  Needs rkv_build_refs on the same K first.  Candidates of
 * position i are the references at positions <= i (for a compressed token,
 * whose position is never a reference, that is the earlier references); ranking
 * is by (distance,
 * ordinal); k_eff = min(k, candidates); the mean is an fp32 sum in ascending
 * ordinal order divided by k_eff; per 32-channel group
 * scale = smallest binary16 >= max|delta| / qmax and
 * code = round-half-even(delta / scale) (qmax 127 or 7).
 * Writes codes, scales and idx.  workspace: device, >= the size from
 * rkv_cache_size; its contents are scratch.
 */
RKV_API rkv_status rkv_compress(const rkv_cache_desc* desc, const void* K, const void* V, void* workspace,
                        uint64_t workspace_bytes, void* stream);

/*
 * The two stages of rkv_compress, for callers that schedule or time them
 * separately; rkv_compress is rkv_search followed by rkv_encode on the same
 * workspace.  rkv_search (paper summary page, "Practical Deployment via
 * Sparse-vLLM": the batched L2 distance kernel of the reference search) writes
 * per compressed token its leading candidate references into the workspace;
 * rkv_encode reads them, fixes the final top-k by exact distance and writes
 * idx, codes and scales.  The workspace must not change in between.
 */
RKV_API rkv_status rkv_search(const rkv_cache_desc* desc, const void* K, void* workspace, uint64_t workspace_bytes,
                              void* stream);
RKV_API rkv_status rkv_encode(const rkv_cache_desc* desc, const void* K, const void* V, void* workspace,
                              uint64_t workspace_bytes, void* stream);

/*
 * One decode step of attention over the compressed cache (paper summary
 * page, "Training and Inference Integration" and "Practical Deployment via
 * Sparse-vLLM": reconstruction fused into attention; news page, "How
 * ResidualKV Works": a token is rebuilt on the fly from its references and
 * residual code when attention needs it).  For every query head g:
 *   out[b][g] = sum_i softmax_i(q[b][g] . K_i / sqrt(D)) V_i
 * over all lengths[b] cached positions, where reference rows are the stored
 * bf16 rows and compressed rows are mean(references) + code * scale.  The
 * reconstructed cache is never written to memory.  A sequence of length 0
 * gives zeros.  workspace: device, scratch, >= rkv_cache_size's size; it holds
 * state between the kernels of one call, so concurrent calls on different
 * streams need different workspaces.  With bf16 inputs, head_dim 128, int4
 * codes, k <= 8 and at most 8 query heads per kv-head the per-token dot
 * products run on the tensor cores (flag RKV_FLAG_DECODE_SIMT turns that off).
 * That form starts reading q and the reference keys while the previous
 * rkv_decode_attn on the same stream is still finishing (it waits for it only
 * before its first write), so q must not be that call's out or lie in its
 * workspace; work of any other kind queued in between is waited for as usual.
 */
RKV_API rkv_status rkv_decode_attn(const rkv_cache_desc* desc, const void* q, void* out, void* workspace,
                           uint64_t workspace_bytes, void* stream);

/*
 * Weights of the learned-coder shapes (config coder = 1), device pointers, bf16, row-major
 * [out][in], D = head_dim: w[0..3] = Wg_K [D][D], Wu_K [D][D], Wo_K [D][D], Wd_K [D][D];
 * w[4..7] the same for V (see rkv_config.coder).  The caller keeps them alive and unchanged
 * while the cache is used; the handle records the pointers (host call, no launch).
 * RKV_ERR_INVALID_ARG for a NULL or misaligned (16-byte) pointer or a cache bound with
 * coder 0.  Compression and decode of a coder-1 cache before this call fail with
 * RKV_ERR_INVALID_ARG.
 */
RKV_API rkv_status rkv_set_coder(rkv_cache_desc* desc, const void* const* w);

/*
 * Current lengths of the sequences of a bound cache (host array of batch entries,
 * 0 <= lengths[b] <= the length the cache was bound with, which is its capacity).
 * rkv_build_refs, rkv_compress, the decodes and rkv_reconstruct then work on the
 * first lengths[b] positions; rkv_append grows them.  Binding sets the current
 * lengths to the bound ones.  Host arguments; queues one small copy on stream.
 */
RKV_API rkv_status rkv_cache_set_lengths(rkv_cache_desc* desc, const int32_t* lengths, void* stream);

/*
 * Incremental compression (paper summary page, "DeltaKV Framework Architecture";
 * news page, "How ResidualKV Works": each new token is stored as a reference or as
 * a residual against its nearest earlier references).  For every sequence b with
 * active[b] != 0 (active: host array of batch flags, NULL = all) the token at
 * position p = current length is added to each kv-head unit: a reference if p is
 * on the schedule, otherwise compressed against the references so far exactly as
 * rkv_compress would (nearest by exact L2 distance, ties to the lower ordinal).
 *   K_new, V_new  device [batch][n_kv_heads][head_dim], the cache's input dtype;
 *                 rows of inactive sequences are not read
 * Two launches: the distances to the references, split over up to 32 CTAs per unit,
 * each keeping its k best; then per unit the merge, the mean and the quantiser.  The
 * candidate lists live in a small scratch section of the cache buffer (about 6 KB per
 * unit, counted by rkv_cache_size), so appends to one cache run on one stream.
 * Fails with RKV_ERR_INVALID_ARG, launching nothing, if an active sequence is at
 * capacity.  The current lengths advance on return (the work is queued on stream).
 */
RKV_API rkv_status rkv_append(rkv_cache_desc* desc, const void* K_new, const void* V_new, const uint8_t* active,
                              void* stream);

/*
 * One decode step over a subset of the cached positions: selective decompression
 * (paper summary page, "Training and Inference Integration": only the tokens that
 * sparse attention selects are rebuilt, from their references and residual codes).
 * For unit u = b * n_kv_heads + h, the G query heads of kv-head h of sequence b attend
 * to positions[u * max_sel + i], i < counts[u]: the same softmax attention as
 * rkv_decode_attn restricted to those rows.  Reference positions use their stored
 * rows; compressed positions are rebuilt from their codes, scales and k reference
 * rows; nothing else of the cache is read.
 *   positions  device int32 [n_units][max_sel], each in [0, lengths[b]), distinct
 *              within a unit, any order; a position outside its sequence is skipped
 *              and reported as RKV_ERR_INVALID_ARG through the device error word
 *   counts     device int32 [n_units], 0 <= counts[u] <= max_sel (larger is clamped);
 *              a unit with count 0 gives zeros
 *   max_sel    >= 1, the row stride of positions
 * q, out, workspace and stream as for rkv_decode_attn.
 */
RKV_API rkv_status rkv_decode_attn_sparse(const rkv_cache_desc* desc, const void* q, const int32_t* positions,
                                          const int32_t* counts, int32_t max_sel, void* out, void* workspace,
                                          uint64_t workspace_bytes, void* stream);

/*
 * Materialises reconstructed rows of one unit (paper summary page, "DeltaKV
 * Framework Architecture", reconstruction KV = KV_delta + KV_R; "Training and
 * Inference Integration", selective decompression of only the rows needed).
 * positions: device int32[n_pos] in [0, length) or NULL for every position
 * 0..length-1 (then n_pos must equal the length).  K_out, V_out: device
 * [n_pos][head_dim] in out_dtype (either may be NULL).  Reference positions
 * return the stored bf16 row; others m + code * scale computed in fp32.
 */
RKV_API rkv_status rkv_reconstruct(const rkv_cache_desc* desc, int32_t seq, int32_t kv_head, const int32_t* positions,
                           int64_t n_pos, void* K_out, void* V_out, int32_t out_dtype, void* stream);

/*
 * rkv_compress without a caller-provided workspace (no counterpart on the
 * pages; this is an interface convenience of this library).
 *
 * Some callers cannot call cudaMalloc or lend a workspace, for instance an
 * engine that has handed all device memory to its own fixed pool.  This entry
 * point does the same work as rkv_compress, with the
 * search -> encoder candidate lists kept in a file-scope device array of
 * RKV_NOALLOC_SCRATCH_BYTES inside the library instead of in a workspace.  It
 * allocates nothing; every GPU that loads the library holds the array until
 * the process exits.
 *   - Limit: the search part of the workspace must fit the array.  With
 *     A(x) = x rounded up to a multiple of 256, rows = the layer's compressed
 *     rows (every unit's n - n_ref, padded up to a multiple of 128),
 *     ref_rows = its reference rows (every unit's n_ref, padded up to a
 *     multiple of 8) and kc = the search's candidate-list width (k + 4 for
 *     k <= 4, 12 for k <= 8, 20 for k <= 16), that part is
 *         A(2 * rows * kc) + A(4 * rows * kc)       candidate ordinals, scores
 *       + A(8 + 8 * rows)                           the encoder's deferred list
 *       + A(2 * ref_rows * head_dim)                only with ref_bits 4: the
 *                                                   stored keys as bf16 rows
 *       + A(8 + 64 * rows)                          only with coder 1: the groups
 *                                                   left to the exact latent pass
 *     Larger caches get RKV_ERR_WORKSPACE before anything is enqueued.  For
 *     example, a layer of 8 kv-heads x 32768 tokens at stride 16, k 4 (kc 8)
 *     needs about 14 MB with bf16 references and 18 MB (too much) with
 *     ref_bits 4.
 *   - Set-up: the first call in a CUDA context (with that context current)
 *     looks up the array's device address, which belongs to the library's
 *     module in that context; a new context (after cudaDeviceReset, say) gets
 *     its own look-up.
 *   - Sharing: all calls on a device use the same array and it keeps the last
 *     call's contents; nothing in it needs to start at zero (the search writes
 *     every entry the encoder reads).  Calls that overlap on the GPU race on it:
 *     serialise them (one stream, or events).
 */
#define RKV_NOALLOC_SCRATCH_BYTES (16u << 20)
RKV_API rkv_status rkv_compress_noalloc(const rkv_cache_desc* desc, const void* K, const void* V, void* stream);

/*
 * Synchronises `stream`, then reads and clears the cache's device error word.
 * The word lives in the cache buffer (one per bound layer, so concurrent
 * layers do not share it), which is why the call takes the cache handle.
 * *device_status gets RKV_OK or the first RKV_ERR_* a kernel recorded since
 * the last read.  Returns RKV_ERR_CUDA if the synchronisation failed.
 */
RKV_API rkv_status rkv_read_device_error(const rkv_cache_desc* desc, void* stream, int32_t* device_status);

/*
 * Self-test of the kernels' bounded waits (every wait on an mbarrier, a flag or a peer gives up
 * after 2 s of the GPU's global timer and records RKV_ERR_TIMEOUT instead of hanging).  Queues
 * one small kernel on `stream` whose thread waits, with that same bounded wait, on an mbarrier
 * phase that nothing completes; when the wait gives up the kernel writes RKV_ERR_TIMEOUT to
 * *err_dev (a caller-owned device int32, 4-byte aligned) and returns.  The call returns RKV_OK
 * once the kernel is queued; the caller synchronises the stream and reads *err_dev.  The kernel
 * takes about 2 s, and the context stays usable afterwards.  RKV_ERR_INVALID_ARG for a null or
 * unaligned err_dev.
 */
RKV_API rkv_status rkv_selftest_wait_timeout(int32_t* err_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RKV_H */
