// Internal layout shared by the host dispatch and the CUDA kernels of librkv.
#pragma once

#include <cstdint>

#include "rkv.h"

namespace rkv {

constexpr int kMaxPhases = 32;
constexpr int kPosTile = 128;      // positions per selection tile
constexpr int kCmpPad = 128;       // compressed rows of a unit are padded to a multiple of this
constexpr int kRefPad = 8;         // reference rows of a unit are padded to a multiple of this
constexpr int kMaxKC = 20;         // candidates kept per token by the reference search
constexpr uint64_t kDescMagic = 0x524B564341434845ull;  // "RKVCACHE"

// Candidates the search keeps per token: k plus a margin re-ranked exactly in the encoder.
inline int search_width(int k) { return k <= 4 ? 8 : (k <= 8 ? 12 : 20); }

// Reference schedule in phases.  Phase p covers positions [start[p], start[p+1]) (the last
// phase is unbounded); its references are start[p] + m * stride[p].  A fixed stride is one phase.
struct Phases {
    int32_t n;
    int32_t pad;
    int32_t start[kMaxPhases];
    int32_t stride[kMaxPhases];
    int32_t first_ord[kMaxPhases];   // ordinal of the phase's first reference
    int32_t first_slot[kMaxPhases];  // compressed slot of the phase's first non-reference position
    // division by stride and by stride - 1 as a multiply and a shift (div_magic below)
    uint64_t m_stride[kMaxPhases];
    uint64_t m_per[kMaxPhases];
    int32_t sh_stride[kMaxPhases];
    int32_t sh_per[kMaxPhases];
};

// n / d for 0 <= n < 2^31 and 1 <= d < 2^31 as (n * m) >> sh, with l = ceil(log2 d),
// sh = 31 + l and m = floor(2^sh / d) + 1 (Granlund and Montgomery, "Division by invariant
// integers using multiplication", 1994: exact because m * d - 2^sh <= d <= 2^l).
inline void div_magic(int64_t d, uint64_t& m, int32_t& sh)
{
    int l = 0;
    while ((int64_t(1) << l) < d)
        ++l;
    sh = 31 + l;
    m = (uint64_t(1) << sh) / static_cast<uint64_t>(d) + 1;
}

// One (sequence, kv-head) unit.  Device table, 32 bytes.
struct UnitMeta {
    int32_t n;        // tokens
    int32_t R;        // references
    int32_t C;        // compressed tokens
    int32_t seq;      // sequence index b
    int64_t ref_row;  // first row of the unit in the reference arrays
    int64_t cmp_row;  // first row of the unit in the compressed arrays
};

// Byte offsets of the cache sections inside the caller's buffer.
struct Sections {
    uint64_t err, units, tiles, pairs, ref_K, ref_V, ref_sK, ref_sV, ref_hn, ref_aug, ref_pos, codes_K, codes_V,
        scale_K, scale_V, idx, append, hn_max, end;
};

// Host-side descriptor stored in rkv_cache_desc::opaque.
struct Desc {
    uint64_t magic;
    rkv_config cfg;
    void* base;
    uint64_t bytes;
    int32_t n_units;
    int32_t n_tiles;
    int32_t n_pairs;
    int32_t pad0;
    int32_t kc;
    int32_t code_bytes;
    int32_t n_groups;
    int32_t max_R;
    int32_t max_C;
    int32_t max_n;
    int64_t total_ref_rows;
    int64_t total_cmp_rows;
    Sections sec;
    Phases ph;
    uint64_t ws_select;   // workspace bytes of the search stage
    uint64_t ws_fix_off;  // offset of the encoder's deferred-token list in that workspace
    uint64_t ws_latent_off;  // offset of the learned coder's exact-pass list (coder 1)
    uint64_t ws_decode;   // workspace bytes of the decode stage
    int32_t len[RKV_MAX_BATCH];
    int32_t R[RKV_MAX_BATCH];
    int32_t C[RKV_MAX_BATCH];
    int32_t Rpad[RKV_MAX_BATCH];
    int32_t Cpad[RKV_MAX_BATCH];
    int64_t ref_seq_row[RKV_MAX_BATCH];
    int64_t cmp_seq_row[RKV_MAX_BATCH];
    int32_t cur_len[RKV_MAX_BATCH];   // current lengths (len[] is the capacity the layout holds)
    const uint16_t* coder_w[8];       // learned-coder weights (coder 1): Wg, Wu, Wo, Wd for K, then V
};
static_assert(sizeof(Desc) <= RKV_CACHE_DESC_BYTES, "descriptor too large");

// Everything a kernel needs about one bound cache, passed by value.
struct CacheArgs {
    int32_t D, Hkv, Hq, G, k, bits, group, in_dtype, out_dtype;
    int32_t n_units, code_bytes, n_groups, kc, max_len, max_refs;
    int32_t ref_bits, coder;   // 16: bf16 reference rows, 4: int4 store; coder 0 identity, 1 learned shapes
    Phases ph;
    const UnitMeta* units;
    int32_t* err;
    uint16_t* ref_K;     // bf16 rows [rows][D], or int4 codes [rows][D/2] bytes (ref_bits 4)
    uint16_t* ref_V;
    uint16_t* ref_sK;    // ref_bits 4: binary16 scales [rows][D/32]
    uint16_t* ref_sV;
    float* ref_hn;
    float* ref_hn_max;   // [units] largest half norm of the unit's references (bits compared as int)
    uint16_t* ref_aug;   // [rows][16] bf16: -hi, -mid, -lo of 0.5|r|^2, then zeros (augmented GEMM column)
    int32_t* ref_pos;
    uint8_t* codes_K;
    uint8_t* codes_V;
    uint16_t* scale_K;
    uint16_t* scale_V;
    uint16_t* idx;
    const uint16_t* cw[8];   // coder 1: Wg, Wu, Wo, Wd (bf16 [D][D]) of K, then of V
};

// Selection work item: one tile of kPosTile positions of one unit (CUDA-core search), or a pair
// of consecutive tiles (tensor-core search; `tile` is then the pair index).
struct Tile {
    int32_t unit;
    int32_t tile;
};

}  // namespace rkv
