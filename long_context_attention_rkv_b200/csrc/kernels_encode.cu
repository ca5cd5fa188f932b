// Residual encoder (ResidualKV paper summary page, "DeltaKV Framework
// Architecture": top-k nearest references, mean reference KV_R, residual
// KV - KV_R; news page "New KV Cache Compression Method Cuts Long-Context
// Inference Costs by 85%", "How ResidualKV Works": quantized residual codes).
//
// Sixteen lanes per compressed token at D = 128 (eight at D = 64; two or four tokens
// per warp); a lane owns 8 consecutive channels, a quarter of a 32-channel group.
// Short per-lane state keeps five 256-thread blocks resident per SM: the kernel is
// bound by the latency of its gathers of reference rows, so resident warps matter.
//  1. Final top-k.  The search handed over its kc best candidates by
//     t = k.r - |r|^2/2 from fp32 accumulation.  With
//     delta = 2^-16 (|k|^2 + max|r|^2) (four times the worst-case error of a
//     128-term fp32 dot product, 2^-18 (|k|^2 + |r|^2), and about 25 times the
//     largest tensor-core vs. CUDA-core difference measured on these inputs): if the (k+1)-th t is more than 2*delta below the k-th, the
//     first k candidates are the top-k (max |r|^2 over all the unit's references, so the
//     bound covers the references outside the list as well).  Otherwise every candidate within 2*delta
//     of the k-th is re-ranked by its exact-order fp32 distance sum_c (k_c - r_c)^2
//     (ties to the lower ordinal); if even the last kept candidate is that close,
//     the list may be incomplete and all candidates are rescanned exactly.  Both
//     slow cases are deferred: the main pass lists them, a rescan kernel gives each
//     token of the second kind a whole block (its candidates split over 256 threads)
//     and rewrites its list as the exact top-k, and a last pass re-ranks and encodes
//     every listed token.
//  2. Mean of the chosen rows in ascending ordinal order (fp32, left to right),
//     one IEEE division by k_eff; residual = x - mean (fp32).
//  3. Per 32-channel group: a = max|residual|, scale = binary16 rounded up from
//     a / qmax, code = round-half-even(residual / scale).  Steps 2-3 use
//     correctly rounded fp32 operations without contraction, so the codes equal an
//     IEEE fp32 evaluation of the same steps bit for bit.
#include <cfloat>

#include "device_common.cuh"
#include "launchers.h"

namespace rkv {

namespace {

constexpr int kWarps = 8;
constexpr int kCpl128 = 8;   // channels per lane at D = 128 (16 lanes per token)

// Sum over the LPT lanes of a token group.
template <int LPT>
__device__ __forceinline__ float tsum(float v)
{
#pragma unroll
    for (int o = 1; o < LPT; o <<= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int LPT>
__device__ __forceinline__ float tmax(float v)
{
#pragma unroll
    for (int o = 1; o < LPT; o <<= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Packed fp32 pairs (sm_100 f32x2): two correctly rounded operations, no contraction, the
// same results as two __fadd_rn / __fsub_rn / __fmul_rn.
__device__ __forceinline__ void add2_rn(float& a0, float& a1, float b0, float b1)
{
    asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
        "add.rn.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
        : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}

__device__ __forceinline__ void sub2_rn(float& d0, float& d1, float a0, float a1, float b0, float b1)
{
    asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %5};\n\t"
        "sub.rn.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
        : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void mul2_rn(float& a0, float& a1, float b0, float b1)
{
    asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
        "mul.rn.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
        : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}

// CPL consecutive bf16 values (CPL = 8 or 16) as floats.
template <int CPL>
__device__ __forceinline__ void load_bf16_row(const uint16_t* p, float (&out)[CPL])
{
#pragma unroll
    for (int h = 0; h < CPL / 8; ++h) {
        const uint4 v = *reinterpret_cast<const uint4*>(p + h * 8);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[h * 8 + 2 * i] = bf16_bits_to_f32(w[i] & 0xffffu);
            out[h * 8 + 2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
        }
    }
}

template <int CPL>
__device__ __forceinline__ void load_input_row(const void* base, int64_t elem, int in_dtype, float (&out)[CPL])
{
    if (in_dtype == RKV_DTYPE_F32) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
#pragma unroll
        for (int h = 0; h < CPL / 4; ++h) {
            const float4 v = p[h];
            out[4 * h] = v.x;
            out[4 * h + 1] = v.y;
            out[4 * h + 2] = v.z;
            out[4 * h + 3] = v.w;
        }
    } else {
        load_bf16_row<CPL>(static_cast<const uint16_t*>(base) + elem, out);
    }
}

// Exact-order fp32 squared distance between this token's key and a reference row's stored
// values (this lane's part, channels c0 ..; sum over the token group with tsum).
template <int CPL, int RB>
__device__ __forceinline__ float part_dist(const CacheArgs& a, const float (&x)[CPL], int64_t row, int c0)
{
    float rv[CPL];
    load_ref<CPL, RB>(a, 0, row, c0, rv);
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const float d = __fsub_rn(x[i], rv[i]);
        s = __fmaf_rn(d, d, s);
    }
    return s;
}

template <int CPL>
__device__ __forceinline__ void quantise_store(const float (&x)[CPL], const float (&m)[CPL], int bits, int sub,
                                               bool store, uint8_t* codes_row, uint16_t* scale_row, int32_t* err)
{
    // lanes per 32-channel group: 2 when CPL = 16, 4 when CPL = 8
    constexpr int LPG = 32 / CPL;
    const int qmax = (bits == 8) ? 127 : 7;
    float d[CPL];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; i += 2)
        sub2_rn(d[i], d[i + 1], x[i], x[i + 1], m[i], m[i + 1]);
#pragma unroll
    for (int i = 0; i < CPL; ++i)
        amax = fmaxf(amax, fabsf(d[i]));
#pragma unroll
    for (int off = 1; off < LPG; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    uint16_t sbits = 0;
    float s = 1.0f;
    if (amax > 0.0f) {
        const __half h = __float2half_ru(__fdiv_rn(amax, static_cast<float>(qmax)));
        sbits = __half_as_ushort(h);
        s = __half2float(h);
        if (store && (sbits & 0x7c00u) == 0x7c00u)
            report(err, RKV_ERR_UNSUPPORTED);
    }
    // code = rint(fl(d / s)).  y = d * fl(1/s) is within 1.5 * 2^-23 |d/s| of fl(d/s), and
    // |d/s| <= qmax < 128, so the two differ by less than 2^-15: unless y lies within 2^-14 of
    // a half-integer, both round to the same integer.  The rare lanes that do take the
    // correctly rounded division for their elements.
    const float rs = __frcp_rn(s);
    float yv[CPL], y[CPL];
#pragma unroll
    for (int i = 0; i < CPL; i += 2) {
        yv[i] = d[i];
        yv[i + 1] = d[i + 1];
        mul2_rn(yv[i], yv[i + 1], rs, rs);
    }
    // Round half to even by adding 1.5 * 2^23 (for |y| < 2^22 the sum's last bits are rint(y)):
    // three adds on the FMA pipe instead of a rounding and a conversion on the slower one.
    // |y| <= qmax (the scale is rounded up), so no code needs clamping.
    constexpr float kRound = 12582912.0f;
    constexpr int kRoundBits = 0x4B400000;
    bool near_half = false;
    int q[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const float t = __fadd_rn(yv[i], kRound);
        q[i] = __float_as_int(t) - kRoundBits;
        y[i] = __fsub_rn(t, kRound);
        near_half |= fabsf(__fsub_rn(yv[i], y[i])) >= 0.5f - 0x1p-14f;
    }
    if (near_half) {
#pragma unroll
        for (int i = 0; i < CPL; ++i)
            q[i] = __float_as_int(__fadd_rn(__fdiv_rn(d[i], s), kRound)) - kRoundBits;
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i)
        q[i] = (amax > 0.0f) ? q[i] : 0;
    if (!store)
        return;
    if (bits == 8) {
        uint32_t w[CPL / 4];
#pragma unroll
        for (int i = 0; i < CPL / 4; ++i)
            w[i] = (q[4 * i] & 0xff) | ((q[4 * i + 1] & 0xff) << 8) | ((q[4 * i + 2] & 0xff) << 16) |
                   (uint32_t(q[4 * i + 3] & 0xff) << 24);
        if constexpr (CPL == 16)
            *reinterpret_cast<uint4*>(codes_row + sub * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        else
            *reinterpret_cast<uint2*>(codes_row + sub * 8) = make_uint2(w[0], w[1]);
    } else {
        uint32_t w[CPL / 8];
#pragma unroll
        for (int i = 0; i < CPL / 8; ++i) {
            uint32_t x8 = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b)
                x8 |= static_cast<uint32_t>(q[8 * i + b] & 0xf) << (4 * b);
            w[i] = x8;
        }
        if constexpr (CPL == 16)
            *reinterpret_cast<uint2*>(codes_row + sub * 8) = make_uint2(w[0], w[1]);
        else
            *reinterpret_cast<uint32_t*>(codes_row + sub * 4) = w[0];
    }
    if ((sub % LPG) == 0)
        scale_row[sub / LPG] = sbits;
}

// Resident blocks per SM the register budget is set for: five (48 registers; 8 bytes spill,
// and 10 % faster than four blocks at 60 registers, six at 40 registers spill more) for the main
// pass at D 128 with up to 12 candidates, two otherwise.
template <int KC, int LPT, bool FIX = false>
constexpr int encode_min_blocks() { return (!FIX && LPT == 16 && KC <= 12) ? 5 : 2; }

// One compressed token per group of LPT lanes: final top-k, mean, residual and quantiser.
// (u, c): the token's unit and compressed slot; inactive groups shadow a valid token and store
// nothing.  FIX false: tokens whose candidate list does not settle the top-k at once (mode 1
// or 2 below: 2 % of them on a 32768-token layer, 10 % on a 131072-token one) are not stored
// but listed, so the main pass stays straight-line: fix[0] counts the mode-1 tokens, listed as
// (unit, slot) pairs from the front of the list, fix[1] the mode-2 tokens, listed from its back
// (the list has fix_cap entries after the two counts).  FIX true: the exact re-rank of the
// listed tokens (the mode-2 ones arrive with their lists already rewritten by the rescan
// kernel as the exact top-k).
template <int CPL, int KC, int LPT, int RB, bool FIX>
__device__ __forceinline__ void encode_group(const CacheArgs& a, const void* __restrict__ K, const void* __restrict__ V,
                                             const uint16_t* __restrict__ cand_idx, const float* __restrict__ cand_t,
                                             int* __restrict__ fix, int fix_cap, int u, int c, bool active)
{
    constexpr int D = CPL * LPT;
    constexpr int kLPT = LPT;                // lanes per token
    constexpr int KM = KC - 4;               // largest k served by this candidate width
    const int lane = threadIdx.x & 31;
    const int sub = lane % kLPT;             // lane within the token group
    const UnitMeta um = a.units[u];
    if (__all_sync(0xffffffffu, !active))
        return;
    const int k = a.k;
    const int cc = active ? c : 0;           // inactive slots shadow token 0 and store nothing
    const int p = slot_pos(a.ph, cc);
    const int ncand = min(refs_upto(a.ph, p), um.R);
    const int64_t row = um.cmp_row + cc;
    const int64_t e = (static_cast<int64_t>(u) * a.max_len + p) * D + sub * CPL;
    float xk[CPL];
    load_input_row<CPL>(K, e, a.in_dtype, xk);
    {
        // the V row is read only at the end (step 3): its lines start towards L2 now, so that
        // read does not add a third memory round trip after the candidates and the gathers
        const char* pv = static_cast<const char*>(V) + e * (a.in_dtype == RKV_DTYPE_F32 ? 4 : 2);
        asm volatile("prefetch.global.L2 [%0];" ::"l"(pv));
    }

    // ---- 1. final top-k -------------------------------------------------------------
    const int nvalid = min(KC, ncand);
    // candidate slot i of this token lives on lane sub == i % 8, register i / 8
    constexpr int PER = (KC + kLPT - 1) / kLPT;
    int co[PER];
    float ct[PER];
    bool bad = false;
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        const int i = r * kLPT + sub;
        co[r] = RKV_IDX_UNUSED;
        ct[r] = -FLT_MAX;
        if (i < nvalid) {
            co[r] = cand_idx[row * KC + i];
            ct[r] = cand_t[row * KC + i];
            bad |= co[r] >= ncand;
        }
    }
    if (__any_sync(0xffffffffu, bad && active)) {
        if (lane == 0)
            report(a.err, RKV_ERR_CORRUPT);
        return;
    }
    auto slot_ord = [&](int i) {   // ordinal of candidate slot i (warp-collective)
        int v = co[0];
#pragma unroll
        for (int r = 1; r < PER; ++r)
            v = (i / kLPT == r) ? co[r] : v;
        return __shfl_sync(0xffffffffu, v, (lane & ~(kLPT - 1)) + i % kLPT);
    };
    auto slot_t = [&](int i) {
        float v = ct[0];
#pragma unroll
        for (int r = 1; r < PER; ++r)
            v = (i / kLPT == r) ? ct[r] : v;
        return __shfl_sync(0xffffffffu, v, (lane & ~(kLPT - 1)) + i % kLPT);
    };
    int keff = min(k, nvalid);
    int chosen[KM];   // chosen ordinals (the same in all 8 lanes of the token)
    // mode: 0 first k by t, 1 exact re-rank of the near set, 2 exhaustive rescan
    int mode = 0;
    // all shuffles below run in every lane (the four tokens of a warp may differ in nvalid)
    float xx = 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; ++i)
        xx = fmaf(xk[i], xk[i], xx);
    xx = tsum<kLPT>(xx);
    const float hm = a.ref_hn_max[u];     // the unit's largest reference half norm
    const float delta = ldexpf(xx + 2.0f * hm, -16);
    const float tk = slot_t(k - 1);
    const float tk1 = slot_t(k);
    const float tlast = slot_t(KC - 1);
    if (nvalid > k && tk1 >= tk - 2.0f * delta)
        mode = ((nvalid == KC) && (ncand > KC) && (tlast >= tk - 2.0f * delta)) ? 2 : 1;
    bool store = active;
    if constexpr (!FIX) {
        // defer the token to the exact passes: listed once (by its group's first lane)
        if (active && mode != 0 && sub == 0) {
            int2* list = reinterpret_cast<int2*>(fix + 2);
            if (mode == 1)
                list[atomicAdd(fix, 1)] = make_int2(u, c);
            else
                list[fix_cap - 1 - atomicAdd(fix + 1, 1)] = make_int2(u, c);
        }
        store = active && mode == 0;
        mode = 0;
    }
    const int any_mode = FIX ? __reduce_max_sync(0xffffffffu, mode) : 0;
    if (any_mode == 0) {
#pragma unroll
        for (int i = 0; i < KM; ++i)
            if (i < k)
                chosen[i] = slot_ord(i);
    } else {
        // warp-collective slow paths, taken by the whole warp; tokens in mode 0 keep the
        // first k candidates
#pragma unroll
        for (int i = 0; i < KM; ++i)
            if (i < k)
                chosen[i] = slot_ord(i);
        if (any_mode >= 1) {
            // exact distances of the near set: candidates i < k, plus those within 2*delta.
            // Every slot's row is read unconditionally (a listed slot's row, else the first
            // slot's), so all the gathers are issued together.  A mode-2 token reaches this
            // pass with its list rewritten as the exact top-k (mode 0); should one still read
            // as mode 2 it is re-ranked within its list like a mode-1 token.
            float dist[KC];
            int ords[KC];
            bool in[KC];
            const bool near = mode != 0;
#pragma unroll
            for (int i = 0; i < KC; ++i) {
                ords[i] = slot_ord(i);
                const float ti = slot_t(i);
                in[i] = near && i < nvalid && (i < k || ti >= tk - 2.0f * delta);
            }
#pragma unroll
            for (int i = 0; i < KC; ++i) {
                const int o = (i < nvalid) ? ords[i] : ords[0];
                dist[i] = tsum<kLPT>(part_dist<CPL, RB>(a, xk, um.ref_row + o, sub * CPL));
            }
            if (near) {
                // rank by (distance, ordinal) within the near set
#pragma unroll
                for (int i = 0; i < KC; ++i) {
                    int rank = 0;
#pragma unroll
                    for (int j2 = 0; j2 < KC; ++j2)
                        rank += (in[j2] && (dist[j2] < dist[i] || (dist[j2] == dist[i] && ords[j2] < ords[i]))) ? 1 : 0;
                    if (in[i] && rank < k) {
#pragma unroll
                        for (int s2 = 0; s2 < KM; ++s2)
                            if (s2 == rank)
                                chosen[s2] = ords[i];
                    }
                }
            }
        }
    }
    // ascending ordinal order of the chosen set, in every lane of the token (odd-even
    // transposition network; unused slots sort last)
    int so[KM];
#pragma unroll
    for (int i = 0; i < KM; ++i)
        so[i] = (i < keff) ? chosen[i] : 0x7fffffff;
#pragma unroll
    for (int pass = 0; pass < KM; ++pass)
#pragma unroll
        for (int i = pass & 1; i + 1 < KM; i += 2) {
            const int lo = min(so[i], so[i + 1]), hi = max(so[i], so[i + 1]);
            so[i] = lo;
            so[i + 1] = hi;
        }
    if (store && sub == 0) {
#pragma unroll
        for (int i = 0; i < KM; ++i)
            if (i < k)
                a.idx[row * k + i] = (i < keff) ? static_cast<uint16_t>(so[i]) : static_cast<uint16_t>(RKV_IDX_UNUSED);
    }

    // ---- 2. mean reference (fp32, ascending ordinals, one division) -------------------
    float mk[CPL], mv[CPL];
    load_ref<CPL, RB>(a, 0, um.ref_row + so[0], sub * CPL, mk);
    load_ref<CPL, RB>(a, 1, um.ref_row + so[0], sub * CPL, mv);
#pragma unroll
    for (int i = 1; i < KM; ++i) {
        if (i < keff) {
            float rk[CPL], rv[CPL];
            load_ref<CPL, RB>(a, 0, um.ref_row + so[i], sub * CPL, rk);
            load_ref<CPL, RB>(a, 1, um.ref_row + so[i], sub * CPL, rv);
#pragma unroll
            for (int j2 = 0; j2 < CPL; j2 += 2) {
                add2_rn(mk[j2], mk[j2 + 1], rk[j2], rk[j2 + 1]);
                add2_rn(mv[j2], mv[j2 + 1], rv[j2], rv[j2 + 1]);
            }
        }
    }
    if (keff & (keff - 1)) {
        const float fk = static_cast<float>(keff);
#pragma unroll
        for (int j2 = 0; j2 < CPL; ++j2) {
            mk[j2] = __fdiv_rn(mk[j2], fk);
            mv[j2] = __fdiv_rn(mv[j2], fk);
        }
    } else {
        // keff a power of two: the division is an exact scaling
        const float inv = 1.0f / static_cast<float>(keff);
#pragma unroll
        for (int j2 = 0; j2 < CPL; j2 += 2) {
            mul2_rn(mk[j2], mk[j2 + 1], inv, inv);
            mul2_rn(mv[j2], mv[j2 + 1], inv, inv);
        }
    }

    // ---- 3. residual and group quantiser ---------------------------------------------
    float xv[CPL];
    load_input_row<CPL>(V, e, a.in_dtype, xv);
    quantise_store<CPL>(xk, mk, a.bits, sub, store, a.codes_K + row * a.code_bytes, a.scale_K + row * a.n_groups,
                        a.err);
    quantise_store<CPL>(xv, mv, a.bits, sub, store, a.codes_V + row * a.code_bytes, a.scale_V + row * a.n_groups,
                        a.err);
}

template <int CPL, int KC, int LPT, int RB, bool FIX>
__global__ void __launch_bounds__(kWarps * 32, (encode_min_blocks<KC, LPT, FIX>())) encode_kernel(
    CacheArgs a, const void* __restrict__ K, const void* __restrict__ V, const uint16_t* __restrict__ cand_idx,
    const float* __restrict__ cand_t, int* __restrict__ fix, int fix_cap)
{
    constexpr int kTPW = 32 / LPT;
    const int warp = threadIdx.x >> 5;
    const int tg = (threadIdx.x & 31) / LPT;
    if constexpr (FIX) {
        // the listed tokens (mode 1 from the front of the list, mode 2 from its back), strided
        // over a grid sized for the device
        const int n1 = *reinterpret_cast<volatile int*>(fix);
        const int n_fix = n1 + *reinterpret_cast<volatile int*>(fix + 1);
        const int2* list = reinterpret_cast<const int2*>(fix + 2);
        for (int base = blockIdx.x * kWarps * kTPW; base < n_fix; base += gridDim.x * kWarps * kTPW) {
            const int t = base + warp * kTPW + tg;
            const bool active = t < n_fix;
            const int2 uc = !active ? make_int2(0, 0) : (t < n1) ? list[t] : list[fix_cap - 1 - (t - n1)];
            encode_group<CPL, KC, LPT, RB, true>(a, K, V, cand_idx, cand_t, fix, fix_cap, uc.x, uc.y, active);
        }
    } else {
        const int u = blockIdx.y;
        const int c = (blockIdx.x * kWarps + warp) * kTPW + tg;
        encode_group<CPL, KC, LPT, RB, false>(a, K, V, cand_idx, cand_t, fix, fix_cap, u, c, c < a.units[u].C);
    }
}

// Exhaustive exact rescan of the mode-2 tokens (candidate lists that may miss a reference):
// one block of 256 threads per listed token, every thread a strided share of the token's
// candidates, each distance the exact-order fp32 sum_c (k_c - r_c)^2 over the channels in
// order; the block's k best by (distance, ordinal) are written back as the token's candidate
// list, with t values that make the last pass take them as they are (slots past k repeat the
// best ordinal with t = -inf).
constexpr int kScanThreads = 256;
constexpr int kScanKM = 16;   // largest k

template <int D, int KC, int RB>
__global__ void __launch_bounds__(kScanThreads) encode_scan_kernel(CacheArgs a, const void* __restrict__ K,
                                                                   uint16_t* __restrict__ cand_idx,
                                                                   float* __restrict__ cand_t,
                                                                   const int* __restrict__ fix, int fix_cap)
{
    constexpr int KM = kScanKM;
    constexpr int NW = kScanThreads / 32;
    __shared__ float xs[D];
    __shared__ float wd[NW][KM];
    __shared__ int wo[NW][KM];
    __shared__ int best[KM];
    const int n2 = *reinterpret_cast<const volatile int*>(fix + 1);
    const int2* list = reinterpret_cast<const int2*>(fix + 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k = a.k;
    for (int e = blockIdx.x; e < n2; e += gridDim.x) {
        const int2 uc = list[fix_cap - 1 - e];
        const UnitMeta um = a.units[uc.x];
        const int p = slot_pos(a.ph, uc.y);
        const int ncand = min(refs_upto(a.ph, p), um.R);
        const int64_t row = um.cmp_row + uc.y;
        const int64_t el = (static_cast<int64_t>(uc.x) * a.max_len + p) * D;
        __syncthreads();   // the previous token's shared state is consumed
        for (int c = tid; c < D; c += kScanThreads)
            xs[c] = (a.in_dtype == RKV_DTYPE_F32) ? static_cast<const float*>(K)[el + c]
                                                  : bf16_bits_to_f32(static_cast<const uint16_t*>(K)[el + c]);
        __syncthreads();
        float bd[KM];
        int bo[KM];
#pragma unroll
        for (int s2 = 0; s2 < KM; ++s2) {
            bd[s2] = FLT_MAX;
            bo[s2] = 0x7fffffff;
        }
        for (int j = tid; j < ncand; j += kScanThreads) {
            float d = 0.0f;
#pragma unroll 4
            for (int c2 = 0; c2 < D; c2 += 8) {
                float rv[8];
                load_ref<8, RB>(a, 0, um.ref_row + j, c2, rv);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float e0 = __fsub_rn(xs[c2 + i], rv[i]);
                    d = __fmaf_rn(e0, e0, d);
                }
            }
            float cv = d;
            int ci = j;
#pragma unroll
            for (int s2 = 0; s2 < KM; ++s2) {
                if (s2 < k) {
                    const bool before = (cv < bd[s2]) || (cv == bd[s2] && ci < bo[s2]);
                    const float fd = bd[s2];
                    const int fo = bo[s2];
                    bd[s2] = before ? cv : fd;
                    bo[s2] = before ? ci : fo;
                    cv = before ? fd : cv;
                    ci = before ? fo : ci;
                }
            }
        }
        // k rounds of a warp-wide minimum over the lanes' sorted lists
        int head = 0;
        for (int r = 0; r < k; ++r) {
            float hd = FLT_MAX;
            int ho = 0x7fffffff;
#pragma unroll
            for (int s2 = 0; s2 < KM; ++s2)
                if (s2 == head) {
                    hd = bd[s2];
                    ho = bo[s2];
                }
            float md = hd;
            int mo = ho;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float od = __shfl_xor_sync(0xffffffffu, md, off);
                const int oo = __shfl_xor_sync(0xffffffffu, mo, off);
                if (od < md || (od == md && oo < mo)) {
                    md = od;
                    mo = oo;
                }
            }
            if (ho == mo && hd == md && ho != 0x7fffffff)
                ++head;
            if (lane == 0) {
                wd[warp][r] = md;
                wo[warp][r] = mo;
            }
        }
        __syncthreads();
        // warp 0: the k best of the NW sorted warp lists (k rounds over their heads)
        if (warp == 0) {
            int wh = 0;   // lane w < NW: head of warp w's list
            for (int r = 0; r < k; ++r) {
                float md = (lane < NW && wh < k) ? wd[lane][wh] : FLT_MAX;
                int mo = (lane < NW && wh < k) ? wo[lane][wh] : 0x7fffffff;
                const float hd = md;
                const int ho = mo;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float od = __shfl_xor_sync(0xffffffffu, md, off);
                    const int oo = __shfl_xor_sync(0xffffffffu, mo, off);
                    if (od < md || (od == md && oo < mo)) {
                        md = od;
                        mo = oo;
                    }
                }
                if (lane < NW && ho == mo && hd == md && ho != 0x7fffffff)
                    ++wh;
                if (lane == 0)
                    best[r] = mo;
            }
        }
        __syncthreads();
        if (tid < KC) {
            const bool in_k = tid < k;
            cand_idx[row * KC + tid] = static_cast<uint16_t>(in_k ? best[tid] : best[0]);
            cand_t[row * KC + tid] = in_k ? 0.0f : -FLT_MAX;
        }
    }
}

// ---- incremental compression: one new token per unit ----------------------------------
// (ResidualKV paper summary page, "DeltaKV Framework Architecture"; news page, "How
// ResidualKV Works": tokens are compressed as they arrive during generation.)  The token at
// position p = n of a unit becomes reference n_ref if p is on the schedule (stored exactly as
// the reference store does), otherwise compressed slot n_cmp: its k nearest references by
// exact distance (double, channel order, no contraction; ties to the lower ordinal: the
// search's definition evaluated directly), the mean in ascending ordinal order and the group
// quantiser of the encoder.  The unit's counts advance on the device.
constexpr int kAppendThreads = 128;
constexpr int kAppendKM = 16;                   // largest k

// Per-unit candidate lists of the append search: chunk c of unit u holds the k best (distance,
// ordinal) of its share of the references, in ascending (distance, ordinal) order.
__host__ __device__ inline int append_chunks(int max_refs)
{
    const int c = (max_refs + kAppendThreads - 1) / kAppendThreads;
    return c < 1 ? 1 : (c > 32 ? 32 : c);
}

__device__ __forceinline__ bool seq_active(const uint32_t (&act)[8], int seq) { return (act[seq >> 5] >> (seq & 31)) & 1u; }

// 1. distances of the new token's key to a chunk of the unit's references, the chunk's k best.
template <int D>
__global__ void __launch_bounds__(kAppendThreads) append_search_kernel(CacheArgs a, const void* __restrict__ Kn,
                                                                        uint32_t act0, uint32_t act1, uint32_t act2,
                                                                        uint32_t act3, uint32_t act4, uint32_t act5,
                                                                        uint32_t act6, uint32_t act7,
                                                                        double* __restrict__ ws_d,
                                                                        int* __restrict__ ws_j, int n_chunks)
{
    constexpr int KM = kAppendKM;
    __shared__ float xs[D];
    __shared__ double bd_s[kAppendThreads / 32][KM];
    __shared__ int bo_s[kAppendThreads / 32][KM];
    const int u = blockIdx.y, ch = blockIdx.x;
    const UnitMeta um = a.units[u];
    const uint32_t act[8] = {act0, act1, act2, act3, act4, act5, act6, act7};
    const int p = um.n;
    if (!seq_active(act, um.seq) || is_ref_pos(a.ph, p))
        return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int R = um.R, k = a.k;
    const int per = (R + n_chunks - 1) / n_chunks;
    const int j_lo = ch * per, j_hi = min(R, j_lo + per);
    const int64_t e_row = static_cast<int64_t>(u) * D;
    for (int c = tid; c < D; c += kAppendThreads)
        xs[c] = (a.in_dtype == RKV_DTYPE_F32) ? static_cast<const float*>(Kn)[e_row + c]
                                              : bf16_bits_to_f32(static_cast<const uint16_t*>(Kn)[e_row + c]);
    __syncthreads();
    double bd[KM];
    int bo[KM];
#pragma unroll
    for (int s2 = 0; s2 < KM; ++s2) {
        bd[s2] = DBL_MAX;
        bo[s2] = 0x7fffffff;
    }
    for (int j = j_lo + tid; j < j_hi; j += kAppendThreads) {
        // distance in double, channels in order, no contraction (the search's definition)
        double d = 0.0;
#pragma unroll 2
        for (int c8 = 0; c8 < D / 8; ++c8) {
            float rv[8];
            load_ref<8>(a, 0, um.ref_row + j, c8 * 8, rv);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const double t = __dsub_rn(static_cast<double>(xs[c8 * 8 + i]), static_cast<double>(rv[i]));
                d = __dadd_rn(d, __dmul_rn(t, t));
            }
        }
        double cv = d;
        int ci = j;
#pragma unroll
        for (int s2 = 0; s2 < KM; ++s2) {
            if (s2 < k) {
                const bool before = (cv < bd[s2]) || (cv == bd[s2] && ci < bo[s2]);
                const double fd = bd[s2];
                const int fo = bo[s2];
                bd[s2] = before ? cv : fd;
                bo[s2] = before ? ci : fo;
                cv = before ? fd : cv;
                ci = before ? fo : ci;
            }
        }
    }
    // k rounds of a warp-wide minimum, then the four warps' lists in thread 0
    int head = 0;
    for (int r2 = 0; r2 < k; ++r2) {
        double hd = DBL_MAX;
        int ho = 0x7fffffff;
#pragma unroll
        for (int s2 = 0; s2 < KM; ++s2)
            if (s2 == head) {
                hd = bd[s2];
                ho = bo[s2];
            }
        double wd = hd;
        int wo = ho;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const double od = __shfl_xor_sync(0xffffffffu, wd, off);
            const int oo = __shfl_xor_sync(0xffffffffu, wo, off);
            if (od < wd || (od == wd && oo < wo)) {
                wd = od;
                wo = oo;
            }
        }
        if (ho == wo && hd == wd)
            ++head;
        if (lane == 0) {
            bd_s[warp][r2] = wd;
            bo_s[warp][r2] = wo;
        }
    }
    __syncthreads();
    if (tid == 0) {
        int hp[kAppendThreads / 32] = {};
        const int64_t base = (static_cast<int64_t>(u) * n_chunks + ch) * KM;
        for (int r2 = 0; r2 < k; ++r2) {
            int bw = 0;
            for (int w2 = 1; w2 < kAppendThreads / 32; ++w2) {
                const double dw = bd_s[w2][hp[w2]], db = bd_s[bw][hp[bw]];
                if (dw < db || (dw == db && bo_s[w2][hp[w2]] < bo_s[bw][hp[bw]]))
                    bw = w2;
            }
            ws_d[base + r2] = bd_s[bw][hp[bw]];
            ws_j[base + r2] = bo_s[bw][hp[bw]];
            ++hp[bw];
        }
    }
}

// 2. the new token itself: a reference row, or the merge of the chunks' lists, the mean and the
// encoder's quantiser.  The unit's counts advance on the device.
template <int D>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(CacheArgs a, const void* __restrict__ Kn,
                                                                 const void* __restrict__ Vn, uint32_t act0,
                                                                 uint32_t act1, uint32_t act2, uint32_t act3,
                                                                 uint32_t act4, uint32_t act5, uint32_t act6,
                                                                 uint32_t act7, const double* __restrict__ ws_d,
                                                                 const int* __restrict__ ws_j, int n_chunks)
{
    constexpr int KM = kAppendKM;
    constexpr int CPL = 8;                      // channels per lane in the encode step
    constexpr int LPT = D / CPL;
    __shared__ int chosen_s[KM];
    const int u = blockIdx.x;
    UnitMeta* um_ptr = const_cast<UnitMeta*>(a.units) + u;
    const UnitMeta um = *um_ptr;
    const uint32_t act[8] = {act0, act1, act2, act3, act4, act5, act6, act7};
    if (!seq_active(act, um.seq))
        return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p = um.n;
    const int64_t e_row = static_cast<int64_t>(u) * D;      // the new rows: [unit][D]
    if (is_ref_pos(a.ph, p)) {
        // reference ordinal um.R, written as the reference store writes it
        if (warp == 0) {
            constexpr int NPL = D / 32;
            const int j = um.R;
            float kx[NPL], vx[NPL];
            load_row_part<NPL>(Kn, e_row + lane * NPL, a.in_dtype, kx);
            load_row_part<NPL>(Vn, e_row + lane * NPL, a.in_dtype, vx);
            float ss = 0.0f;
            const int64_t row = um.ref_row + j;
            if (a.ref_bits == 4) {
                float rk[NPL], rv[NPL];
                ref_quantise_store<NPL>(kx, lane, reinterpret_cast<uint8_t*>(a.ref_K) + row * (D / 2),
                                        a.ref_sK + row * (D / 32), rk, a.err);
                ref_quantise_store<NPL>(vx, lane, reinterpret_cast<uint8_t*>(a.ref_V) + row * (D / 2),
                                        a.ref_sV + row * (D / 32), rv, a.err);
#pragma unroll
                for (int i = 0; i < NPL; ++i)
                    ss = fmaf(rk[i], rk[i], ss);
            } else {
                const int64_t o = row * D + lane * NPL;
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    const uint16_t kb = f32_to_bf16_bits(kx[i]);
                    const uint16_t vb = f32_to_bf16_bits(vx[i]);
                    a.ref_K[o + i] = kb;
                    a.ref_V[o + i] = vb;
                    const float r = bf16_bits_to_f32(kb);
                    ss = fmaf(r, r, ss);
                }
            }
            ss = warp_sum(ss);
            if (lane == 0) {
                const float hn = 0.5f * ss;
                a.ref_hn[um.ref_row + j] = hn;
                a.ref_pos[um.ref_row + j] = p;
                atomicMax(reinterpret_cast<int*>(a.ref_hn_max + u), __float_as_int(hn));
                const uint16_t hi = f32_to_bf16_bits(hn);
                const float r1 = hn - bf16_bits_to_f32(hi);
                const uint16_t mid = f32_to_bf16_bits(r1);
                const uint16_t lo = f32_to_bf16_bits(r1 - bf16_bits_to_f32(mid));
                uint4* aug = reinterpret_cast<uint4*>(a.ref_aug + (um.ref_row + j) * 16);
                aug[0] = make_uint4((hi ^ 0x8000u) | ((mid ^ 0x8000u) << 16), lo ^ 0x8000u, 0u, 0u);
                aug[1] = make_uint4(0u, 0u, 0u, 0u);
                __threadfence();
                um_ptr->R = j + 1;
                um_ptr->n = p + 1;
            }
        }
        return;
    }
    // ---- compressed token: the k best of the chunks' lists -------------------------------
    const int R = um.R;
    const int k = a.k;
    const int keff = min(k, R);
    if (tid == 0) {
        int hp[32] = {};
        int ch[KM];
        const int64_t base = static_cast<int64_t>(u) * n_chunks * KM;
        for (int r2 = 0; r2 < keff; ++r2) {
            int bc = 0;
            for (int c2 = 1; c2 < n_chunks; ++c2) {
                const double dc = (hp[c2] < k) ? ws_d[base + c2 * KM + hp[c2]] : DBL_MAX;
                const int jc = (hp[c2] < k) ? ws_j[base + c2 * KM + hp[c2]] : 0x7fffffff;
                const double db = (hp[bc] < k) ? ws_d[base + bc * KM + hp[bc]] : DBL_MAX;
                const int jb = (hp[bc] < k) ? ws_j[base + bc * KM + hp[bc]] : 0x7fffffff;
                if (dc < db || (dc == db && jc < jb))
                    bc = c2;
            }
            ch[r2] = ws_j[base + bc * KM + hp[bc]];
            ++hp[bc];
        }
        // ascending ordinal order
        for (int i2 = 1; i2 < keff; ++i2)
            for (int j2 = i2; j2 > 0 && ch[j2 - 1] > ch[j2]; --j2) {
                const int t = ch[j2];
                ch[j2] = ch[j2 - 1];
                ch[j2 - 1] = t;
            }
        for (int i2 = 0; i2 < KM; ++i2)
            chosen_s[i2] = (i2 < keff) ? ch[i2] : 0;
        const int64_t row = um.cmp_row + um.C;
        for (int i2 = 0; i2 < k; ++i2)
            a.idx[row * k + i2] = (i2 < keff) ? static_cast<uint16_t>(ch[i2]) : static_cast<uint16_t>(RKV_IDX_UNUSED);
    }
    __syncthreads();
    // ---- mean, residual and quantiser: warp 0, LPT lanes of CPL channels (lanes past LPT
    // shadow lane 0 and store nothing)
    if (warp == 0) {
        const int sub = (lane < LPT) ? lane : 0;
        const bool store = lane < LPT;
        const int64_t row = um.cmp_row + um.C;
        float xk[CPL], xv[CPL], mk[CPL], mv[CPL];
        load_input_row<CPL>(Kn, e_row + sub * CPL, a.in_dtype, xk);
        load_input_row<CPL>(Vn, e_row + sub * CPL, a.in_dtype, xv);
        {
            const int o = chosen_s[0];
            load_ref<CPL>(a, 0, um.ref_row + o, sub * CPL, mk);
            load_ref<CPL>(a, 1, um.ref_row + o, sub * CPL, mv);
        }
        for (int i2 = 1; i2 < keff; ++i2) {
            const int o = chosen_s[i2];
            float rk[CPL], rv[CPL];
            load_ref<CPL>(a, 0, um.ref_row + o, sub * CPL, rk);
            load_ref<CPL>(a, 1, um.ref_row + o, sub * CPL, rv);
#pragma unroll
            for (int j2 = 0; j2 < CPL; ++j2) {
                mk[j2] = __fadd_rn(mk[j2], rk[j2]);
                mv[j2] = __fadd_rn(mv[j2], rv[j2]);
            }
        }
        if (keff & (keff - 1)) {
            const float fk = static_cast<float>(keff);
#pragma unroll
            for (int j2 = 0; j2 < CPL; ++j2) {
                mk[j2] = __fdiv_rn(mk[j2], fk);
                mv[j2] = __fdiv_rn(mv[j2], fk);
            }
        } else {
            const float inv = 1.0f / static_cast<float>(keff);
#pragma unroll
            for (int j2 = 0; j2 < CPL; ++j2) {
                mk[j2] = __fmul_rn(mk[j2], inv);
                mv[j2] = __fmul_rn(mv[j2], inv);
            }
        }
        quantise_store<CPL>(xk, mk, a.bits, sub, store, a.codes_K + row * a.code_bytes,
                            a.scale_K + row * a.n_groups, a.err);
        quantise_store<CPL>(xv, mv, a.bits, sub, store, a.codes_V + row * a.code_bytes,
                            a.scale_V + row * a.n_groups, a.err);
        __syncwarp();
        if (lane == 0) {
            __threadfence();
            um_ptr->C = um.C + 1;
            um_ptr->n = p + 1;
        }
    }
}

template <int CPL, int KC, int LPT, int RB>
void launch_pair(const CacheArgs& a, dim3 grid, const void* K, const void* V, uint16_t* ci, float* ct, int* fix,
                 int fix_cap, int fix_grid, int scan_grid, cudaStream_t st)
{
    encode_kernel<CPL, KC, LPT, RB, false><<<grid, kWarps * 32, 0, st>>>(a, K, V, ci, ct, fix, fix_cap);
    encode_scan_kernel<CPL * LPT, KC, RB><<<scan_grid, kScanThreads, 0, st>>>(a, K, ci, ct, fix, fix_cap);
    encode_kernel<CPL, KC, LPT, RB, true><<<fix_grid, kWarps * 32, 0, st>>>(a, K, V, ci, ct, fix, fix_cap);
}

template <int CPL, int LPT>
cudaError_t launch_cpl(const CacheArgs& a, int max_C, const void* K, const void* V, uint16_t* ci, float* ct,
                       int* fix, int fix_cap, int sms, cudaStream_t st)
{
    const int per_block = kWarps * (32 / LPT);
    const dim3 grid((max_C + per_block - 1) / per_block, a.n_units);
    // the deferred pass: a few blocks per SM stride over the list (a few percent of the tokens)
    const int fix_need = (fix_cap + per_block - 1) / per_block;
    const int fix_grid = fix_need < 4 * sms ? (fix_need > 0 ? fix_need : 1) : 4 * sms;
    const int scan_grid = 2 * sms;   // blocks of the rescan, striding over the mode-2 list
    if (a.ref_bits == 4) {
        switch (a.kc) {
        case 8: launch_pair<CPL, 8, LPT, 4>(a, grid, K, V, ci, ct, fix, fix_cap, fix_grid, scan_grid, st); break;
        case 12: launch_pair<CPL, 12, LPT, 4>(a, grid, K, V, ci, ct, fix, fix_cap, fix_grid, scan_grid, st); break;
        default: launch_pair<CPL, 20, LPT, 4>(a, grid, K, V, ci, ct, fix, fix_cap, fix_grid, scan_grid, st); break;
        }
        return cudaGetLastError();
    }
    switch (a.kc) {
    case 8: launch_pair<CPL, 8, LPT, 16>(a, grid, K, V, ci, ct, fix, fix_cap, fix_grid, scan_grid, st); break;
    case 12: launch_pair<CPL, 12, LPT, 16>(a, grid, K, V, ci, ct, fix, fix_cap, fix_grid, scan_grid, st); break;
    default: launch_pair<CPL, 20, LPT, 16>(a, grid, K, V, ci, ct, fix, fix_cap, fix_grid, scan_grid, st); break;
    }
    return cudaGetLastError();
}

}  // namespace

uint64_t append_scratch_bytes(int n_units)
{
    return static_cast<uint64_t>(n_units) * 32 * kAppendKM * (sizeof(double) + sizeof(int));
}

cudaError_t launch_append(const CacheArgs& a, const void* K_new, const void* V_new, const uint32_t (&active)[8],
                          void* scratch, cudaStream_t st)
{
    const int nc = append_chunks(a.max_refs);
    double* ws_d = static_cast<double*>(scratch);
    int* ws_j = reinterpret_cast<int*>(ws_d + static_cast<int64_t>(a.n_units) * 32 * kAppendKM);
    const uint32_t* b = active;
    if (a.D == 128) {
        append_search_kernel<128><<<dim3(nc, a.n_units), kAppendThreads, 0, st>>>(
            a, K_new, b[0], b[1], b[2], b[3], b[4], b[5], b[6], b[7], ws_d, ws_j, nc);
        append_kernel<128><<<a.n_units, kAppendThreads, 0, st>>>(a, K_new, V_new, b[0], b[1], b[2], b[3], b[4], b[5],
                                                               b[6], b[7], ws_d, ws_j, nc);
    } else {
        append_search_kernel<64><<<dim3(nc, a.n_units), kAppendThreads, 0, st>>>(
            a, K_new, b[0], b[1], b[2], b[3], b[4], b[5], b[6], b[7], ws_d, ws_j, nc);
        append_kernel<64><<<a.n_units, kAppendThreads, 0, st>>>(a, K_new, V_new, b[0], b[1], b[2], b[3], b[4], b[5],
                                                              b[6], b[7], ws_d, ws_j, nc);
    }
    return cudaGetLastError();
}

cudaError_t launch_encode(const CacheArgs& a, int max_C, const void* K, const void* V, uint16_t* cand_idx,
                          float* cand_t, int* fix, int fix_cap, cudaStream_t st)
{
    if (max_C <= 0)
        return cudaSuccess;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    e = cudaMemsetAsync(fix, 0, 2 * sizeof(int), st);
    if (e != cudaSuccess)
        return e;
    return (a.D == 128) ? launch_cpl<kCpl128, 128 / kCpl128>(a, max_C, K, V, cand_idx, cand_t, fix, fix_cap, sms, st)
                        : launch_cpl<8, 8>(a, max_C, K, V, cand_idx, cand_t, fix, fix_cap, sms, st);
}

}  // namespace rkv
