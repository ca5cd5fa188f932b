// CPU ORACLE for residual KV-cache compression (ResidualKV / DeltaKV).
//
// TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
// statement of what the CUDA path computes.  It shares no code, header, table
// or helper with the CUDA library; only tests/, the smoke check and the
// bench's CPU-baseline leg may load it.  The product path never calls it.
//
// Sources (web pages on the method; cited by page title and section):
//   [P1] "ResidualKV: Residual-Based KV Cache Compression for Efficient
//        Long-Context Inference" (paper summary page), section "DeltaKV
//        Framework Architecture": strided reference set T, top-k nearest
//        references by L2 distance, mean reference KV_R, residual, and
//        reconstruction KV = KV_delta + KV_R.
//   [P3] "New KV Cache Compression Method Cuts Long-Context Inference Costs by
//        85%", section "How ResidualKV Works": quantized residual codes and
//        dynamic-stride scheduling with roughly logarithmic reference growth.
//
// Readings of what the pages leave open (each is listed with its reason in
// the design notes of this repository):
//   * the learned compressor is replaced by the identity and the learned coder
//     by a symmetric group quantiser: one fp16 scale per 32-channel group,
//     scale = smallest binary16 >= max|delta| / qmax, code = round-half-even
//     (delta / scale), qmax = 127 (int8) or 7 (int4);
//   * dynamic stride: the stride doubles after every refs_per_phase references;
//   * references are stored in bf16 (fp32 inputs rounded to nearest even) and
//     selection, mean and residual use the stored values;
//   * int4 reference store (optional): each reference row is quantised by
//     itself with the residuals' group quantiser, the scale rounded up to a
//     power of two (so code * scale is an exact bf16 value); the stored value
//     is code * scale and every step uses it (the "_f" entry points take the
//     stored values as fp32);
//   * candidates of position i are the references at positions <= i; the
//     distance is on the key vector only and one index set serves K and V;
//   * top-k ranks by (distance, ordinal), keeps k_eff = min(k, #candidates),
//     and stores the chosen ordinals in ascending order, 0xFFFF padding;
//   * the mean is an fp32 sum in ascending-ordinal order followed by one fp32
//     division by k_eff; the residual is an fp32 subtraction;
//   * attention: softmax(q.K/sqrt(D)) V over all n cached positions, double.
//
// Arithmetic: doubles for distances and attention (exact differences and
// squares of float inputs), IEEE fp32 for the mean/residual/quantiser steps.
// Built with -O2 -ffp-contract=off so no fused multiply-add changes a result.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <utility>
#include <vector>

namespace {

// bf16 bits -> float: the bf16 value is the top half of the fp32 pattern.
float bf16_value(uint16_t b)
{
    uint32_t u = static_cast<uint32_t>(b) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// float -> bf16 bits, round to nearest, ties to even (IEEE 754 roundTiesToEven
// applied to the 16 dropped fraction bits).  Inputs here are finite.
uint16_t bf16_round(float f)
{
    uint32_t u;
    std::memcpy(&u, &f, 4);
    const uint32_t keep = u >> 16;
    const uint32_t drop = u & 0xffffu;
    uint32_t r = keep;
    if (drop > 0x8000u || (drop == 0x8000u && (keep & 1u)))
        r += 1;
    return static_cast<uint16_t>(r);
}

// Smallest IEEE binary16 value >= f (rounding toward +infinity), for f >= 0.
// binary16: 5 exponent bits (bias 15), 10 fraction bits; subnormal spacing
// 2^-24 below 2^-14; largest finite 65504.  Returns the bit pattern; sets
// *overflow when the result is +infinity.
uint16_t fp16_round_up(float f, int* overflow)
{
    const double v = static_cast<double>(f);
    if (!(v > 0.0))
        return 0;
    if (v > 65504.0) {
        *overflow = 1;
        return 0x7c00;
    }
    int e = 0;
    std::frexp(v, &e);            // v = fr * 2^e with fr in [0.5, 1)
    const int E = e - 1;          // 2^E <= v < 2^(E+1)
    const double quantum = (E < -14) ? std::ldexp(1.0, -24) : std::ldexp(1.0, E - 10);
    const double m = std::ceil(v / quantum);  // v / quantum is exact (power-of-two scaling)
    const double r = m * quantum;             // the rounded value, exact
    if (r < std::ldexp(1.0, -14))
        return static_cast<uint16_t>(m);      // subnormal: fraction = r / 2^-24
    int e2 = 0;
    std::frexp(r, &e2);
    const int E2 = e2 - 1;
    const double frac = r / std::ldexp(1.0, E2 - 10) - 1024.0;  // in [0, 1023]
    return static_cast<uint16_t>(((E2 + 15) << 10) | static_cast<int>(frac));
}

// Smallest power of two >= f (f >= 0) as binary16 bits, within binary16's powers of two
// 2^-24 .. 2^15; above 2^15 sets *overflow and returns +infinity.
uint16_t pow2_round_up(float f, int* overflow)
{
    const double v = static_cast<double>(f);
    if (!(v > 0.0))
        return 0;
    int e = 0;
    const double fr = std::frexp(v, &e);   // v = fr * 2^e, fr in [0.5, 1)
    int E = (fr == 0.5) ? e - 1 : e;       // smallest E with 2^E >= v
    if (E > 15) {
        *overflow = 1;
        return 0x7c00;
    }
    if (E < -24)
        E = -24;
    return (E >= -14) ? static_cast<uint16_t>((E + 15) << 10) : static_cast<uint16_t>(1u << (E + 24));
}

float fp16_value(uint16_t h)
{
    const int exp = (h >> 10) & 0x1f;
    const int frac = h & 0x3ff;
    double v;
    if (exp == 0)
        v = std::ldexp(static_cast<double>(frac), -24);
    else if (exp == 31)
        v = INFINITY;
    else
        v = std::ldexp(static_cast<double>(1024 + frac), exp - 25);
    return static_cast<float>((h & 0x8000) ? -v : v);
}

// Mean reference of one token: acc = r_j1; acc += r_j2; ...; acc / k_eff (fp32), over the
// stored reference values (bf16 rows widened, or int4 rows dequantised).
void mean_reference(int D, const float* refs, const uint16_t* idx, int keff, float* m)
{
    for (int c = 0; c < D; ++c) {
        float acc = refs[static_cast<int64_t>(idx[0]) * D + c];
        for (int l = 1; l < keff; ++l)
            acc = acc + refs[static_cast<int64_t>(idx[l]) * D + c];
        m[c] = acc / static_cast<float>(keff);
    }
}

// Stored values of bf16 reference rows.
std::vector<float> widen_bf16(const uint16_t* rows, int64_t count)
{
    std::vector<float> out(static_cast<size_t>(count));
    for (int64_t i = 0; i < count; ++i)
        out[i] = bf16_value(rows[i]);
    return out;
}

// The symmetric group quantiser of one row of D values ([P3] "How ResidualKV Works":
// quantized codes; with one fp16 scale per group).  Per group: a = max|v|; a == 0 -> scale 0
// and codes 0; else scale = fp16_round_up(a / qmax) and code = clamp(round_half_even(v /
// scale), -qmax, qmax).  Packing: int8 one byte per channel (two's complement); int4 two
// channels per byte, the even channel in the low nibble.  Returns 1 when a scale overflowed
// binary16, else 0.
int quantize_groups(int D, int bits, int group, const float* v, uint8_t* out, uint16_t* scales, bool pow2 = false)
{
    int overflow = 0;
    const int qmax = (bits == 8) ? 127 : 7;
    const int code_bytes = D * bits / 8;
    std::memset(out, 0, code_bytes);
    for (int g = 0; g < D / group; ++g) {
        float a = 0.0f;
        for (int c = g * group; c < (g + 1) * group; ++c)
            a = std::max(a, std::fabs(v[c]));
        uint16_t sbits = 0;
        if (a > 0.0f)
            sbits = pow2 ? pow2_round_up(a / static_cast<float>(qmax), &overflow)
                         : fp16_round_up(a / static_cast<float>(qmax), &overflow);
        scales[g] = sbits;
        const float s = fp16_value(sbits);
        for (int c = g * group; c < (g + 1) * group; ++c) {
            int code = 0;
            if (a > 0.0f) {
                const float qv = v[c] / s;
                code = static_cast<int>(std::nearbyintf(qv));  // default rounding: ties to even
                code = std::min(qmax, std::max(-qmax, code));
            }
            if (bits == 8) {
                out[c] = static_cast<uint8_t>(static_cast<int8_t>(code));
            } else {
                const uint8_t nib = static_cast<uint8_t>(code & 0xf);
                out[c / 2] |= (c & 1) ? static_cast<uint8_t>(nib << 4) : nib;
            }
        }
    }
    return overflow;
}

int count_keff(const uint16_t* idx, int k)
{
    int n = 0;
    while (n < k && idx[n] != 0xffffu)
        ++n;
    return n;
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Reference schedule ([P1] "DeltaKV Framework Architecture", strided reference
// selection; [P3] "How ResidualKV Works", dynamic-stride scheduling).
// Fixed stride (refs_per_phase == 0): T = {0, s, 2s, ...} intersected with [0, n).
// Dynamic: phase p has stride s*2^p and refs_per_phase positions starting at
// P_p, with P_0 = 0 and P_{p+1} = P_p + refs_per_phase * s * 2^p.
// Returns |T| and writes up to cap positions (ascending) when pos != NULL.
// ---------------------------------------------------------------------------
int64_t orc_schedule(int64_t n, int32_t stride0, int32_t refs_per_phase, int32_t* pos, int64_t cap)
{
    int64_t count = 0;
    if (refs_per_phase <= 0) {
        for (int64_t p = 0; p < n; p += stride0) {
            if (pos && count < cap)
                pos[count] = static_cast<int32_t>(p);
            ++count;
        }
        return count;
    }
    int64_t start = 0;
    int64_t stride = stride0;
    while (start < n) {
        for (int64_t m = 0; m < refs_per_phase; ++m) {
            const int64_t p = start + m * stride;
            if (p >= n)
                return count;
            if (pos && count < cap)
                pos[count] = static_cast<int32_t>(p);
            ++count;
        }
        start += refs_per_phase * stride;
        stride *= 2;
    }
    return count;
}

// Reference store: rows of X at the reference positions, rounded to bf16.
void orc_build_refs(int D, const float* X, const int32_t* ref_pos, int64_t R, uint16_t* ref_out)
{
    for (int64_t j = 0; j < R; ++j)
        for (int c = 0; c < D; ++c)
            ref_out[j * D + c] = bf16_round(X[static_cast<int64_t>(ref_pos[j]) * D + c]);
}

void orc_bf16_round(const float* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = bf16_round(x[i]);
}

// L2 distance, straight from its definition: sum_c (a_c - b_c)^2 in double.
double orc_l2(int D, const float* a, const float* b)
{
    double d = 0.0;
    for (int c = 0; c < D; ++c) {
        const double t = static_cast<double>(a[c]) - static_cast<double>(b[c]);
        d += t * t;
    }
    return d;
}

// ---------------------------------------------------------------------------
// Top-k nearest references ([P1] "DeltaKV Framework Architecture": the top-k
// nearest tokens of the reference set T by L2 distance).
// For token t (position tok_pos[t], key x[t]): candidates are the references
// at positions <= tok_pos[t]; they are ranked by (distance, ordinal) and the
// first k_eff = min(k, #candidates) are written in ascending ordinal order,
// padded with 0xFFFF.  dist_out[t][0..k] gets the k+1 smallest distances in
// rank order (NaN where there are fewer candidates).
// ---------------------------------------------------------------------------
// refK holds the stored reference values (fp32): orc_select passes bf16 rows widened,
// orc_select_f rows given as values (the int4 reference store, dequantised).
void orc_select_f(int D, int64_t n_tok, const float* x, const int32_t* tok_pos, int64_t R, const float* rf,
                  const int32_t* ref_pos, int k, uint16_t* idx_out, int32_t* keff_out, double* dist_out)
{
    std::vector<std::pair<double, int64_t>> cand;
    for (int64_t t = 0; t < n_tok; ++t) {
        cand.clear();
        for (int64_t j = 0; j < R && ref_pos[j] <= tok_pos[t]; ++j)
            cand.emplace_back(orc_l2(D, x + t * D, rf + j * D), j);
        const int64_t take = std::min<int64_t>(static_cast<int64_t>(k) + 1, static_cast<int64_t>(cand.size()));
        std::partial_sort(cand.begin(), cand.begin() + take, cand.end());  // (distance, ordinal) order
        const int keff = static_cast<int>(std::min<int64_t>(k, static_cast<int64_t>(cand.size())));
        std::vector<int64_t> chosen;
        for (int l = 0; l < keff; ++l)
            chosen.push_back(cand[l].second);
        std::sort(chosen.begin(), chosen.end());
        for (int l = 0; l < k; ++l)
            idx_out[t * k + l] = (l < keff) ? static_cast<uint16_t>(chosen[l]) : static_cast<uint16_t>(0xffffu);
        if (keff_out)
            keff_out[t] = keff;
        if (dist_out)
            for (int l = 0; l <= k; ++l)
                dist_out[t * (k + 1) + l] = (l < take) ? cand[l].first : NAN;
    }
}

void orc_select(int D, int64_t n_tok, const float* x, const int32_t* tok_pos, int64_t R, const uint16_t* refK,
                const int32_t* ref_pos, int k, uint16_t* idx_out, int32_t* keff_out, double* dist_out)
{
    const std::vector<float> rf = widen_bf16(refK, R * D);
    orc_select_f(D, n_tok, x, tok_pos, R, rf.data(), ref_pos, k, idx_out, keff_out, dist_out);
}

// ---------------------------------------------------------------------------
// Residual encoding ([P1] "DeltaKV Framework Architecture", residual
// computation, with the compressor taken as the identity; [P3] "How
// ResidualKV Works", compact quantized residual codes).
// For each token: m = mean of its references (fp32, ascending ordinals),
// delta = x - m (fp32).  Per group of `group` channels: a = max|delta|;
// a == 0 -> scale 0 and codes 0; else scale = fp16_round_up(a / qmax) and
// code = clamp(round_half_even(delta / scale), -qmax, qmax).
// Packing: int8 one byte per channel (two's complement); int4 two channels
// per byte, the even channel in the low nibble (two's complement nibbles).
// bits == 0: no quantisation; delta is returned exactly (double) in
// delta_exact and codes/scales are untouched.
// Returns 0, or 1 when a scale overflowed binary16.
// ---------------------------------------------------------------------------
// refs: stored reference values (fp32), as for orc_select_f.  The number of reference rows
// is not needed (idx addresses them).
int orc_encode_f(int D, int bits, int group, int64_t n_tok, const float* X, const float* refs, const uint16_t* idx,
                 int k, uint8_t* codes, uint16_t* scales, float* mean_out, float* delta_out, double* delta_exact)
{
    int overflow = 0;
    const int code_bytes = D * bits / 8;
    const int ngroups = D / group;
    std::vector<float> m(D), delta(D);
    for (int64_t t = 0; t < n_tok; ++t) {
        const uint16_t* id = idx + t * k;
        const int keff = count_keff(id, k);
        mean_reference(D, refs, id, keff, m.data());
        const float* x = X + t * D;
        for (int c = 0; c < D; ++c)
            delta[c] = x[c] - m[c];
        if (mean_out)
            std::memcpy(mean_out + t * D, m.data(), sizeof(float) * D);
        if (delta_out)
            std::memcpy(delta_out + t * D, delta.data(), sizeof(float) * D);
        if (bits == 0) {
            for (int c = 0; c < D; ++c)
                delta_exact[t * D + c] = static_cast<double>(x[c]) - static_cast<double>(m[c]);
            continue;
        }
        overflow |= quantize_groups(D, bits, group, delta.data(), codes + t * code_bytes, scales + t * ngroups);
    }
    return overflow;
}

int orc_encode(int D, int bits, int group, int64_t n_tok, const float* X, const uint16_t* refs, int64_t n_refs,
               const uint16_t* idx, int k, uint8_t* codes, uint16_t* scales, float* mean_out, float* delta_out,
               double* delta_exact)
{
    const std::vector<float> rf = widen_bf16(refs, n_refs * D);
    return orc_encode_f(D, bits, group, n_tok, X, rf.data(), idx, k, codes, scales, mean_out, delta_out,
                        delta_exact);
}

// ---------------------------------------------------------------------------
// Quantised rows (the int4 reference store: [P1] "Improvements for AI systems" and "Impact
// and Future Directions", full-pipeline quantisation applying 4-bit quantization uniformly
// to the compressed residuals and to the uncompressed components).  Each row of X is
// quantised by itself with the residuals' group quantiser, except that the scale is rounded
// up to a power of two (pow2 != 0): a 4-bit code times a power of two is then an exact bf16
// value, so the stored reference is the same number in every stage, the bf16 tensor-core
// search included.  The stored value of a channel is code * scale in fp32.
// ---------------------------------------------------------------------------
int orc_quantize_rows(int D, int bits, int group, int pow2, int64_t n, const float* X, uint8_t* codes,
                      uint16_t* scales)
{
    int overflow = 0;
    for (int64_t i = 0; i < n; ++i)
        overflow |= quantize_groups(D, bits, group, X + i * D, codes + i * (D * bits / 8), scales + i * (D / group),
                                    pow2 != 0);
    return overflow;
}

// Unpack one token's codes into integers.
void orc_unpack_codes(int D, int bits, const uint8_t* codes, int32_t* out)
{
    for (int c = 0; c < D; ++c) {
        if (bits == 8) {
            out[c] = static_cast<int8_t>(codes[c]);
        } else {
            int nib = (c & 1) ? (codes[c / 2] >> 4) & 0xf : codes[c / 2] & 0xf;
            out[c] = (nib >= 8) ? nib - 16 : nib;
        }
    }
}

// Stored values of quantised rows: code * scale (fp32).
void orc_dequantize_rows(int D, int bits, int group, int64_t n, const uint8_t* codes, const uint16_t* scales,
                         float* out)
{
    std::vector<int32_t> q(D);
    for (int64_t i = 0; i < n; ++i) {
        orc_unpack_codes(D, bits, codes + i * (D * bits / 8), q.data());
        for (int c = 0; c < D; ++c)
            out[i * D + c] = static_cast<float>(q[c]) * fp16_value(scales[i * (D / group) + c / group]);
    }
}

// ---------------------------------------------------------------------------
// Reconstruction ([P1] "DeltaKV Framework Architecture": the decoded residual
// plus the mean reference).  x_hat = m + code * scale in fp32.  bits == 0
// uses delta_exact: x_hat = m + delta (double, written to out_exact).
// ---------------------------------------------------------------------------
void orc_reconstruct_f(int D, int bits, int group, int64_t n_tok, const float* refs, const uint16_t* idx, int k,
                       const uint8_t* codes, const uint16_t* scales, const double* delta_exact, float* out,
                       double* out_exact)
{
    const int code_bytes = D * bits / 8;
    const int ngroups = (group > 0) ? D / group : 0;
    std::vector<float> m(D);
    std::vector<int32_t> q(D);
    for (int64_t t = 0; t < n_tok; ++t) {
        const uint16_t* id = idx + t * k;
        const int keff = count_keff(id, k);
        mean_reference(D, refs, id, keff, m.data());
        if (bits == 0) {
            for (int c = 0; c < D; ++c)
                out_exact[t * D + c] = static_cast<double>(m[c]) + delta_exact[t * D + c];
            continue;
        }
        orc_unpack_codes(D, bits, codes + t * code_bytes, q.data());
        for (int c = 0; c < D; ++c) {
            const float s = fp16_value(scales[t * ngroups + c / group]);
            const float d = static_cast<float>(q[c]) * s;
            out[t * D + c] = m[c] + d;
        }
    }
}

void orc_reconstruct(int D, int bits, int group, int64_t n_tok, const uint16_t* refs, int64_t n_refs,
                     const uint16_t* idx, int k, const uint8_t* codes, const uint16_t* scales,
                     const double* delta_exact, float* out, double* out_exact)
{
    const std::vector<float> rf = widen_bf16(refs, n_refs * D);
    orc_reconstruct_f(D, bits, group, n_tok, rf.data(), idx, k, codes, scales, delta_exact, out, out_exact);
}

// ---------------------------------------------------------------------------
// Attention of G query heads over n cached positions, all in double:
// l_i = (q . K_i) / sqrt(D); out = sum_i exp(l_i - max l) V_i / sum_i exp(l_i - max l).
// n == 0 writes zeros.
// ---------------------------------------------------------------------------
void orc_attention(int64_t n, int D, int G, const double* q, const double* K, const double* V, double* out)
{
    const double scale = 1.0 / std::sqrt(static_cast<double>(D));
    std::vector<double> l(static_cast<size_t>(n));
    for (int g = 0; g < G; ++g) {
        double* o = out + static_cast<int64_t>(g) * D;
        for (int c = 0; c < D; ++c)
            o[c] = 0.0;
        if (n == 0)
            continue;
        double mx = -INFINITY;
        for (int64_t i = 0; i < n; ++i) {
            double s = 0.0;
            for (int c = 0; c < D; ++c)
                s += q[g * D + c] * K[i * D + c];
            l[i] = s * scale;
            mx = std::max(mx, l[i]);
        }
        double den = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            const double p = std::exp(l[i] - mx);
            den += p;
            for (int c = 0; c < D; ++c)
                o[c] += p * V[i * D + c];
        }
        for (int c = 0; c < D; ++c)
            o[c] /= den;
    }
}

// Conversions exposed for the oracle's own pins.
uint16_t orc_fp16_round_up(float f, int32_t* overflow)
{
    int ov = 0;
    const uint16_t r = fp16_round_up(f, &ov);
    if (overflow)
        *overflow = ov;
    return r;
}

float orc_fp16_value(uint16_t h) { return fp16_value(h); }

// ---------------------------------------------------------------------------
// Learned-coder shapes ([P1] "DeltaKV Framework Architecture": the residual is taken after
// a compressor, z = fc(KV) - fc(KV_R), and a token is rebuilt as fd(z) + KV_R; "Improvements
// for AI systems": fc a SwiGLU block, fd a bias-free linear projection).  The weights are
// inputs (random in the tests; the trained ones are not available), row-major [out][in]:
//   fc(x) = Wo (silu(Wg x) * (Wu x)),  Wg, Wu [H][D], Wo [L][H],  silu(a) = a / (1 + e^-a)
//   fd(z) = Wd z,                      Wd [D][L]
// Everything in double from the exact inputs.  The latent residual is rounded to fp32 and
// then quantised by the residuals' group quantiser, with each group's scale rounded up to a
// power of two (as the int4 reference store's are): the pages fix no format for the coder's
// codes, and a power-of-two scale keeps the stored codes a reproducible function of a
// network output whose last bits depend on how it is evaluated (boundaries a factor of 2
// apart instead of 2^-10).
// ---------------------------------------------------------------------------
static void fc_apply(int D, int H, int L, const float* Wg, const float* Wu, const float* Wo, const double* x,
                     double* out)
{
    std::vector<double> h(H);
    for (int j = 0; j < H; ++j) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < D; ++c) {
            g += static_cast<double>(Wg[static_cast<int64_t>(j) * D + c]) * x[c];
            u += static_cast<double>(Wu[static_cast<int64_t>(j) * D + c]) * x[c];
        }
        h[j] = g / (1.0 + std::exp(-g)) * u;
    }
    for (int l = 0; l < L; ++l) {
        double acc = 0.0;
        for (int j = 0; j < H; ++j)
            acc += static_cast<double>(Wo[static_cast<int64_t>(l) * H + j]) * h[j];
        out[l] = acc;
    }
}

void orc_coder_fc(int D, int H, int L, int64_t n, const float* X, const float* Wg, const float* Wu, const float* Wo,
                  double* out)
{
    std::vector<double> x(D);
    for (int64_t t = 0; t < n; ++t) {
        for (int c = 0; c < D; ++c)
            x[c] = X[t * D + c];
        fc_apply(D, H, L, Wg, Wu, Wo, x.data(), out + t * L);
    }
}

// Latent residual codes: per token m = mean reference (fp32, as the identity coder forms
// it), z = fc(x) - fc(m) (double, rounded to fp32), then the group quantiser over the L
// latent channels with power-of-two scales.  z_out (optional) gets z in double.  Returns 1 on
// a binary16 overflow.
int orc_encode_latent(int D, int H, int L, int bits, int group, int64_t n_tok, const float* X, const float* refs,
                      const uint16_t* idx, int k, const float* Wg, const float* Wu, const float* Wo, uint8_t* codes,
                      uint16_t* scales, double* z_out)
{
    int overflow = 0;
    std::vector<float> m(D), zf(L);
    std::vector<double> xd(D), md(D), fx(L), fm(L);
    for (int64_t t = 0; t < n_tok; ++t) {
        const uint16_t* id = idx + t * k;
        mean_reference(D, refs, id, count_keff(id, k), m.data());
        for (int c = 0; c < D; ++c) {
            xd[c] = X[t * D + c];
            md[c] = m[c];
        }
        fc_apply(D, H, L, Wg, Wu, Wo, xd.data(), fx.data());
        fc_apply(D, H, L, Wg, Wu, Wo, md.data(), fm.data());
        for (int l = 0; l < L; ++l) {
            const double z = fx[l] - fm[l];
            if (z_out)
                z_out[t * L + l] = z;
            zf[l] = static_cast<float>(z);
        }
        if (bits > 0)
            overflow |= quantize_groups(L, bits, group, zf.data(), codes + t * (L * bits / 8), scales + t * (L / group),
                                        true);
    }
    return overflow;
}

// Rebuilt rows x = m + fd(z_hat) in double, z_hat = code * scale (or z_exact when bits == 0).
void orc_reconstruct_latent(int D, int L, int bits, int group, int64_t n_tok, const float* refs, const uint16_t* idx,
                            int k, const uint8_t* codes, const uint16_t* scales, const double* z_exact,
                            const float* Wd, double* out)
{
    std::vector<float> m(D);
    std::vector<int32_t> q(L);
    std::vector<double> zh(L);
    for (int64_t t = 0; t < n_tok; ++t) {
        const uint16_t* id = idx + t * k;
        mean_reference(D, refs, id, count_keff(id, k), m.data());
        if (bits == 0) {
            for (int l = 0; l < L; ++l)
                zh[l] = z_exact[t * L + l];
        } else {
            orc_unpack_codes(L, bits, codes + t * (L * bits / 8), q.data());
            for (int l = 0; l < L; ++l)
                zh[l] = static_cast<double>(q[l]) * fp16_value(scales[t * (L / group) + l / group]);
        }
        for (int c = 0; c < D; ++c) {
            double acc = m[c];
            for (int l = 0; l < L; ++l)
                acc += static_cast<double>(Wd[static_cast<int64_t>(c) * L + l]) * zh[l];
            out[t * D + c] = acc;
        }
    }
}

}  // extern "C"
