// Learned-coder shapes on the 5th-generation tensor cores: the latent residual of every
// compressed token (ResidualKV paper summary page, "DeltaKV Framework Architecture": the
// residual is taken after the compressor, z = fc(KV) - fc(KV_R); "Improvements for AI
// systems": fc a SwiGLU block).  fc(v) = Wo h(v), h(v) = silu(Wg v) * (Wu v), all weights bf16
// [128][128]; since Wo is linear, z = Wo (h(x) - h(m)), m the encoder's mean reference.
//
// One CTA of 16 warps per SM, persistent over 128-token tiles (all of a unit's tiles, then the
// next unit's).  Per tile:
//   1. the warps stage x (an exact bf16 operand) and e = x - m as a hi + mid + lo bf16 triple
//      (the 24 bits of fp32) in shared memory, K-major with the 128-byte swizzle; a half-warp
//      takes one token at a time, so every load reads a whole 256-byte row;
//   2. one thread issues the hidden layer as tcgen05 MMAs (M 128, N 128, K 16) into four
//      TMEM accumulators of 128 columns: g(x) = Wg x, u(x) = Wu x, Wg e, Wu e; forming g(m)
//      as g(x) - Wg e lets the accumulation error of g(x) cancel in h(x) - h(m) (forming g(m)
//      from m directly moved about 0.3 % of the groups' binary16 scales);
//   3. warp w reads the accumulators of TMEM lanes 32 (w % 4) .. + 31 (the lanes a warp may
//      read) for the quarter w / 4 of the hidden units, forms d = h(x) - h(m) and writes it as
//      another bf16 triple over the staging buffers;
//   4. one thread issues z = Wo d (three MMAs per K step) into the first accumulator;
//   5. every thread reads one 32-channel group of z of its token and quantises it: the
//      residuals' quantiser with the scale rounded up to a power of two (the learned coder's
//      code format); the whole group sits in one thread, so the group maximum needs no
//      shuffle.  A group whose a/7 lies within 2^-12 (relative) of a power of two, where the
//      tensor cores' fp32 evaluation of z could round the scale the other way than an exact
//      one, is listed for the exact pass.
// The exact pass (encode_latent_exact_kernel) recomputes the listed groups from scratch in
// double: h(x) and h(m) for all hidden units, then the group's 32 latent channels, rounded to
// fp32 and quantised; it overwrites the group's codes and scale.
// Every wait on an mbarrier is bounded; a wait that gives up records RKV_ERR_TIMEOUT and the
// CTA stops, freeing its TMEM.
#include <cfloat>

#include "device_common.cuh"
#include "launchers.h"
#include "sm100_ptx.cuh"

namespace rkv {

namespace {

using namespace sm100;

constexpr int kCD = 128;                       // head dim = hidden = latent width
constexpr int kCTile = 128;                    // tokens per tile (MMA M, TMEM lanes)
constexpr int kCThreads = 512;
constexpr uint32_t kCTileBytes = kCTile * kCD * 2;   // one K-major bf16 operand tile (two 64-column atoms)

struct CoderTcSmem {
    // A operands of the hidden layer (x, e hi / mid / lo); the second product's A operand
    // (d hi / mid / lo) reuses the first three
    uint8_t a[4][kCTileBytes];
    uint8_t w[3][kCTileBytes];                 // B operands: Wg, Wu, Wo ([n][k] = [out][in])
    uint64_t bar;
    uint32_t tmem_base;
    int abort;
};

// Byte offset of element (row, k) in a K-major 128-row bf16 tile stored as two 64-column atoms
// in the 128-byte-swizzle layout (16-byte chunk c of row r sits at chunk c ^ (r % 8)).
__device__ __forceinline__ uint32_t sw128_off(int row, int k)
{
    return static_cast<uint32_t>((k >> 6) * (kCTile * 128) + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4) +
                                 ((k & 7) << 1));
}

// Eight consecutive columns k0 .. k0 + 7 (k0 a multiple of 8) of one row: one 16-byte chunk.
__device__ __forceinline__ void put8(uint8_t* tile, int row, int k0, uint4 v)
{
    *reinterpret_cast<uint4*>(tile + sw128_off(row, k0)) = v;
}

// Two fp32 values x0, x1 as bf16 pairs hi + mid + lo (x0 in the low halves): each part is the
// top 16 bits of what is left (truncation), so hi, mid and lo take 8, 8 and 8 of the 24
// significant bits and their sum is x exactly; no conversion instruction is involved.
__device__ __forceinline__ void split3_pair(float x0, float x1, uint32_t& hi, uint32_t& mid, uint32_t& lo)
{
    const uint32_t a0 = __float_as_uint(x0), a1 = __float_as_uint(x1);
    hi = __byte_perm(a0, a1, 0x7632);
    const float r0 = x0 - __uint_as_float(a0 & 0xffff0000u), r1 = x1 - __uint_as_float(a1 & 0xffff0000u);
    const uint32_t b0 = __float_as_uint(r0), b1 = __float_as_uint(r1);
    mid = __byte_perm(b0, b1, 0x7632);
    const float s0 = r0 - __uint_as_float(b0 & 0xffff0000u), s1 = r1 - __uint_as_float(b1 & 0xffff0000u);
    lo = __byte_perm(__float_as_uint(s0), __float_as_uint(s1), 0x7632);
}

// silu(g) = g sigmoid(g); one exponential and one fast reciprocal (for g below about -88 the
// denominator is infinite and the quotient the right limit, -0).
__device__ __forceinline__ float silu_c(float g) { return __fdividef(g, 1.0f + expf(-g)); }

// Unit u and tile t0 within it of the CTA's tile number (tiles numbered unit by unit).
__device__ __forceinline__ void locate_tile(const CacheArgs& a, int tile, int& u, int& t0)
{
    u = 0;
    t0 = tile;
    while (u < a.n_units) {
        const int nt = (a.units[u].C + kCTile - 1) / kCTile;
        if (t0 < nt)
            break;
        t0 -= nt;
        ++u;
    }
}

// Every thread waits on the barrier (bounded); the CTA goes on only if all of them saw the phase
// complete, so that a wait that gave up ends the tile loop in all threads together.
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort)
{
    const bool w = mbar_wait(bar, parity, abort);
    if (!w)
        *abort = 1;
    return __syncthreads_and(w ? 1 : 0) != 0;
}

// Bits of the smallest binary16 power of two >= r (r > 0; 2^-24 at least), its value in *s and
// its exponent in *e; sets *over when it would exceed 2^15.
__device__ __forceinline__ uint16_t pow2_scale(float r, float* s, int* e, bool* over)
{
    int ex = 0;
    const float fr = frexpf(r, &ex);            // r = fr * 2^ex, fr in [0.5, 1)
    int E = (fr == 0.5f) ? ex - 1 : ex;         // smallest E with 2^E >= r
    E = max(E, -24);
    *over = E > 15;
    E = min(E, 15);
    *e = E;
    *s = ldexpf(1.0f, E);
    return (E >= -14) ? static_cast<uint16_t>((E + 15) << 10) : static_cast<uint16_t>(1u << (E + 24));
}

// Relative half-width of the band around a power of two inside which the exact pass decides a
// group's scale: far above the relative error of the tensor-core evaluation of a group maximum
// (a few 1e-6), and wide enough to cover it with margin.
constexpr float kLatentBand = 1.0f / 4096.0f;

// Entry of the exact pass's list: (unit | side << 24 | group << 28, compressed slot).
__device__ __forceinline__ int2 latent_entry(int u, int side, int g, int c)
{
    return make_int2(u | (side << 24) | (g << 28), c);
}

template <int SIDE>
__global__ void __launch_bounds__(kCThreads, 1) encode_latent_tc_kernel(CacheArgs a, const void* __restrict__ X,
                                                                         int total_tiles, int* __restrict__ flist)
{
    extern __shared__ uint8_t coder_raw[];
    const uint32_t raw_addr = smem_addr(coder_raw);
    CoderTcSmem& S = *reinterpret_cast<CoderTcSmem*>(coder_raw + ((1024 - (raw_addr & 1023)) & 1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int trow = 32 * (warp & 3) + (tid & 31);   // this thread's token in the tile = its TMEM lane
    const int cq = warp >> 2;                         // its quarter of the channels / units / groups
    volatile int* abort = &S.abort;

    if (warp == 0)
        tmem_alloc(&S.tmem_base, 512);
    if (tid == 0) {
        mbar_init(&S.bar, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    // the side's weights, once: row n of W is the B operand's row n (K-major)
    for (int i = tid; i < kCD * kCD / 8; i += kCThreads) {
        const int n = i / (kCD / 8), k0 = (i % (kCD / 8)) * 8;
#pragma unroll
        for (int m = 0; m < 3; ++m)
            put8(S.w[m], n, k0, reinterpret_cast<const uint4*>(a.cw[4 * SIDE + m])[i]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t lane_tm = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);   // this warp's TMEM lanes
    constexpr uint32_t idesc = idesc_bf16_f32(kCTile, kCD);
    const uint16_t* Xb = static_cast<const uint16_t*>(X);
    const uint16_t* refs = SIDE ? a.ref_V : a.ref_K;
    uint8_t* codes = SIDE ? a.codes_V : a.codes_K;
    uint16_t* scales = SIDE ? a.scale_V : a.scale_K;
    uint32_t phase = 0;
    bool ok = true;

    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        int u, t0;
        locate_tile(a, tile, u, t0);
        const UnitMeta um = a.units[u];
        const int c = t0 * kCTile + trow;           // this thread's token
        const bool valid = c < um.C;

        // ---- 1. x and e = x - m (hi, mid, lo): warp w stages the tile rows 8w .. 8w + 7, each
        //      half-warp two rows at a time; lane l of a half holds channels 8l .. 8l + 7, so that
        //      a half-warp load reads one whole 256-byte row, and the rows of a batch (x and four
        //      references of both tokens) are all requested before any is used
        {
            const int hl = lane & 15;
#pragma unroll 1
            for (int b = 0; b < 2; ++b) {
                const int r0 = 8 * warp + 4 * (lane >> 4) + 2 * b;
                int ord[2][8];
                int keff[2];
                uint4 xv[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int cj = t0 * kCTile + r0 + j;
                    keff[j] = 0;
                    xv[j] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int l = 0; l < 8; ++l)
                        ord[j][l] = 0;
                    if (cj < um.C) {
                        xv[j] = reinterpret_cast<const uint4*>(
                            Xb + (static_cast<int64_t>(u) * a.max_len + slot_pos(a.ph, cj)) * kCD)[hl];
                        const uint16_t* id = a.idx + (um.cmp_row + cj) * a.k;
#pragma unroll
                        for (int l = 0; l < 8; ++l)
                            ord[j][l] = (l < a.k) ? static_cast<int>(id[l]) : RKV_IDX_UNUSED;
                        int ke = 0;
#pragma unroll
                        for (int l = 0; l < 8; ++l)
                            ke += (ke == l && ord[j][l] != RKV_IDX_UNUSED && ord[j][l] < um.R) ? 1 : 0;
                        keff[j] = ke;
                    }
                }
                const int kmax = max(keff[0], keff[1]);
                float m[2][8];
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        m[j][i] = 0.0f;
#pragma unroll
                for (int lb = 0; lb < 8; lb += 4) {   // four reference rows of both tokens in flight
                    if (lb < kmax) {
                        uint4 rv[2][4];
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int l = 0; l < 4; ++l)
                                if (lb + l < keff[j])
                                    rv[j][l] =
                                        reinterpret_cast<const uint4*>(refs + (um.ref_row + ord[j][lb + l]) * kCD)[hl];
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int l = 0; l < 4; ++l)
                                if (lb + l < keff[j]) {
                                    const uint32_t w[4] = {rv[j][l].x, rv[j][l].y, rv[j][l].z, rv[j][l].w};
#pragma unroll
                                    for (int i = 0; i < 4; ++i) {
                                        const float r0v = __uint_as_float(w[i] << 16);
                                        const float r1v = __uint_as_float(w[i] & 0xffff0000u);
                                        m[j][2 * i] = (lb + l == 0) ? r0v : __fadd_rn(m[j][2 * i], r0v);
                                        m[j][2 * i + 1] = (lb + l == 0) ? r1v : __fadd_rn(m[j][2 * i + 1], r1v);
                                    }
                                }
                    }
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    // the mean: the sum times the rounded reciprocal of the count (exact for 1, 2, 4
                    // and 8 references); a row past the unit's tokens has no reference and e = x
                    const float inv = keff[j] > 0 ? __frcp_rn(static_cast<float>(keff[j])) : 0.0f;
                    const uint32_t w[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
                    uint32_t eh[4], em[4], el[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        split3_pair(__fsub_rn(__uint_as_float(w[i] << 16), __fmul_rn(m[j][2 * i], inv)),
                                    __fsub_rn(__uint_as_float(w[i] & 0xffff0000u), __fmul_rn(m[j][2 * i + 1], inv)),
                                    eh[i], em[i], el[i]);
                    put8(S.a[0], r0 + j, 8 * hl, xv[j]);
                    put8(S.a[1], r0 + j, 8 * hl, make_uint4(eh[0], eh[1], eh[2], eh[3]));
                    put8(S.a[2], r0 + j, 8 * hl, make_uint4(em[0], em[1], em[2], em[3]));
                    put8(S.a[3], r0 + j, 8 * hl, make_uint4(el[0], el[1], el[2], el[3]));
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- 2. hidden layer: four accumulators of 128 columns ---------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t wg = smem_addr(S.w[0]), wu = smem_addr(S.w[1]);
#pragma unroll
            for (int kk = 0; kk < kCD / 16; ++kk) {
                const uint32_t off = (kk / 4) * (kCTile * 128) + (kk % 4) * 32;
                const uint32_t acc = kk > 0 ? 1u : 0u;
                const uint64_t dg = smem_desc_sw128(wg + off), du = smem_desc_sw128(wu + off);
                mma_f16(tmem + 0, smem_desc_sw128(smem_addr(S.a[0]) + off), dg, idesc, acc);
                mma_f16(tmem + 128, smem_desc_sw128(smem_addr(S.a[0]) + off), du, idesc, acc);
#pragma unroll
                for (int part = 1; part <= 3; ++part) {
                    const uint64_t de = smem_desc_sw128(smem_addr(S.a[part]) + off);
                    mma_f16(tmem + 256, de, dg, idesc, (kk > 0 || part > 1) ? 1u : 0u);
                    mma_f16(tmem + 384, de, du, idesc, (kk > 0 || part > 1) ? 1u : 0u);
                }
            }
            mma_commit(&S.bar);
        }
        if (!wait_all(&S.bar, phase, abort)) {
            ok = false;
            break;
        }
        phase ^= 1u;
        tc_fence_after();

        // ---- 3. d = h(x) - h(m) of the thread's 32 units, 16 at a time, as bf16 hi / mid / lo
        //      over the staging buffers
#pragma unroll 1
        for (int q = 0; q < 2; ++q) {
            const int col = 32 * cq + 16 * q;
            float gx[16], ux[16], ge[16], ue[16];
            tmem_ld16(lane_tm + 0 + col, gx);
            tmem_ld16(lane_tm + 128 + col, ux);
            tmem_ld16(lane_tm + 256 + col, ge);
            tmem_ld16(lane_tm + 384 + col, ue);
#pragma unroll
            for (int j0 = 0; j0 < 16; j0 += 8) {
                uint32_t dh[4], dm[4], dl[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int j = j0 + 2 * i + h;
                        v[h] = silu_c(gx[j]) * ux[j] - silu_c(gx[j] - ge[j]) * (ux[j] - ue[j]);
                    }
                    split3_pair(v[0], v[1], dh[i], dm[i], dl[i]);
                }
                put8(S.a[0], trow, col + j0, make_uint4(dh[0], dh[1], dh[2], dh[3]));
                put8(S.a[1], trow, col + j0, make_uint4(dm[0], dm[1], dm[2], dm[3]));
                put8(S.a[2], trow, col + j0, make_uint4(dl[0], dl[1], dl[2], dl[3]));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- 4. z = Wo d into the first accumulator ---------------------------------------
        if (tid == 0) {
            tc_fence_after();
            const uint32_t wo = smem_addr(S.w[2]);
#pragma unroll
            for (int kk = 0; kk < kCD / 16; ++kk) {
                const uint32_t off = (kk / 4) * (kCTile * 128) + (kk % 4) * 32;
                const uint64_t db = smem_desc_sw128(wo + off);
#pragma unroll
                for (int part = 0; part < 3; ++part)
                    mma_f16(tmem + 0, smem_desc_sw128(smem_addr(S.a[part]) + off), db, idesc,
                            (kk > 0 || part > 0) ? 1u : 0u);
            }
            mma_commit(&S.bar);
        }
        if (!wait_all(&S.bar, phase, abort)) {
            ok = false;
            break;
        }
        phase ^= 1u;
        tc_fence_after();

        // ---- 5. the quantiser on the thread's 32-channel group of z (power-of-two scale) -------
        {
            const int qmax = (a.bits == 8) ? 127 : 7;
            const int64_t row = um.cmp_row + (valid ? c : 0);
            float z[32];
            tmem_ld32(lane_tm + 32 * cq, z);
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                amax = fmaxf(amax, fabsf(z[i]));
            uint16_t sbits = 0;
            float inv = 0.0f;
            if (amax > 0.0f) {
                const float r = __fdiv_rn(amax, static_cast<float>(qmax));
                float sc, slo, shi;
                int e, elo, ehi;
                bool over, o2;
                sbits = pow2_scale(r, &sc, &e, &over);
                pow2_scale(r * (1.0f - kLatentBand), &slo, &elo, &o2);
                pow2_scale(r * (1.0f + kLatentBand), &shi, &ehi, &o2);
                if (valid && over)
                    report(a.err, RKV_ERR_UNSUPPORTED);
                if (valid && elo != ehi) {
                    // the scale could round the other way in an exact evaluation: the exact pass
                    // decides this group
                    const int slot = atomicAdd(flist, 1);
                    reinterpret_cast<int2*>(flist + 2)[slot] = latent_entry(u, SIDE, cq, c);
                }
                inv = ldexpf(1.0f, -e);   // exact: 1 / s for a power of two s
            }
            // code = rint(z / s): z times 1/s is exact (a power of two), and the addition of
            // 1.5 * 2^23 in the same fused operation rounds it half to even
            constexpr float kRound = 12582912.0f;
            constexpr int kRoundBits = 0x4B400000;
            uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int qv = max(-qmax, min(qmax, __float_as_int(__fmaf_rn(z[i], inv, kRound)) - kRoundBits));
                w[i >> 3] |= static_cast<uint32_t>(qv & 0xf) << (4 * (i & 7));
            }
            if (valid) {
                *reinterpret_cast<uint4*>(codes + row * a.code_bytes + 16 * cq) = make_uint4(w[0], w[1], w[2], w[3]);
                scales[row * a.n_groups + cq] = sbits;
            }
        }
        tc_fence_before();
        __syncthreads();   // TMEM and the staging buffers are reused by the next tile
    }
    if (!ok && tid == 0)
        report(a.err, RKV_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
        tmem_relinquish();
    }
}

// The exact pass: one block of 128 threads per listed (token, side, group).  Thread j forms
// hidden unit j of x and of m in double (g = Wg v, u = Wu v, h = silu(g) u); the first warp then
// forms the group's 32 latent channels z = Wo h(x) - Wo h(m), rounds them to fp32 and quantises
// them (power-of-two scale), overwriting the fast pass's codes and scale of the group.  m is the
// mean reference as the oracle defines it: the fp32 sum in ascending ordinal order, divided by
// k_eff.  The double evaluation is exact to far below fp32 rounding, so the result equals an
// exact evaluation's except where z or a/7 sits within about 1e-15 of a rounding boundary.
constexpr int kExactThreads = 128;

__global__ void __launch_bounds__(kExactThreads) encode_latent_exact_kernel(CacheArgs a, const void* __restrict__ K,
                                                                             const void* __restrict__ V,
                                                                             const int* __restrict__ flist)
{
    __shared__ double xs[kCD], ms[kCD], hx[kCD], hm[kCD];
    const int n = *reinterpret_cast<const volatile int*>(flist);
    const int2* list = reinterpret_cast<const int2*>(flist + 2);
    const int tid = threadIdx.x;
    for (int e = blockIdx.x; e < n; e += gridDim.x) {
        const int2 en = list[e];
        const int u = en.x & 0xffffff, side = (en.x >> 24) & 1, g = (en.x >> 28) & 3, c = en.y;
        const UnitMeta um = a.units[u];
        const int64_t row = um.cmp_row + c;
        const uint16_t* Xb = static_cast<const uint16_t*>(side ? V : K);
        const uint16_t* refs = side ? a.ref_V : a.ref_K;
        const uint16_t* id = a.idx + row * a.k;
        __syncthreads();   // the previous entry's shared values are consumed
        {
            const int ch = tid;   // kExactThreads == kCD: one channel per thread
            xs[ch] = static_cast<double>(
                bf16_bits_to_f32(Xb[(static_cast<int64_t>(u) * a.max_len + slot_pos(a.ph, c)) * kCD + ch]));
            float acc = 0.0f;
            int keff = 0;
            for (int l = 0; l < a.k; ++l) {
                const int o = id[l];
                if (o == RKV_IDX_UNUSED || o >= um.R)
                    break;
                const float r = bf16_bits_to_f32(refs[(um.ref_row + o) * kCD + ch]);
                acc = (keff == 0) ? r : __fadd_rn(acc, r);
                ++keff;
            }
            ms[ch] = static_cast<double>(keff > 0 ? __fdiv_rn(acc, static_cast<float>(keff)) : 0.0f);
        }
        __syncthreads();
        {
            const int j = tid;    // hidden unit
            const uint16_t* Wg = a.cw[4 * side + 0] + j * kCD;
            const uint16_t* Wu = a.cw[4 * side + 1] + j * kCD;
            double gx = 0.0, ux = 0.0, gm = 0.0, um2 = 0.0;
            // the thread's rows of Wg and Wu, eight weights per 16-byte load (the lanes read
            // different rows); the products are summed in channel order as before
            for (int c8 = 0; c8 < kCD; c8 += 8) {
                const uint4 g8 = *reinterpret_cast<const uint4*>(Wg + c8);
                const uint4 u8 = *reinterpret_cast<const uint4*>(Wu + c8);
                const uint32_t gw[4] = {g8.x, g8.y, g8.z, g8.w}, uw[4] = {u8.x, u8.y, u8.z, u8.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int ch = c8 + i;
                    const double wg = bf16_bits_to_f32((i & 1) ? (gw[i >> 1] >> 16) : (gw[i >> 1] & 0xffffu));
                    const double wu = bf16_bits_to_f32((i & 1) ? (uw[i >> 1] >> 16) : (uw[i >> 1] & 0xffffu));
                    gx = fma(wg, xs[ch], gx);
                    ux = fma(wu, xs[ch], ux);
                    gm = fma(wg, ms[ch], gm);
                    um2 = fma(wu, ms[ch], um2);
                }
            }
            hx[j] = gx / (1.0 + exp(-gx)) * ux;
            hm[j] = gm / (1.0 + exp(-gm)) * um2;
        }
        __syncthreads();
        if (tid < 32) {
            const int l = 32 * g + tid;   // latent channel
            const uint16_t* Wo = a.cw[4 * side + 2] + l * kCD;
            double fx = 0.0, fm = 0.0;
            for (int j8 = 0; j8 < kCD; j8 += 8) {
                const uint4 o8 = *reinterpret_cast<const uint4*>(Wo + j8);
                const uint32_t ow[4] = {o8.x, o8.y, o8.z, o8.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const double w = bf16_bits_to_f32((i & 1) ? (ow[i >> 1] >> 16) : (ow[i >> 1] & 0xffffu));
                    fx = fma(w, hx[j8 + i], fx);
                    fm = fma(w, hm[j8 + i], fm);
                }
            }
            const float z = static_cast<float>(fx - fm);
            float amax = fabsf(z);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const int qmax = (a.bits == 8) ? 127 : 7;
            uint16_t sbits = 0;
            int q = 0;
            if (amax > 0.0f) {
                float sc;
                int ex;
                bool over;
                sbits = pow2_scale(__fdiv_rn(amax, static_cast<float>(qmax)), &sc, &ex, &over);
                if (over)
                    report(a.err, RKV_ERR_UNSUPPORTED);
                q = max(-qmax, min(qmax, static_cast<int>(rintf(z * ldexpf(1.0f, -ex)))));
            }
            // pack: lane pairs (2i, 2i + 1) form byte i of the group's 16 code bytes
            const uint32_t nib = static_cast<uint32_t>(q & 0xf);
            const uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
            uint8_t* codes = (side ? a.codes_V : a.codes_K) + row * a.code_bytes + 16 * g;
            if ((tid & 1) == 0)
                codes[tid >> 1] = static_cast<uint8_t>(nib | (other << 4));
            if (tid == 0)
                (side ? a.scale_V : a.scale_K)[row * a.n_groups + g] = sbits;
        }
    }
}

}  // namespace

int encode_latent_tiles(int C) { return (C + kCTile - 1) / kCTile; }

uint64_t encode_latent_list_bytes(int64_t cmp_rows) { return 8ull + 8ull * 8ull * static_cast<uint64_t>(cmp_rows); }

cudaError_t launch_encode_latent(const CacheArgs& a, const void* K, const void* V, int total_tiles, int* flist,
                                 cudaStream_t st)
{
    if (a.D != kCD || a.in_dtype != RKV_DTYPE_BF16 || a.bits != 4)
        return cudaErrorNotSupported;
    if (total_tiles <= 0)
        return cudaSuccess;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const size_t smem = sizeof(CoderTcSmem) + 1024;
    const int grid = total_tiles < sms ? total_tiles : sms;
    e = cudaFuncSetAttribute(encode_latent_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(encode_latent_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    e = cudaMemsetAsync(flist, 0, sizeof(int), st);
    if (e != cudaSuccess)
        return e;
    encode_latent_tc_kernel<0><<<grid, kCThreads, smem, st>>>(a, K, total_tiles, flist);
    encode_latent_tc_kernel<1><<<grid, kCThreads, smem, st>>>(a, V, total_tiles, flist);
    // the listed groups (a small share): a few blocks per SM stride over the list
    encode_latent_exact_kernel<<<4 * sms, kExactThreads, 0, st>>>(a, K, V, flist);
    return cudaGetLastError();
}

}  // namespace rkv
