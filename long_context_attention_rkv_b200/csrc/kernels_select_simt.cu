// Reference search on CUDA cores (ResidualKV paper summary page, "DeltaKV
// Framework Architecture": top-k nearest references by L2 distance; "Practical
// Deployment via Sparse-vLLM": a batched L2 distance kernel for the search).
//
// |k - r|^2 = |k|^2 - 2 (k.r - |r|^2/2), and |k|^2 is the same for every
// candidate of a token, so ranking by largest t = k.r - |r|^2/2 is ranking by
// smallest distance.  This kernel keeps, per token, the kc largest t (ties to
// the lower ordinal) among the references at earlier positions; the encoder
// re-ranks the leading ones by exact fp32 distance.
//
// Used for fp32 inputs (exact fp32 products) and as a cross-check of the
// tensor-core search.  One CTA = one tile of 128 positions of one unit, one
// thread per position with its key row in registers; reference rows stream
// through shared memory in chunks of 64 and are read as broadcasts.
#include <cfloat>

#include "device_common.cuh"
#include "launchers.h"

namespace rkv {

namespace {

constexpr int kChunk = 64;

// Inserts (t, j) into the list sorted by (t descending, ordinal ascending).
template <int KC>
__device__ __forceinline__ void topk_insert(float (&tv)[KC], int (&ti)[KC], float t, int j)
{
    float cv = t;
    int ci = j;
#pragma unroll
    for (int s = 0; s < KC; ++s) {
        const bool before = (cv > tv[s]) || (cv == tv[s] && ci < ti[s]);
        const float ft = tv[s];
        const int it = ti[s];
        tv[s] = before ? cv : ft;
        ti[s] = before ? ci : it;
        cv = before ? ft : cv;
        ci = before ? it : ci;
    }
}

template <int D, int KC>
__global__ void __launch_bounds__(128) select_simt_kernel(CacheArgs a, const Tile* __restrict__ tiles,
                                                          const void* __restrict__ K, uint16_t* __restrict__ cand_idx,
                                                          float* __restrict__ cand_t)
{
    __shared__ __align__(16) float sr[kChunk][D];
    __shared__ float shn[kChunk];

    const Tile tl = tiles[blockIdx.x];
    const UnitMeta um = a.units[tl.unit];
    const int p0 = tl.tile * kPosTile;
    const int p = p0 + threadIdx.x;
    const bool in = p < um.n;
    const bool valid = in && !is_ref_pos(a.ph, p);
    const int ncand = valid ? refs_upto(a.ph, p) : 0;
    const int p_last = min(p0 + kPosTile, um.n) - 1;
    const int nc_max = min(refs_upto(a.ph, p_last), um.R);

    float x[D];
    if (valid) {
        const int64_t e = (static_cast<int64_t>(tl.unit) * a.max_len + p) * D;
#pragma unroll
        for (int c = 0; c < D; c += 4)
            load_row_part<4>(K, e + c, a.in_dtype, &x[c]);
    } else {
#pragma unroll
        for (int c = 0; c < D; ++c)
            x[c] = 0.0f;
    }

    float tv[KC];
    int ti[KC];
#pragma unroll
    for (int s = 0; s < KC; ++s) {
        tv[s] = -FLT_MAX;
        ti[s] = 0x7fffffff;
    }

    for (int j0 = 0; j0 < nc_max; j0 += kChunk) {
        __syncthreads();
        const int nrow = min(kChunk, nc_max - j0);
        for (int i = threadIdx.x; i < kChunk * D / 4; i += blockDim.x) {
            const int r = i / (D / 4);
            const int c = (i % (D / 4)) * 4;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (r < nrow)
                load_ref<4>(a, 0, um.ref_row + j0 + r, c, v);
            *reinterpret_cast<float4*>(&sr[r][c]) = make_float4(v[0], v[1], v[2], v[3]);
        }
        if (threadIdx.x < kChunk)
            shn[threadIdx.x] = (static_cast<int>(threadIdx.x) < nrow) ? a.ref_hn[um.ref_row + j0 + threadIdx.x] : 0.f;
        __syncthreads();
        const int jend = min(nrow, ncand - j0);
        for (int jj = 0; jj < jend; ++jj) {
            float dot = 0.0f;
#pragma unroll
            for (int c = 0; c < D; c += 4) {
                const float4 r4 = *reinterpret_cast<const float4*>(&sr[jj][c]);
                dot = fmaf(x[c], r4.x, dot);
                dot = fmaf(x[c + 1], r4.y, dot);
                dot = fmaf(x[c + 2], r4.z, dot);
                dot = fmaf(x[c + 3], r4.w, dot);
            }
            const float t = dot - shn[jj];
            if (t > tv[KC - 1])
                topk_insert<KC>(tv, ti, t, j0 + jj);
        }
    }

    if (valid) {
        const int64_t row = um.cmp_row + (p - ncand);
        const int nv = min(KC, ncand);
#pragma unroll
        for (int s = 0; s < KC; ++s) {
            cand_idx[row * KC + s] = (s < nv) ? static_cast<uint16_t>(ti[s]) : static_cast<uint16_t>(RKV_IDX_UNUSED);
            cand_t[row * KC + s] = (s < nv) ? tv[s] : -FLT_MAX;
        }
    }
}

template <int D>
cudaError_t launch_d(const CacheArgs& a, const Tile* tiles, int n_tiles, const void* K, uint16_t* ci, float* ct,
                     cudaStream_t st)
{
    switch (a.kc) {
    case 8: select_simt_kernel<D, 8><<<n_tiles, 128, 0, st>>>(a, tiles, K, ci, ct); break;
    case 12: select_simt_kernel<D, 12><<<n_tiles, 128, 0, st>>>(a, tiles, K, ci, ct); break;
    default: select_simt_kernel<D, 20><<<n_tiles, 128, 0, st>>>(a, tiles, K, ci, ct); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_simt(const CacheArgs& a, const Tile* tiles, int n_tiles, const void* K, uint16_t* cand_idx,
                               float* cand_t, cudaStream_t st)
{
    if (n_tiles <= 0)
        return cudaSuccess;
    return (a.D == 128) ? launch_d<128>(a, tiles, n_tiles, K, cand_idx, cand_t, st)
                        : launch_d<64>(a, tiles, n_tiles, K, cand_idx, cand_t, st);
}

}  // namespace rkv
