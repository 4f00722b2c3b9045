// nl_resort.cu -- re-sorting the atoms along the curve inside a rebuild.
//
// Tessera abstract: atoms are sorted along a space-filling curve so that
// neighbor search stays local as the system grows.  Over a long run atoms
// drift away from the order of the last sort; re-sorting at each rebuild
// keeps the array order on the Hilbert curve of the current positions.
// The caller's arrays are permuted in place (their device addresses are
// fixed inside a replayed graph): positions, and optionally an int32 id per
// atom and one float4 of per-atom state (velocities, say).  The sort is the
// same stable (key, slot) sort as nl_sort_hilbert.
#include "nl_internal.cuh"

namespace nl {
namespace {

// tmp[k] = src[perm[k]] for each array present.
__global__ void k_permute_gather(int64_t n, const uint32_t *__restrict__ perm,
                                 const float4 *__restrict__ pos, float4 *__restrict__ pos_tmp,
                                 const int32_t *__restrict__ ids, int32_t *__restrict__ ids_tmp,
                                 const float4 *__restrict__ aux, float4 *__restrict__ aux_tmp,
                                 const uint32_t *flags)
{
    if (timed_out(flags)) return;   // perm may not be a permutation
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride) {
        const uint32_t i = perm[k];
        pos_tmp[k] = pos[i];
        if (ids) ids_tmp[k] = ids[i];
        if (aux) aux_tmp[k] = aux[i];
    }
}

// src[k] = tmp[k] for each array present.
__global__ void k_permute_back(int64_t n, float4 *__restrict__ pos,
                               const float4 *__restrict__ pos_tmp, int32_t *__restrict__ ids,
                               const int32_t *__restrict__ ids_tmp, float4 *__restrict__ aux,
                               const float4 *__restrict__ aux_tmp, const uint32_t *flags)
{
    if (timed_out(flags)) return;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride) {
        pos[k] = pos_tmp[k];
        if (ids) ids[k] = ids_tmp[k];
        if (aux) aux[k] = aux_tmp[k];
    }
}

}  // namespace

cudaError_t launch_resort(nl_ctx *ctx, int64_t n, float4 *pos, int32_t *ids, float4 *aux,
                          float Lx, float Ly, float Lz, float Sx, float Sy, float Sz,
                          cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    NL_CUDA_TRY(cudaMemsetAsync(ctx->hist, 0, sizeof(uint32_t) * kKeyPasses * kRadixBins, s));
    {
        ProfScope ps(ctx, PH_KEYS, s);
        NL_CUDA_TRY(launch_keys(ctx, n, pos, Lx, Ly, Lz, Sx, Sy, Sz, 0, s));
    }
    {
        ProfScope ps(ctx, PH_KEY_SCAN, s);
        NL_CUDA_TRY(launch_hist_scan(ctx, s));
    }
    // the permutation goes to atom_rank; cell_pos, atom_cell and ref hold the
    // permuted copies.  All four are rewritten by the build that follows.
    uint32_t *perm = ctx->atom_rank;
    {
        ProfScope ps(ctx, PH_SORT, s);
        const SortRecompute rk{pos, n, Lx, Ly, Lz, Sx, Sy, Sz, 0};
        NL_CUDA_TRY(launch_radix_passes(ctx, n, nullptr, perm, s, rk));
    }
    {
        ProfScope ps(ctx, PH_GATHER, s);
        const unsigned blocks = resident_grid(ctx, k_permute_gather, 256, 0, (n + 255) / 256);
        int32_t *ids_tmp = reinterpret_cast<int32_t *>(ctx->atom_cell);
        k_permute_gather<<<(unsigned)blocks, 256, 0, s>>>(n, perm, pos, ctx->cell_pos, ids, ids_tmp,
                                                          aux, ctx->ref, ctx->flags);
        NL_CUDA_TRY(cudaGetLastError());
        k_permute_back<<<(unsigned)blocks, 256, 0, s>>>(n, pos, ctx->cell_pos, ids, ids_tmp, aux,
                                                        ctx->ref, ctx->flags);
        NL_CUDA_TRY(cudaGetLastError());
    }
    return cudaSuccess;
}

}  // namespace nl
