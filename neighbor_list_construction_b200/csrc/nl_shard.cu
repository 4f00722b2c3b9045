// nl_shard.cu -- halo selection for equal-count shards along the curve.
//
// Tessera abstract: atoms are sorted along a space-filling curve and cut
// into equal-count shards, one per GPU; each GPU needs, besides its own
// atoms, every atom within the search radius of them (its halo).  The halo
// is found on a coarse periodic grid whose cells are at least rl wide, so
// two atoms within rl lie in the same or in adjacent coarse cells:
//   1. each rank marks the coarse cells its atoms occupy with its rank bit;
//   2. the marks are summed over ranks (an all-reduce; distinct bits, so the
//      sum is the bitwise or) -- occupied-by masks per coarse cell;
//   3. needed[c] = or of the masks over the 27 cells around c;
//   4. an atom in cell c is sent to every rank q != self with bit q in
//      needed[c] (count, then fill), and the ranks exchange those atoms.
// Positions carry the atom's global id in the fourth lane (int32 bits), so
// rows built over own + halo atoms map back to global ids.
#include <cmath>

#include "nl_internal.cuh"
#include "nl_shard.h"

namespace nl {
namespace {

__device__ __forceinline__ int coarse_cell(const float4 p, float Lx, float Ly, float Lz, float Tx,
                                           float Ty, float Tz, int nx, int ny, int nz)
{
    const int cx = cell_coord(wrap_coord(p.x, Lx), Tx, nx);
    const int cy = cell_coord(wrap_coord(p.y, Ly), Ty, ny);
    const int cz = cell_coord(wrap_coord(p.z, Lz), Tz, nz);
    return (cz * ny + cy) * nx + cx;
}

struct Coarse {
    float Lx, Ly, Lz, Tx, Ty, Tz;
    int nx, ny, nz;
};

__global__ void k_halo_mark(const float4 *__restrict__ pos, int64_t n, Coarse C, uint32_t bit,
                            int32_t *__restrict__ occ)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int c = coarse_cell(pos[i], C.Lx, C.Ly, C.Lz, C.Tx, C.Ty, C.Tz, C.nx, C.ny, C.nz);
        occ[c] = (int32_t)bit;   // every writer stores the same value
    }
}

__global__ void k_halo_needed(Coarse C, const int32_t *__restrict__ occ, int32_t *__restrict__ need)
{
    const int64_t nc = (int64_t)C.nx * C.ny * C.nz;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < nc; c += stride) {
        const int cx = (int)(c % C.nx);
        const int cy = (int)((c / C.nx) % C.ny);
        const int cz = (int)(c / ((int64_t)C.nx * C.ny));
        uint32_t m = 0u;
        for (int dz = -1; dz <= 1; ++dz) {
            const int z = (cz + dz + C.nz) % C.nz;
            for (int dy = -1; dy <= 1; ++dy) {
                const int y = (cy + dy + C.ny) % C.ny;
                for (int dx = -1; dx <= 1; ++dx) {
                    const int x = (cx + dx + C.nx) % C.nx;
                    m |= (uint32_t)occ[((int64_t)z * C.ny + y) * C.nx + x];
                }
            }
        }
        need[c] = (int32_t)m;
    }
}

// counts[q] += atoms of this rank that rank q needs (q != rank); one atomic
// per destination and warp.
__global__ void k_halo_count(const float4 *__restrict__ pos, int64_t n, Coarse C,
                             const int32_t *__restrict__ need, int rank, int nranks,
                             int32_t *__restrict__ counts)
{
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t n_up = (n + 31) & ~int64_t(31);   // whole warps take part in the votes
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_up; i += stride) {
        uint32_t m = 0u;
        if (i < n) {
            const int c =
                coarse_cell(pos[i], C.Lx, C.Ly, C.Lz, C.Tx, C.Ty, C.Tz, C.nx, C.ny, C.nz);
            m = (uint32_t)need[c] & ~(1u << rank);
        }
        for (int q = 0; q < nranks; ++q) {
            const uint32_t b = __ballot_sync(0xffffffffu, (m >> q) & 1u);
            if (lane == 0 && b) atomicAdd(&counts[q], __popc(b));
        }
    }
}

// Writes the atoms counted by k_halo_count to send[offset[q] + k], k from
// the cursor of q (zero before); order inside a destination is arbitrary.
// block > 0: fixed blocks instead, destination q at q * block, at most
// `block` atoms each; a count above it raises kFlagHalo in flags.
__global__ void k_halo_fill(const float4 *__restrict__ pos, int64_t n, Coarse C,
                            const int32_t *__restrict__ need, int rank, int nranks,
                            const int32_t *__restrict__ offset, const int32_t *__restrict__ counts,
                            int32_t *__restrict__ cursor, float4 *__restrict__ send, int32_t block,
                            uint32_t *flags)
{
    if (block > 0 && blockIdx.x == 0 && threadIdx.x < (unsigned)nranks &&
        counts[threadIdx.x] > block)
        atomicOr(flags, kFlagHalo);
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t n_up = (n + 31) & ~int64_t(31);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_up; i += stride) {
        uint32_t m = 0u;
        float4 p = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (i < n) {
            p = pos[i];
            const int c = coarse_cell(p, C.Lx, C.Ly, C.Lz, C.Tx, C.Ty, C.Tz, C.nx, C.ny, C.nz);
            m = (uint32_t)need[c] & ~(1u << rank);
        }
        for (int q = 0; q < nranks; ++q) {
            const bool mine = (m >> q) & 1u;
            const uint32_t b = __ballot_sync(0xffffffffu, mine);
            if (!b) continue;
            const int leader = __ffs(b) - 1;
            int32_t base = 0;
            if (lane == leader) base = atomicAdd(&cursor[q], __popc(b));
            base = __shfl_sync(0xffffffffu, base, leader);
            const int32_t k = base + __popc(b & lanemask_lt());
            // k < counts[q] unless the inputs changed since k_halo_count
            if (block > 0) {
                if (mine && k < counts[q] && k < block) send[(int64_t)q * block + k] = p;
            } else if (mine && k < counts[q]) {
                send[offset[q] + k] = p;
            }
        }
    }
}

// Appends the received blocks to the own atoms: block q (recv[q * block ..])
// holds min(recv_counts[q], block) atoms, which go to pos_all after the
// n_own own atoms and the blocks before q; the total lands in *n_all_out.
// A count above `block`, or a total above n_max, raises kFlagHalo (atoms
// past n_max are dropped).
__global__ void k_halo_pack(int nranks, int32_t block, const int32_t *__restrict__ recv_counts,
                            const float4 *__restrict__ recv, int64_t n_own, int64_t n_max,
                            float4 *__restrict__ pos_all, int64_t *n_all_out, uint32_t *flags)
{
    __shared__ int64_t s_off[33];
    if (threadIdx.x == 0) {
        int64_t off = 0;
        bool bad = false;
        for (int q = 0; q < nranks; ++q) {
            const int32_t c = recv_counts[q];
            bad |= c > block || c < 0;
            s_off[q] = off;
            off += c < 0 ? 0 : (c < block ? c : block);
        }
        s_off[nranks] = off;
        if (n_own + off > n_max) bad = true;
        if (bad && blockIdx.x == 0) atomicOr(flags, kFlagHalo);
        if (blockIdx.x == 0) *n_all_out = n_own + off < n_max ? n_own + off : n_max;
    }
    __syncthreads();
    const int64_t total = (int64_t)nranks * block;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
        const int q = (int)(e / block);
        const int32_t k = (int32_t)(e - (int64_t)q * block);
        const int64_t c = s_off[q + 1] - s_off[q];
        const int64_t dst = n_own + s_off[q] + k;
        if (k < c && dst < n_max) pos_all[dst] = recv[e];
    }
}

// Row entries (indices into pos_all) replaced by the global ids in the
// fourth lane of pos_all; -1 stays.  With counts, a warp takes a row and
// maps its first min(count, K) entries only (the rest is -1).
__global__ void k_map_ids(int64_t entries, int32_t *__restrict__ nbr, const float4 *__restrict__ pos_all,
                          int64_t n_all)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < entries; e += stride) {
        const int32_t j = nbr[e];
        if (j >= 0 && j < n_all) nbr[e] = __float_as_int(pos_all[j].w);
    }
}

__global__ void k_map_ids_rows(int64_t n_rows, int32_t K, int32_t *__restrict__ nbr,
                               const int32_t *__restrict__ counts,
                               const float4 *__restrict__ pos_all, int64_t n_all)
{
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n_rows; i += nw) {
        int32_t c = counts[i];
        c = c < K ? c : K;
        int32_t *row = nbr + i * (int64_t)K;
        for (int32_t s = lane; s < c; s += 32) {
            const int32_t j = row[s];
            if (j >= 0 && j < n_all) row[s] = __float_as_int(pos_all[j].w);
        }
    }
}

bool make_coarse(const float *box, const int32_t dims[3], Coarse *C)
{
    if (!box || !dims) return false;
    for (int a = 0; a < 3; ++a)
        if (!(std::isfinite(box[a]) && box[a] > 0.0f) || dims[a] < 1 || dims[a] > 1024) return false;
    C->Lx = box[0];
    C->Ly = box[1];
    C->Lz = box[2];
    volatile float tx = (float)dims[0] / box[0];
    volatile float ty = (float)dims[1] / box[1];
    volatile float tz = (float)dims[2] / box[2];
    C->Tx = tx;
    C->Ty = ty;
    C->Tz = tz;
    C->nx = dims[0];
    C->ny = dims[1];
    C->nz = dims[2];
    return (int64_t)dims[0] * dims[1] * dims[2] <= (int64_t(1) << 30);
}

}  // namespace
}  // namespace nl

using namespace nl;

extern "C" {

nl_status nl_halo_grid(const float *box, float cutoff, float skin, int32_t dims_out[3])
{
    if (!box || !dims_out || !std::isfinite(cutoff) || !std::isfinite(skin) || cutoff < 0.0f ||
        skin < 0.0f)
        return NL_ERR_ARG;
    volatile float rl = cutoff + skin;
    if (!(rl > 0.0f)) return NL_ERR_ARG;
    for (int a = 0; a < 3; ++a) {
        if (!(std::isfinite(box[a]) && box[a] > 0.0f)) return NL_ERR_ARG;
        // cells wider than rl by a margin (2^-10 rl + 2^-16 L) far above the
        // fp32 rounding of floor(w * dims / L) for dims <= 1024, so atoms
        // within rl always fall in the same or adjacent cells
        const double L = box[a];
        double m = std::floor(L / ((double)rl * (1.0 + std::ldexp(1.0, -10)) + L * std::ldexp(1.0, -16)));
        if (m < 1.0) m = 1.0;
        if (m > 1024.0) m = 1024.0;
        dims_out[a] = (int32_t)m;
    }
    return NL_OK;
}

nl_status nl_halo_mark(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                       const int32_t dims[3], int32_t rank, int32_t *occ_out, void *stream)
{
    Coarse C;
    if (!ctx || n < 0 || rank < 0 || rank >= 32 || !occ_out || !make_coarse(box, dims, &C))
        return NL_ERR_ARG;
    if (n > 0 && (!pos || (reinterpret_cast<uintptr_t>(pos) & 15u))) return NL_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t nc = (int64_t)C.nx * C.ny * C.nz;
    if (cudaMemsetAsync(occ_out, 0, sizeof(int32_t) * nc, s) != cudaSuccess) return NL_ERR_CUDA;
    if (n > 0)
        k_halo_mark<<<resident_grid(ctx, k_halo_mark, 256, 0, (n + 255) / 256), 256, 0, s>>>(
            reinterpret_cast<const float4 *>(pos), n, C, 1u << rank, occ_out);
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

nl_status nl_halo_needed(nl_ctx *ctx, const float *box, const int32_t dims[3],
                         const int32_t *occ_all, int32_t *need_out, void *stream)
{
    Coarse C;
    if (!ctx || !occ_all || !need_out || !make_coarse(box, dims, &C)) return NL_ERR_ARG;
    const int64_t nc = (int64_t)C.nx * C.ny * C.nz;
    k_halo_needed<<<resident_grid(ctx, k_halo_needed, 256, 0, (nc + 255) / 256), 256, 0,
                    reinterpret_cast<cudaStream_t>(stream)>>>(
        C, occ_all, need_out);
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

nl_status nl_halo_count(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                        const int32_t dims[3], const int32_t *need, int32_t rank, int32_t nranks,
                        int32_t *counts_out, void *stream)
{
    Coarse C;
    if (!ctx || n < 0 || nranks < 1 || nranks > 32 || rank < 0 || rank >= nranks || !need ||
        !counts_out || !make_coarse(box, dims, &C))
        return NL_ERR_ARG;
    if (n > 0 && (!pos || (reinterpret_cast<uintptr_t>(pos) & 15u))) return NL_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * nranks, s) != cudaSuccess)
        return NL_ERR_CUDA;
    if (n > 0)
        k_halo_count<<<resident_grid(ctx, k_halo_count, 256, 0, (n + 255) / 256), 256, 0, s>>>(
            reinterpret_cast<const float4 *>(pos), n, C, need, rank, nranks, counts_out);
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

nl_status nl_halo_fill(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                       const int32_t dims[3], const int32_t *need, int32_t rank, int32_t nranks,
                       const int32_t *offsets, const int32_t *counts, int32_t *cursor,
                       float *send_out, void *stream)
{
    Coarse C;
    if (!ctx || n < 0 || nranks < 1 || nranks > 32 || rank < 0 || rank >= nranks || !need ||
        !offsets || !counts || !cursor || !make_coarse(box, dims, &C))
        return NL_ERR_ARG;
    if (n > 0 && (!pos || (reinterpret_cast<uintptr_t>(pos) & 15u))) return NL_ERR_ARG;
    if (send_out && (reinterpret_cast<uintptr_t>(send_out) & 15u)) return NL_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(cursor, 0, sizeof(int32_t) * nranks, s) != cudaSuccess) return NL_ERR_CUDA;
    if (n > 0 && send_out)
        k_halo_fill<<<resident_grid(ctx, k_halo_fill, 256, 0, (n + 255) / 256), 256, 0, s>>>(
            reinterpret_cast<const float4 *>(pos), n, C, need, rank, nranks, offsets, counts,
            cursor, reinterpret_cast<float4 *>(send_out), 0, ctx->flags);
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

nl_status nl_halo_fill_blocks(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                              const int32_t dims[3], const int32_t *need, int32_t rank,
                              int32_t nranks, int32_t block, const int32_t *counts,
                              int32_t *cursor, float *send_out, void *stream)
{
    Coarse C;
    if (!ctx || n < 0 || nranks < 1 || nranks > 32 || rank < 0 || rank >= nranks || block < 1 ||
        !need || !counts || !cursor || !send_out || !make_coarse(box, dims, &C))
        return NL_ERR_ARG;
    if (n > 0 && (!pos || (reinterpret_cast<uintptr_t>(pos) & 15u))) return NL_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(send_out) & 15u) return NL_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(cursor, 0, sizeof(int32_t) * nranks, s) != cudaSuccess) return NL_ERR_CUDA;
    const int64_t want = n > 0 ? (n + 255) / 256 : 1;
    k_halo_fill<<<resident_grid(ctx, k_halo_fill, 256, 0, want), 256, 0, s>>>(
        reinterpret_cast<const float4 *>(pos), n, C, need, rank, nranks, nullptr, counts, cursor,
        reinterpret_cast<float4 *>(send_out), block, ctx->flags);
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

nl_status nl_halo_pack(nl_ctx *ctx, int32_t nranks, int32_t block, const int32_t *recv_counts,
                       const float *recv, int64_t n_own, int64_t n_max, float *pos_all,
                       int64_t *n_all_out, void *stream)
{
    if (!ctx || nranks < 1 || nranks > 32 || block < 1 || n_own < 0 || n_max < n_own ||
        !recv_counts || !recv || !pos_all || !n_all_out ||
        (reinterpret_cast<uintptr_t>(recv) & 15u) || (reinterpret_cast<uintptr_t>(pos_all) & 15u))
        return NL_ERR_ARG;
    const int64_t total = (int64_t)nranks * block;
    k_halo_pack<<<resident_grid(ctx, k_halo_pack, 256, 0, (total + 255) / 256), 256, 0,
                  reinterpret_cast<cudaStream_t>(stream)>>>(
        nranks, block, recv_counts, reinterpret_cast<const float4 *>(recv), n_own, n_max,
        reinterpret_cast<float4 *>(pos_all), n_all_out, ctx->flags);
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

nl_status nl_map_ids(nl_ctx *ctx, int64_t n_rows, int32_t capacity, int32_t *nbr,
                     const int32_t *counts, int64_t n_all, const float *pos_all, void *stream)
{
    if (!ctx || n_rows < 0 || capacity < 1 || n_all < 0) return NL_ERR_ARG;
    if (n_rows == 0) return NL_OK;
    if (!nbr || !pos_all || (reinterpret_cast<uintptr_t>(pos_all) & 15u)) return NL_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const float4 *p4 = reinterpret_cast<const float4 *>(pos_all);
    if (counts) {
        k_map_ids_rows<<<resident_grid(ctx, k_map_ids_rows, 256, 0, (n_rows + 7) / 8), 256, 0, s>>>(
            n_rows, capacity, nbr, counts, p4, n_all);
    } else {
        const int64_t entries = n_rows * (int64_t)capacity;
        k_map_ids<<<resident_grid(ctx, k_map_ids, 256, 0, (entries + 255) / 256), 256, 0, s>>>(
            entries, nbr, p4, n_all);
    }
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

}  // extern "C"
