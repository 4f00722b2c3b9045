// nl_cells.cu -- cell binning: count, single-pass scan, scatter, in-cell sort.
//
// The cells are the middle level of the neighbor search (Tessera abstract:
// "three-level neighbor search"; read here as curve order -> cells -> pairs).
// Cells are at least rl wide on every axis, numbered x fastest, so the three
// cells (cx-1, cx, cx+1) of one (cy, cz) row are contiguous in memory.
// Inside a cell atoms are ordered by (wrapped x, index), which makes every
// such row sorted by x and the result independent of atomic ordering.
#include "nl_internal.cuh"

namespace nl {
namespace {

// Largest cell the in-cell sort handles (8 atoms per lane).
constexpr int kCellSortMax = 256;

__global__ void __launch_bounds__(256)
k_bin_count(const float4 *__restrict__ pos, int64_t n, CellGrid g, uint32_t *__restrict__ atom_cell,
            uint32_t *__restrict__ atom_rank, int32_t *__restrict__ cell_count,
            float4 *__restrict__ ref)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) - lane;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const uint32_t lt = lanemask_lt();
    for (int64_t b = warp0; b < n; b += stride) {
        const int64_t i = b + lane;
        uint32_t c = 0xffffffffu;
        if (i < n) {
            const float4 p = pos[i];
            ref[i] = p;
            const int cx = cell_coord(wrap_coord(p.x, g.Lx), g.Tx, g.nx);
            const int cy = cell_coord(wrap_coord(p.y, g.Ly), g.Ty, g.ny);
            const int cz = cell_coord(wrap_coord(p.z, g.Lz), g.Tz, g.nz);
            c = (uint32_t)(((int64_t)cz * g.ny + cy) * g.nx + cx);
        }
        // warp-aggregated increment: one atomic per distinct cell
        const uint32_t peers = __match_any_sync(0xffffffffu, c);
        const int leader = __ffs(peers) - 1;
        uint32_t old = 0u;
        if (lane == leader && c != 0xffffffffu)
            old = (uint32_t)atomicAdd(&cell_count[c], __popc(peers));
        old = __shfl_sync(0xffffffffu, old, leader);
        if (i < n) {
            atom_cell[i] = c;
            atom_rank[i] = old + __popc(peers & lt);
        }
    }
}

// Exclusive scan of cell_count[0, ncell) into cell_start[0, ncell], with
// cell_start[ncell] = total, in one pass: tiles by ticket, decoupled
// look-back on one status word per tile.
__global__ void __launch_bounds__(kScanThreads)
k_cell_scan(const int32_t *__restrict__ count, int32_t *__restrict__ start, int64_t ncell,
            uint32_t *status, uint32_t *ticket, uint32_t *flags)
{
    __shared__ uint32_t s_tile;
    __shared__ uint32_t s_wtot[kScanThreads / 32];
    __shared__ uint32_t s_excl;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    if (t == 0) s_tile = atomicAdd(ticket, 1u);
    __syncthreads();
    const uint32_t tile = s_tile;
    const int64_t base = (int64_t)tile * kScanTile + (int64_t)t * kScanItems;

    uint32_t v[kScanItems];
    uint32_t sum = 0u;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        v[k] = base + k < ncell ? (uint32_t)count[base + k] : 0u;
        sum += v[k];
    }
    uint32_t x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_wtot[w] = x;
    __syncthreads();
    uint32_t wbefore = 0u, total = 0u;
#pragma unroll
    for (int i = 0; i < kScanThreads / 32; ++i) {
        if (i < w) wbefore += s_wtot[i];
        total += s_wtot[i];
    }
    if (t == 0) {
        uint32_t excl = 0u;
        uint32_t *st = status + tile;
        if (tile == 0) {
            st_volatile_u32(st, kStPrefix | total);
        } else {
            st_volatile_u32(st, kStAggregate | total);
            int64_t j = (int64_t)tile - 1;
            uint32_t spins = 0u;
            while (j >= 0) {
                const uint32_t s = ld_volatile_u32(status + j);
                const uint32_t f = s & ~kStValue;
                if (f == 0u) {
                    if (++spins >= kSpinLimit) {
                        atomicOr(flags, kFlagTimeout);
                        break;
                    }
                    if (spins > 64u) __nanosleep(64);
                    continue;
                }
                excl += s & kStValue;
                if (f == kStPrefix) break;
                --j;
            }
            st_volatile_u32(st, kStPrefix | ((excl + total) & kStValue));
        }
        s_excl = excl;
    }
    __syncthreads();
    uint32_t run = s_excl + wbefore + x - sum;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        if (base + k < ncell) start[base + k] = (int32_t)run;
        if (base + k == ncell - 1) start[ncell] = (int32_t)(run + v[k]);
        run += v[k];
    }
}

__global__ void __launch_bounds__(256)
k_bin_scatter(const float4 *__restrict__ pos, int64_t n, CellGrid g,
              const uint32_t *__restrict__ atom_cell, const uint32_t *__restrict__ atom_rank,
              const int32_t *__restrict__ cell_start, float4 *__restrict__ cell_pos,
              const uint32_t *flags)
{
    if (timed_out(flags)) return;   // cell starts may not be monotonic
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float4 p = pos[i];
        const int64_t dst = (int64_t)cell_start[atom_cell[i]] + atom_rank[i];
        cell_pos[dst] = make_float4(wrap_coord(p.x, g.Lx), wrap_coord(p.y, g.Ly),
                                    wrap_coord(p.z, g.Lz), __int_as_float((int)i));
    }
}

__device__ __forceinline__ bool before_xi(float xa, int ia, float xb, int ib)
{
    return xa < xb || (xa == xb && ia < ib);
}

// Sorts the atoms of cell c by (x, index) in place and writes the cell's x
// sub-bin table: byte b (b = 0..15) = number of the cell's atoms whose x is
// below the cell's low x face plus b/16 of its width (bin of an atom =
// floor((x - face) * 16 / width), clamped to 0..15).  The pair search reads
// these to find x-windows.  Half-warp version for cells of at most 16 atoms:
// lane hl of the half owns atom hl, ranks it with shuffles inside the half
// and computes table entry hl.
__device__ __forceinline__ void sort_small_cell(float4 *__restrict__ cell_pos, int32_t s, int m,
                                                float face, float inv_bin, uint8_t *tab, int hl,
                                                bool real)
{
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (hl < m) v = cell_pos[s + hl];
    const int id = __float_as_int(v.w);
    const int bin = max(0, min(15, (int)floorf((v.x - face) * inv_bin)));
    int r = 0, below = 0;
    // both halves run to the larger of their two cells
    const int mm = max(m, __shfl_xor_sync(0xffffffffu, m, 16));
    for (int j = 0; j < mm; ++j) {
        const float xj = __shfl_sync(0xffffffffu, v.x, j, 16);
        const int ij = __shfl_sync(0xffffffffu, id, j, 16);
        const int bj = __shfl_sync(0xffffffffu, bin, j, 16);
        if (j < m) {
            r += before_xi(xj, ij, v.x, id) ? 1 : 0;
            below += bj < hl ? 1 : 0;
        }
    }
    __syncwarp();
    if (!real) return;   // a half with no cell only takes part in the shuffles
    if (hl < m && m > 1) cell_pos[s + r] = v;
    tab[hl] = (uint8_t)below;
}

// Full-warp version for cells of 17..kCellSortMax atoms (8 atoms per lane).
__device__ __forceinline__ void sort_large_cell(float4 *__restrict__ cell_pos, int32_t s, int m,
                                                float face, float inv_bin, uint8_t *tab, int lane)
{
    constexpr int E = kCellSortMax / 32;
    float4 v[E];
    int r[E], bin[E];
    int below = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        r[e] = 0;
        v[e] = e * 32 + lane < m ? cell_pos[s + e * 32 + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
        bin[e] = max(0, min(15, (int)floorf((v[e].x - face) * inv_bin)));
    }
#pragma unroll
    for (int es = 0; es < E; ++es) {
        if (es * 32 >= m) break;
        const float xs = v[es].x;
        const int is = __float_as_int(v[es].w);
        const int bs = bin[es];
        const int lim = m - es * 32 < 32 ? m - es * 32 : 32;
        for (int l = 0; l < lim; ++l) {
            const float xj = __shfl_sync(0xffffffffu, xs, l);
            const int ij = __shfl_sync(0xffffffffu, is, l);
            const int bj = __shfl_sync(0xffffffffu, bs, l);
            below += bj < lane ? 1 : 0;
#pragma unroll
            for (int e = 0; e < E; ++e)
                r[e] += before_xi(xj, ij, v[e].x, __float_as_int(v[e].w)) ? 1 : 0;
        }
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e * 32 + lane < m) cell_pos[s + r[e]] = v[e];
    if (lane < 16) tab[lane] = (uint8_t)below;
}

// Two cells per warp, one per half.  A cell of at most 16 atoms is sorted
// here; a larger one (up to kCellSortMax) is listed for k_cell_sort_large,
// and one above kCellSortMax stays in scatter order and raises `unsorted`.
// Keeping the large path out of this kernel keeps its register count low, so
// enough warps are resident to cover the two dependent global loads per cell.
__global__ void __launch_bounds__(256)
k_cell_sort(float4 *__restrict__ cell_pos, const int32_t *__restrict__ cell_start, int64_t ncell,
            int nx, float side_x, float inv_bin, uint8_t *__restrict__ cell_tab,
            uint32_t *__restrict__ large_list, uint32_t *large_count, uint32_t *unsorted,
            const uint32_t *flags)
{
    if (timed_out(flags)) return;
    const int lane = threadIdx.x & 31, half = lane >> 4, hl = lane & 15;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    // the next iteration's cell range is loaded one iteration ahead, so only
    // the position load stays on each iteration's dependent chain
    int32_t s_next = 0, e_next = 0;
    if (2 * warp + half < ncell) {
        s_next = cell_start[2 * warp + half];
        e_next = cell_start[2 * warp + half + 1];
    }
    for (int64_t c0 = 2 * warp; c0 < ncell; c0 += 2 * nwarps) {
        const int64_t c = c0 + half;
        const bool have = c < ncell;
        const int32_t s = have ? s_next : 0;
        const int m = have ? e_next - s_next : 0;
        const int64_t cn = c + 2 * nwarps;
        if (cn < ncell) {
            s_next = cell_start[cn];
            e_next = cell_start[cn + 1];
        }
        const float face = (float)(int)(c % nx) * side_x;
        const bool small = m <= 16;
        sort_small_cell(cell_pos, s, small ? m : 0, face, inv_bin, cell_tab + (have ? c : 0) * 16,
                        hl, have && small);
        if (have && !small && hl == 0) {
            if (m > kCellSortMax)
                atomicOr(unsorted, 1u);
            else
                large_list[atomicAdd(large_count, 1u)] = (uint32_t)c;
        }
    }
}

// The listed cells of 17..kCellSortMax atoms, one warp per cell.
__global__ void __launch_bounds__(256)
k_cell_sort_large(float4 *__restrict__ cell_pos, const int32_t *__restrict__ cell_start, int nx,
                  float side_x, float inv_bin, uint8_t *__restrict__ cell_tab,
                  const uint32_t *__restrict__ large_list, const uint32_t *large_count,
                  const uint32_t *flags)
{
    if (timed_out(flags)) return;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const uint32_t nlisted = *large_count;
    for (int64_t e = warp; e < (int64_t)nlisted; e += nwarps) {
        const int64_t c = large_list[e];
        const int32_t s = cell_start[c];
        const int m = cell_start[c + 1] - s;
        const float face = (float)(int)(c % nx) * side_x;
        sort_large_cell(cell_pos, s, m, face, inv_bin, cell_tab + c * 16, lane);
    }
}

}  // namespace

cudaError_t launch_binning(nl_ctx *ctx, int64_t n, const float4 *pos, const CellGrid &g,
                           cudaStream_t s)
{
    const int64_t scan_tiles = (g.ncell + kScanTile - 1) / kScanTile;
    NL_CUDA_TRY(cudaMemsetAsync(ctx->cell_count, 0, sizeof(int32_t) * g.ncell, s));
    NL_CUDA_TRY(cudaMemsetAsync(ctx->scan_status, 0, sizeof(uint32_t) * scan_tiles, s));
    NL_CUDA_TRY(cudaMemsetAsync(ctx->scan_ctr, 0, sizeof(uint32_t), s));
    NL_CUDA_TRY(cudaMemsetAsync(ctx->unsorted, 0, sizeof(uint32_t), s));
    {
        ProfScope ps(ctx, PH_BIN_COUNT, s);
        if (n > 0)
            k_bin_count<<<resident_grid(ctx, k_bin_count, 256, 0, (n + 255) / 256), 256, 0, s>>>(
                pos, n, g, ctx->atom_cell, ctx->atom_rank, ctx->cell_count, ctx->ref);
        NL_CUDA_TRY(cudaGetLastError());
    }
    {
        ProfScope ps(ctx, PH_CELL_SCAN, s);
        k_cell_scan<<<(unsigned)scan_tiles, kScanThreads, 0, s>>>(
            ctx->cell_count, ctx->cell_start, g.ncell, ctx->scan_status, ctx->scan_ctr, ctx->flags);
        NL_CUDA_TRY(cudaGetLastError());
    }
    if (n <= 0) return cudaSuccess;
    {
        ProfScope ps(ctx, PH_BIN_SCATTER, s);
        k_bin_scatter<<<resident_grid(ctx, k_bin_scatter, 256, 0, (n + 255) / 256), 256, 0, s>>>(pos, n, g, ctx->atom_cell,
                                                             ctx->atom_rank, ctx->cell_start,
                                                             ctx->cell_pos, ctx->flags);
        NL_CUDA_TRY(cudaGetLastError());
    }
    {
        // cells above 16 atoms are listed in fb_list (free until the pair
        // search, which resets fb_count before it lists its own tiles)
        ProfScope ps(ctx, PH_CELL_SORT, s);
        const float side_x = g.Lx / (float)g.nx;
        NL_CUDA_TRY(cudaMemsetAsync(ctx->fb_count, 0, sizeof(uint32_t), s));
        // several waves of CTAs over the cells: measured faster than one
        // resident wave striding over them
        int64_t sort_blocks = (g.ncell * 16 + 255) / 256;
        if (sort_blocks > (int64_t)ctx->sm_count * 32) sort_blocks = (int64_t)ctx->sm_count * 32;
        k_cell_sort<<<(unsigned)sort_blocks, 256, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, g.ncell, g.nx, side_x, 16.0f / side_x, ctx->cell_tab,
            ctx->fb_list, ctx->fb_count, ctx->unsorted, ctx->flags);
        NL_CUDA_TRY(cudaGetLastError());
        k_cell_sort_large<<<(unsigned)(ctx->sm_count * 2), 256, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, g.nx, side_x, 16.0f / side_x, ctx->cell_tab,
            ctx->fb_list, ctx->fb_count, ctx->flags);
        NL_CUDA_TRY(cudaGetLastError());
    }
    return cudaSuccess;
}

}  // namespace nl
