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

// Largest cell the in-cell sort handles: its table counts must fit a byte.
constexpr int kCellSortMax = 255;
// In-cell sort: cells per CTA, atoms a CTA stages at once, threads.
constexpr int kSortCells = 128;
constexpr int kSortCap = 768;
constexpr int kSortThreads2 = 256;

// Binning kernels: each warp takes kBinUnroll groups of 32 consecutive
// atoms per round and issues all their loads (and atomics) before using any,
// so several memory round trips are in flight per warp.
constexpr int kBinUnroll = 4;

__global__ void __launch_bounds__(256)
k_bin_count(const float4 *__restrict__ pos, int64_t n, CellGrid g, uint32_t *__restrict__ atom_cell,
            uint32_t *__restrict__ atom_rank, int32_t *__restrict__ cell_count,
            float4 *__restrict__ ref)
{
    n = atoms_of(g, n);
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t stride = ((int64_t)gridDim.x * blockDim.x) * kBinUnroll;
    const uint32_t lt = lanemask_lt();
    for (int64_t b = warp * 32 * kBinUnroll; b < n; b += stride) {
        uint32_t c[kBinUnroll];
#pragma unroll
        for (int u = 0; u < kBinUnroll; ++u) {
            const int64_t i = b + 32 * u + lane;
            c[u] = 0xffffffffu;
            if (i < n) {
                const float4 p = pos[i];
                ref[i] = p;
                const int cx = cell_coord(wrap_coord(p.x, g.Lx), g.Tx, g.nx);
                const int cy = cell_coord(wrap_coord(p.y, g.Ly), g.Ty, g.ny);
                const int cz = cell_coord(wrap_coord(p.z, g.Lz), g.Tz, g.nz);
                c[u] = (uint32_t)(((int64_t)cz * g.ny + cy) * g.nx + cx);
            }
        }
        // warp-aggregated increments: one atomic per distinct cell and group
        uint32_t peers[kBinUnroll], old[kBinUnroll];
#pragma unroll
        for (int u = 0; u < kBinUnroll; ++u) {
            peers[u] = __match_any_sync(0xffffffffu, c[u]);
            old[u] = 0u;
            if (lane == __ffs(peers[u]) - 1 && c[u] != 0xffffffffu)
                old[u] = (uint32_t)atomicAdd(&cell_count[c[u]], __popc(peers[u]));
        }
#pragma unroll
        for (int u = 0; u < kBinUnroll; ++u) {
            const int64_t i = b + 32 * u + lane;
            const uint32_t o = __shfl_sync(0xffffffffu, old[u], __ffs(peers[u]) - 1);
            if (i < n) {
                atom_cell[i] = c[u];
                atom_rank[i] = o + __popc(peers[u] & lt);
            }
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
    if (w == 0) {
        // look-back by the first warp: lane l reads the status of tile
        // j - l, so 32 predecessors are read per round; the words before the
        // first prefix or unpublished one are aggregates to add
        uint32_t excl = 0u;
        uint32_t *st = status + tile;
        if (tile == 0) {
            if (lane == 0) st_volatile_u32(st, kStPrefix | total);
        } else {
            if (lane == 0) st_volatile_u32(st, kStAggregate | total);
            int64_t j = (int64_t)tile - 1;
            uint32_t spins = 0u;
            for (;;) {
                const int64_t jj = j - lane;
                const uint32_t s = jj >= 0 ? ld_volatile_u32(status + jj) : kStPrefix;
                const uint32_t f = s & ~kStValue;
                const uint32_t pre = __ballot_sync(0xffffffffu, f == kStPrefix);
                const uint32_t stop = pre | __ballot_sync(0xffffffffu, f == 0u);
                const int first = stop ? __ffs(stop) - 1 : 32;
                const bool done = first < 32 && ((pre >> first) & 1u);
                uint32_t v = (lane < first || (done && lane == first)) ? (s & kStValue) : 0u;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                excl += v;
                if (done) break;
                j -= first;
                if (first < 32) {   // tile j not yet published: poll it again
                    if (++spins >= kSpinLimit) {
                        if (lane == 0) atomicOr(flags, kFlagTimeout);
                        break;
                    }
                    if (spins > 64u) __nanosleep(64);
                }
            }
            if (lane == 0) st_volatile_u32(st, kStPrefix | ((excl + total) & kStValue));
        }
        if (lane == 0) s_excl = excl;
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
    n = atoms_of(g, n);
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t stride = ((int64_t)gridDim.x * blockDim.x) * kBinUnroll;
    for (int64_t b = warp * 32 * kBinUnroll; b < n; b += stride) {
        float4 p[kBinUnroll];
        uint32_t c[kBinUnroll], r[kBinUnroll];
#pragma unroll
        for (int u = 0; u < kBinUnroll; ++u) {
            const int64_t i = b + 32 * u + lane;
            if (i < n) {
                p[u] = pos[i];
                c[u] = atom_cell[i];
                r[u] = atom_rank[i];
            }
        }
        int32_t st[kBinUnroll];
#pragma unroll
        for (int u = 0; u < kBinUnroll; ++u)
            if (b + 32 * u + lane < n) st[u] = cell_start[c[u]];
#pragma unroll
        for (int u = 0; u < kBinUnroll; ++u) {
            const int64_t i = b + 32 * u + lane;
            if (i < n)
                cell_pos[(int64_t)st[u] + r[u]] =
                    make_float4(wrap_coord(p[u].x, g.Lx), wrap_coord(p[u].y, g.Ly),
                                wrap_coord(p[u].z, g.Lz), __int_as_float((int)i));
        }
    }
}

// (x, index) order of wrapped atoms as one unsigned 64-bit key: x is in
// [0, L), where the bits of a float (sign cleared, so -0 equals +0) order
// as the values do, and indices are non-negative.
__device__ __forceinline__ uint64_t xi_key(float x, int i)
{
    return ((uint64_t)(__float_as_uint(x) & 0x7fffffffu) << 32) | (uint32_t)i;
}

// In-cell sort, one CTA per run of kSortCells consecutive cells (a
// contiguous range of the cell-ordered array).  The CTA stages the range's
// atoms in shared memory with coalesced loads -- whole cells, at most
// kSortCap atoms at a time -- ranks each atom by (x, index) inside its cell,
// writes the cell back sorted (coalesced again) and writes each cell's x
// sub-bin table: byte b (b = 0..15) = number of the cell's atoms whose x is
// below the cell's low x face plus b/16 of its width (bin of an atom =
// floor((x - face) * 16 / width), clamped to 0..15), stored 16 bytes per
// cell.  The pair search reads these to find x-windows.  Entry b is also the
// in-cell index of the first sorted atom whose bin is b or more, so the
// atoms write the table: sorted atom k covers the entries after its
// predecessor's bin up to its own, and the last atom the entries above its
// bin (with the cell's count); entries before the first atom's bin stay 0.
// A cell of more than kCellSortMax atoms (its table counts would not fit a
// byte) stays in scatter order with a zero table and raises `unsorted`,
// which sends the pair search to its per-atom path.
__global__ void __launch_bounds__(kSortThreads2)
k_cell_sort(float4 *__restrict__ cell_pos, const int32_t *__restrict__ cell_start, int64_t ncell,
            int nx, float side_x, float inv_bin, uint8_t *__restrict__ cell_tab,
            uint32_t *unsorted, const uint32_t *flags)
{
    // cell starts may not be monotonic; one decision for the whole CTA
    if (__syncthreads_or(timed_out(flags))) return;
    static_assert(kSortCells <= 256, "a staged atom's cell is kept in a byte");
    __shared__ float4 s_pos[kSortCap];
    __shared__ uint64_t s_key[kSortCap];                     // (x bits, index): the sort key
    __shared__ uint8_t s_sbin[kSortCap];                     // bins in sorted order
    __shared__ uint8_t s_cof[kSortCap];                      // cell of each staged slot
    __shared__ __align__(16) uint8_t s_tab[kSortCells][16];
    __shared__ int32_t s_cs[kSortCells + 1];
    __shared__ float s_face[kSortCells];                     // low x face of each cell
    const int t = threadIdx.x;
    const int64_t c0 = (int64_t)blockIdx.x * kSortCells;
    const int nc = (int)(ncell - c0 < kSortCells ? ncell - c0 : kSortCells);
    for (int k = t; k <= nc; k += blockDim.x) s_cs[k] = cell_start[c0 + k];
    for (int k = t; k < nc; k += blockDim.x) {
        s_face[k] = (float)(int)((c0 + k) % nx) * side_x;
        *reinterpret_cast<uint4 *>(s_tab[k]) = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    int cb = 0;
    while (cb < nc) {
        // the longest run of whole cells from cb whose atoms fit the stage
        // (at least one cell; a cell alone beyond the stage is left unsorted)
        const int fit = __syncthreads_count(t >= cb && t < nc &&
                                            s_cs[t + 1] - s_cs[cb] <= kSortCap);
        const int ce = cb + (fit > 0 ? fit : 1);
        const int a0 = s_cs[cb];
        const int m = s_cs[ce] - a0;
        if (m > kSortCap) {
            if (t == 0) atomicOr(unsorted, 1u);
            cb = ce;
            continue;
        }
        for (int k = t; k < m; k += blockDim.x) {
            const float4 v = cell_pos[a0 + k];
            s_pos[k] = v;
            s_key[k] = xi_key(v.x, __float_as_int(v.w));
        }
        for (int c = cb + t; c < ce; c += blockDim.x)
            for (int q = s_cs[c] - a0; q < s_cs[c + 1] - a0; ++q) s_cof[q] = (uint8_t)c;
        __syncthreads();
        // each atom: its bin and its rank by (x, index) among its cell's atoms
        for (int k = t; k < m; k += blockDim.x) {
            const int c = s_cof[k];
            const int s0 = s_cs[c] - a0, s1 = s_cs[c + 1] - a0;
            if (s1 - s0 > kCellSortMax) continue;   // too large: left in scatter order
            const float4 v = s_pos[k];
            const uint64_t key = s_key[k];
            int r = 0;
            for (int q = s0; q < s1; ++q) r += s_key[q] < key ? 1 : 0;
            s_sbin[s0 + r] = (uint8_t)max(0, min(15, (int)floorf((v.x - s_face[c]) * inv_bin)));
            cell_pos[a0 + s0 + r] = v;
        }
        __syncthreads();
        // the tables, written by the sorted atoms (a cell's slots are the
        // same before and after its sort)
        for (int k = t; k < m; k += blockDim.x) {
            const int c = s_cof[k];
            const int s0 = s_cs[c] - a0, s1 = s_cs[c + 1] - a0;
            if (s1 - s0 > kCellSortMax) {
                if (k == s0) atomicOr(unsorted, 1u);
                continue;
            }
            const int kk = k - s0, b1 = s_sbin[k];
            for (int b = kk > 0 ? s_sbin[k - 1] + 1 : b1 + 1; b <= b1; ++b)
                s_tab[c][b] = (uint8_t)kk;
            if (k == s1 - 1)
                for (int b = b1 + 1; b < 16; ++b) s_tab[c][b] = (uint8_t)(s1 - s0);
        }
        __syncthreads();   // the stage is reused by the next run of cells
        cb = ce;
    }
    // the CTA's tables, 16 bytes per cell
    for (int c = t; c < nc; c += blockDim.x)
        reinterpret_cast<uint4 *>(cell_tab)[c0 + c] = *reinterpret_cast<const uint4 *>(s_tab[c]);
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
            k_bin_count<<<resident_grid(ctx, k_bin_count, 256, 0,
                                        (n + 256 * kBinUnroll - 1) / (256 * kBinUnroll)),
                          256, 0, s>>>(
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
        k_bin_scatter<<<resident_grid(ctx, k_bin_scatter, 256, 0,
                                      (n + 256 * kBinUnroll - 1) / (256 * kBinUnroll)),
                        256, 0, s>>>(pos, n, g, ctx->atom_cell, ctx->atom_rank, ctx->cell_start,
                                     ctx->cell_pos, ctx->flags);
        NL_CUDA_TRY(cudaGetLastError());
    }
    {
        ProfScope ps(ctx, PH_CELL_SORT, s);
        const float side_x = g.Lx / (float)g.nx;
        const int64_t blocks = (g.ncell + kSortCells - 1) / kSortCells;
        k_cell_sort<<<(unsigned)blocks, kSortThreads2, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, g.ncell, g.nx, side_x, 16.0f / side_x, ctx->cell_tab,
            ctx->unsorted, ctx->flags);
        NL_CUDA_TRY(cudaGetLastError());
    }
    return cudaSuccess;
}

}  // namespace nl
