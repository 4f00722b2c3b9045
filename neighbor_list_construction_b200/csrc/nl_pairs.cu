// nl_pairs.cu -- pair search and padded-row output.
//
// Tessera abstract: neighbor topology is held fixed between rebuilds, so the
// list is a fixed-capacity tensor (rows padded with -1, overflow reported).
//
// Minimum image without division.  For wrapped coordinates d = w_j - w_i lies
// in (-L, L).  When every axis has at least 5 cells, two atoms in the same or
// adjacent (non-wrapping) cells have |d| <= 2L/5 plus rounding, so
// rintf(d/L) == 0 and the literal formula leaves d unchanged; across the
// periodic face (home cell n-1, neighbor cell 0, or the reverse) |d| >= 3L/5,
// so rintf(d/L) == -+1 and the literal formula gives exactly fl(d + L) or
// fl(d - L).  The shift S in {-L, 0, +L} is therefore known per neighbor cell
// and fl(fl(w_j - w_i) + S) equals the literal d - L*rintf(d/L) bit for bit.
// Boxes with 3 or 4 cells on an axis use the literal formula.
#include "nl_internal.cuh"

namespace nl {
namespace {

// ---------------------------------------------------------------------------
// Per-atom search: one thread per atom, the 27 neighbor cells straight from
// global memory, hits stored directly into the atom's row.  Used for boxes
// with fewer than 5 cells on an axis (literal minimum image), for tiles the
// staged kernel cannot take, and when the staged kernel's preconditions fail.
// ---------------------------------------------------------------------------
template <bool LITERAL>
__device__ __forceinline__ void pair_row_per_atom(int64_t k, const float4 *__restrict__ cell_pos,
                                                  const int32_t *__restrict__ cell_start,
                                                  const uint32_t *__restrict__ atom_cell,
                                                  const CellGrid &g, int32_t K,
                                                  int32_t *__restrict__ nbr,
                                                  int32_t *__restrict__ counts, uint32_t *flags)
{
    const float4 p = cell_pos[k];
    const int i = __float_as_int(p.w);
    const uint32_t c = atom_cell[i];
    const int cx = (int)(c % (uint32_t)g.nx);
    const int cy = (int)((c / (uint32_t)g.nx) % (uint32_t)g.ny);
    const int cz = (int)(c / ((uint32_t)g.nx * (uint32_t)g.ny));
    int32_t *row = nbr + (int64_t)i * K;
    int cnt = 0;
    for (int oz = -1; oz <= 1; ++oz) {
        int z = cz + oz;
        float sz = 0.0f;
        if (z < 0) { z += g.nz; sz = -g.Lz; } else if (z >= g.nz) { z -= g.nz; sz = g.Lz; }
        for (int oy = -1; oy <= 1; ++oy) {
            int y = cy + oy;
            float sy = 0.0f;
            if (y < 0) { y += g.ny; sy = -g.Ly; } else if (y >= g.ny) { y -= g.ny; sy = g.Ly; }
            for (int ox = -1; ox <= 1; ++ox) {
                int x = cx + ox;
                float sx = 0.0f;
                if (x < 0) { x += g.nx; sx = -g.Lx; } else if (x >= g.nx) { x -= g.nx; sx = g.Lx; }
                const int64_t c2 = ((int64_t)z * g.ny + y) * g.nx + x;
                const int32_t j0 = cell_start[c2], j1 = cell_start[c2 + 1];
                for (int32_t j = j0; j < j1; ++j) {
                    const float4 q = cell_pos[j];
                    const int jid = __float_as_int(q.w);
                    if (jid == i) continue;
                    float dx = __fsub_rn(q.x, p.x);
                    float dy = __fsub_rn(q.y, p.y);
                    float dz = __fsub_rn(q.z, p.z);
                    if (LITERAL) {
                        dx = min_image_literal(dx, g.Lx);
                        dy = min_image_literal(dy, g.Ly);
                        dz = min_image_literal(dz, g.Lz);
                    } else {
                        if (sx != 0.0f) dx = __fadd_rn(dx, sx);
                        if (sy != 0.0f) dy = __fadd_rn(dy, sy);
                        if (sz != 0.0f) dz = __fadd_rn(dz, sz);
                    }
                    if (r2_of(dx, dy, dz) < g.rl2) {
                        if (cnt < K) row[cnt] = jid;
                        ++cnt;
                    }
                }
            }
        }
    }
    counts[i] = cnt;
    for (int e = cnt < K ? cnt : K; e < K; ++e) row[e] = -1;
    if (cnt > K) atomicOr(flags, kFlagOverflow);
}

template <bool LITERAL>
__global__ void __launch_bounds__(128)
k_pairs_per_atom(const float4 *__restrict__ cell_pos, const int32_t *__restrict__ cell_start,
                 const uint32_t *__restrict__ atom_cell, int64_t n, CellGrid g, int32_t K,
                 int32_t *__restrict__ nbr, int32_t *__restrict__ counts, uint32_t *flags)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
        pair_row_per_atom<LITERAL>(k, cell_pos, cell_start, atom_cell, g, K, nbr, counts, flags);
}

// ---------------------------------------------------------------------------
// Staged search.  A tile is a run of kTileCells cells along x at one (cy, cz).
// Its 9 neighbor rows (dy, dz in -1..1), each covering cells cx0-1 .. cx0+G
// along x, are contiguous ranges of the cell-ordered array (plus at most one
// periodic image cell at either end); they are copied into shared memory with
// cp.async.bulk and an mbarrier.  Each lane owns one home atom.  Because the
// atoms of a row are sorted by x, the candidates of a home atom in a row lie
// in one index window [x - h, x + h], with h = sqrt(rl^2 - d_perp^2) from the
// atom's distance to the row's (y, z) cell face (plus a margin); every lane
// walks the same number of candidates from its own window start, so a lane
// may test a few atoms outside its window -- harmless, since every tested
// pair is decided by the exact predicate.  Hits are kept as 16-bit staged
// slot numbers in a per-lane row in shared memory and written out at the end
// of the chunk as full 16-byte row vectors.
// ---------------------------------------------------------------------------
constexpr int kTileCells = 4;
constexpr int kStageMin = 2560;   // fewest staged atoms worth a launch
constexpr int kRuns = 9;
constexpr int kMaxSegs = 3 * kRuns;

struct TileInfo {
    int run_off[kRuns];
    int run_len[kRuns];
    int run_lend[kRuns];   // [0, lend): periodic image on the low x side (shift -Lx)
    int run_rbeg[kRuns];   // [rbeg, len): periodic image on the high x side (shift +Lx)
    float run_sy[kRuns];
    float run_sz[kRuns];
    int seg_src[kMaxSegs];
    int seg_dst[kMaxSegs];
    int seg_cnt[kMaxSegs];
    int nseg;
    int total;
    int home_begin, home_end;
    int fallback;
};

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// One contiguous global -> shared copy completing on `bar` (16-byte multiples).
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// First index j of the run with image-corrected x(j) >= v (le = false) or > v
// (le = true).  The run is sorted by x up to rounding at cell faces, far
// below the window margin.
template <bool LE>
__device__ __forceinline__ int run_bound(const float4 *run, int len, int lend, int rbeg, float Lx,
                                         float v)
{
    int lo = 0, n = len;
    while (n > 0) {
        const int half = n >> 1;
        const int mid = lo + half;
        float xm = run[mid].x;
        xm = mid < lend ? xm - Lx : (mid >= rbeg ? xm + Lx : xm);
        const bool before = LE ? (xm <= v) : (xm < v);
        if (before) {
            lo = mid + 1;
            n -= half + 1;
        } else {
            n = half;
        }
    }
    return lo;
}

template <bool XS, bool YZ, bool SELF, bool CLAMP>
__device__ __forceinline__ void scan_run(const float4 *__restrict__ run, int st, int L,
                                         const float4 me, float Lx, int lend, int rbeg, float sy,
                                         float sz, float rl2, uint16_t *&bp, uint16_t *bend,
                                         int slot0)
{
    const int myid = __float_as_int(me.w);
#pragma unroll 4
    for (int k = 0; k < L; ++k) {
        const int j = st + k;
        const float4 q = run[j];
        float dx = __fsub_rn(q.x, me.x);
        float dy = __fsub_rn(q.y, me.y);
        float dz = __fsub_rn(q.z, me.z);
        if (XS) dx = __fadd_rn(dx, j < lend ? -Lx : (j >= rbeg ? Lx : 0.0f));
        if (YZ) {
            dy = __fadd_rn(dy, sy);
            dz = __fadd_rn(dz, sz);
        }
        bool hit = r2_of(dx, dy, dz) < rl2;
        if (SELF) hit = hit && (__float_as_int(q.w) != myid);
        if (hit) {
            uint16_t *p = bp;
            if (CLAMP && p > bend) p = bend;
            *p = (uint16_t)(slot0 + j);
            ++bp;
        }
    }
}

struct StagedParams {
    const float4 *cell_pos;
    const int32_t *cell_start;
    int32_t *nbr;
    int32_t *counts;
    uint32_t *flags;
    const uint32_t *unsorted;
    uint32_t *fb_list;
    uint32_t *fb_count;
    int tiles_x;
    int K;
    int stage_max;          // staged atoms per tile (shared memory left after the rows)
    float side_y, side_z;   // cell widths
    float eps;              // window margin
    float rl2_margin;       // rl2 * (1 + 1e-4)
};

__global__ void __launch_bounds__(128)
k_pairs_staged(const CellGrid g, const StagedParams P)
{
    extern __shared__ __align__(16) unsigned char pairs_smem[];
    float4 *stage = reinterpret_cast<float4 *>(pairs_smem);
    uint16_t *rows = reinterpret_cast<uint16_t *>(pairs_smem + sizeof(float4) * P.stage_max);
    __shared__ TileInfo ti;
    __shared__ __align__(8) uint64_t bar;

    const int W = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int RS = P.K + 4;   // row stride in 16-bit slots; slot K is the overflow dummy
    const int tile = blockIdx.x;
    const int tx = tile % P.tiles_x;
    const int rest = tile / P.tiles_x;
    const int cy = rest % g.ny;
    const int cz = rest / g.ny;
    const int cx0 = tx * kTileCells;
    const int G = min(kTileCells, g.nx - cx0);

    if (threadIdx.x == 0) {
        int total = 0, nseg = 0;
        for (int r = 0; r < kRuns; ++r) {
            const int dy = r % 3 - 1, dz = r / 3 - 1;
            int y = cy + dy, z = cz + dz;
            float sy = 0.0f, sz = 0.0f;
            if (y < 0) { y += g.ny; sy = -g.Ly; } else if (y >= g.ny) { y -= g.ny; sy = g.Ly; }
            if (z < 0) { z += g.nz; sz = -g.Lz; } else if (z >= g.nz) { z -= g.nz; sz = g.Lz; }
            const int64_t rowc = ((int64_t)z * g.ny + y) * g.nx;
            ti.run_off[r] = total;
            ti.run_sy[r] = sy;
            ti.run_sz[r] = sz;
            int len = 0;
            // low periodic image: conceptual cell -1 is cell nx-1
            if (cx0 == 0) {
                const int a = P.cell_start[rowc + g.nx - 1], b = P.cell_start[rowc + g.nx];
                ti.seg_src[nseg] = a; ti.seg_dst[nseg] = total + len; ti.seg_cnt[nseg] = b - a;
                ++nseg;
                len += b - a;
            }
            ti.run_lend[r] = len;
            const int first = cx0 == 0 ? 0 : cx0 - 1;
            const int last = cx0 + G <= g.nx - 1 ? cx0 + G : g.nx - 1;
            {
                const int a = P.cell_start[rowc + first], b = P.cell_start[rowc + last + 1];
                ti.seg_src[nseg] = a; ti.seg_dst[nseg] = total + len; ti.seg_cnt[nseg] = b - a;
                ++nseg;
                if (r == 4) {
                    ti.home_begin = total + len + (P.cell_start[rowc + cx0] - a);
                    ti.home_end = total + len + (P.cell_start[rowc + cx0 + G] - a);
                }
                len += b - a;
            }
            ti.run_rbeg[r] = len;
            // high periodic image: conceptual cell nx is cell 0
            if (cx0 + G == g.nx) {
                const int a = P.cell_start[rowc], b = P.cell_start[rowc + 1];
                ti.seg_src[nseg] = a; ti.seg_dst[nseg] = total + len; ti.seg_cnt[nseg] = b - a;
                ++nseg;
                len += b - a;
            }
            ti.run_len[r] = len;
            total += len;
        }
        ti.nseg = nseg;
        ti.total = total;
        ti.fallback = (total > P.stage_max || *P.unsorted != 0u) ? 1 : 0;
        if (ti.fallback) {
            const uint32_t slot = atomicAdd(P.fb_count, 1u);
            P.fb_list[slot] = (uint32_t)tile;
        } else {
            mbar_init(&bar, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
    }
    __syncthreads();
    if (ti.fallback) return;

    if (warp == 0) {
        if (lane == 0) mbar_arrive_expect_tx(&bar, (uint32_t)ti.total * (uint32_t)sizeof(float4));
        __syncwarp();
        for (int sg = lane; sg < ti.nseg; sg += 32)
            if (ti.seg_cnt[sg] > 0)
                bulk_g2s(stage + ti.seg_dst[sg], P.cell_pos + ti.seg_src[sg],
                         (uint32_t)ti.seg_cnt[sg] * (uint32_t)sizeof(float4), &bar);
    }
    {
        uint32_t spins = 0;
        while (!mbar_try_wait(&bar, 0)) {
            if (++spins >= kSpinLimit) {
                if (threadIdx.x == 0) atomicOr(P.flags, kFlagTimeout);
                return;
            }
        }
    }

    const float rl2 = g.rl2;
    const int nhome = ti.home_end - ti.home_begin;
    const int nchunks = (nhome + 31) >> 5;
    uint16_t *mybuf = rows + (size_t)(warp * 32 + lane) * RS;
    uint16_t *bend = mybuf + P.K;
    const float ylo = (float)cy * P.side_y, yhi = (float)(cy + 1) * P.side_y;
    const float zlo = (float)cz * P.side_z, zhi = (float)(cz + 1) * P.side_z;

    for (int c = warp; c < nchunks; c += W) {
        const int a = ti.home_begin + c * 32 + lane;
        const bool valid = a < ti.home_end;
        const float4 me = valid ? stage[a] : make_float4(-1e30f, -1e30f, -1e30f, __int_as_float(-1));
        uint16_t *bp = mybuf;
        for (int r = 0; r < kRuns; ++r) {
            const int dy = r % 3 - 1, dz = r / 3 - 1;
            const float4 *run = stage + ti.run_off[r];
            const int len = ti.run_len[r], lend = ti.run_lend[r], rbeg = ti.run_rbeg[r];
            float py = dy < 0 ? me.y - ylo : (dy > 0 ? yhi - me.y : 0.0f);
            float pz = dz < 0 ? me.z - zlo : (dz > 0 ? zhi - me.z : 0.0f);
            py = fmaxf(py - P.eps, 0.0f);
            pz = fmaxf(pz - P.eps, 0.0f);
            const float h2 = P.rl2_margin - (py * py + pz * pz);
            int lo = 0, hi = 0;
            if (valid && h2 > 0.0f) {
                const float h = sqrtf(h2) + P.eps;
                lo = run_bound<false>(run, len, lend, rbeg, g.Lx, me.x - h);
                hi = run_bound<true>(run, len, lend, rbeg, g.Lx, me.x + h);
            }
            const int L = __reduce_max_sync(0xffffffffu, hi - lo);
            if (L == 0) continue;
            const int st = lo < len - L ? lo : len - L;
            const bool xs = lend > 0 || rbeg < len;
            const bool yz = ti.run_sy[r] != 0.0f || ti.run_sz[r] != 0.0f;
            const bool clamp = __any_sync(0xffffffffu, (int)(bp - mybuf) + L > P.K);
            const float sy = ti.run_sy[r], sz = ti.run_sz[r];
            const int slot0 = ti.run_off[r];
            if (r == 4) {
                if (xs) {
                    if (clamp) scan_run<true, false, true, true>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                    else scan_run<true, false, true, false>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                } else {
                    if (clamp) scan_run<false, false, true, true>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                    else scan_run<false, false, true, false>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                }
            } else if (!yz) {
                if (xs) {
                    if (clamp) scan_run<true, false, false, true>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                    else scan_run<true, false, false, false>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                } else {
                    if (clamp) scan_run<false, false, false, true>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                    else scan_run<false, false, false, false>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                }
            } else {
                if (xs) {
                    if (clamp) scan_run<true, true, false, true>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                    else scan_run<true, true, false, false>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                } else {
                    if (clamp) scan_run<false, true, false, true>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                    else scan_run<false, true, false, false>(run, st, L, me, g.Lx, lend, rbeg, sy, sz, rl2, bp, bend, slot0);
                }
            }
        }
        const int cnt = (int)(bp - mybuf);
        const int myid = __float_as_int(me.w);
        if (valid) {
            P.counts[myid] = cnt;
            if (cnt > P.K) atomicOr(P.flags, kFlagOverflow);
        }
        __syncwarp();
        // write the chunk's rows: 16-byte vectors, hits then -1
        const int nvalid = min(32, ti.home_end - (ti.home_begin + c * 32));
        for (int rr = 0; rr < nvalid; ++rr) {
            const int cr = __shfl_sync(0xffffffffu, cnt, rr);
            const int ir = __shfl_sync(0xffffffffu, myid, rr);
            const int nv = cr < P.K ? cr : P.K;
            const uint16_t *rb = rows + (size_t)(warp * 32 + rr) * RS;
            int4 *dst = reinterpret_cast<int4 *>(P.nbr + (int64_t)ir * P.K);
            for (int v = lane; v < (P.K >> 2); v += 32) {
                const int e0 = v << 2;
                const uint2 pk = *reinterpret_cast<const uint2 *>(rb + e0);
                const int s0 = e0 + 0 < nv ? (int)(pk.x & 0xffffu) : 0;
                const int s1 = e0 + 1 < nv ? (int)(pk.x >> 16) : 0;
                const int s2 = e0 + 2 < nv ? (int)(pk.y & 0xffffu) : 0;
                const int s3 = e0 + 3 < nv ? (int)(pk.y >> 16) : 0;
                int4 o;
                o.x = e0 + 0 < nv ? __float_as_int(stage[s0].w) : -1;
                o.y = e0 + 1 < nv ? __float_as_int(stage[s1].w) : -1;
                o.z = e0 + 2 < nv ? __float_as_int(stage[s2].w) : -1;
                o.w = e0 + 3 < nv ? __float_as_int(stage[s3].w) : -1;
                dst[v] = o;
            }
        }
        __syncwarp();
    }
}

// Rows of the tiles the staged kernel listed: per-atom search over their
// home atoms.
__global__ void __launch_bounds__(128)
k_pairs_listed(const float4 *__restrict__ cell_pos, const int32_t *__restrict__ cell_start,
               const uint32_t *__restrict__ atom_cell, CellGrid g, int32_t K, int tiles_x,
               const uint32_t *__restrict__ fb_list, const uint32_t *__restrict__ fb_count,
               int32_t *__restrict__ nbr, int32_t *__restrict__ counts, uint32_t *flags)
{
    const uint32_t nlisted = *fb_count;
    for (uint32_t e = blockIdx.x; e < nlisted; e += gridDim.x) {
        const int tile = (int)fb_list[e];
        const int tx = tile % tiles_x;
        const int rest = tile / tiles_x;
        const int cy = rest % g.ny;
        const int cz = rest / g.ny;
        const int cx0 = tx * kTileCells;
        const int G = min(kTileCells, g.nx - cx0);
        const int64_t rowc = ((int64_t)cz * g.ny + cy) * g.nx;
        const int32_t k0 = cell_start[rowc + cx0], k1 = cell_start[rowc + cx0 + G];
        for (int32_t k = k0 + threadIdx.x; k < k1; k += blockDim.x)
            pair_row_per_atom<false>(k, cell_pos, cell_start, atom_cell, g, K, nbr, counts, flags);
    }
}

constexpr size_t kStagedSmemCap = 200 * 1024;

size_t rows_smem(int W, int K) { return (size_t)W * 32 * (size_t)(K + 4) * sizeof(uint16_t); }

}  // namespace

cudaError_t pairs_set_attributes()
{
    return cudaFuncSetAttribute(k_pairs_staged, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kStagedSmemCap);
}

cudaError_t launch_pairs(nl_ctx *ctx, int64_t n, const CellGrid &g, int32_t capacity,
                         int32_t *nbr, int32_t *counts, cudaStream_t s, int *used_fast)
{
    *used_fast = 0;
    if (n <= 0) return cudaSuccess;
    // Two CTAs per SM when the rows of 3-4 warps fit beside a useful stage
    // (110 KB each), else one CTA with up to 200 KB.
    int W = 0, stage_max = 0;
    if (!g.literal && capacity % 4 == 0 && (reinterpret_cast<uintptr_t>(nbr) & 15u) == 0 &&
        n < (int64_t(1) << 31)) {
        for (int w = 4; w >= 1; --w) {
            const size_t budget = w >= 3 ? 110 * 1024 : kStagedSmemCap;
            const size_t rs = rows_smem(w, capacity);
            if (rs + sizeof(float4) * kStageMin <= budget) {
                W = w;
                stage_max = (int)((budget - rs) / sizeof(float4));
                if (stage_max > 8192) stage_max = 8192;
                break;
            }
        }
    }
    if (W > 0) {
        ProfScope ps(ctx, PH_PAIRS, s);
        StagedParams P;
        P.cell_pos = ctx->cell_pos;
        P.cell_start = ctx->cell_start;
        P.nbr = nbr;
        P.counts = counts;
        P.flags = ctx->flags;
        P.unsorted = ctx->unsorted;
        P.fb_list = ctx->fb_list;
        P.fb_count = ctx->fb_count;
        P.tiles_x = (g.nx + kTileCells - 1) / kTileCells;
        P.K = capacity;
        P.stage_max = stage_max;
        P.side_y = g.Ly / (float)g.ny;
        P.side_z = g.Lz / (float)g.nz;
        const float rl = sqrtf(g.rl2);
        const float Lmax = fmaxf(g.Lx, fmaxf(g.Ly, g.Lz));
        P.eps = 1e-3f * rl + 4e-6f * Lmax;
        P.rl2_margin = g.rl2 * (1.0f + 1e-4f);
        const int64_t ntiles = (int64_t)P.tiles_x * g.ny * g.nz;
        NL_CUDA_TRY(cudaMemsetAsync(ctx->fb_count, 0, sizeof(uint32_t), s));
        k_pairs_staged<<<(unsigned)ntiles, W * 32,
                         sizeof(float4) * stage_max + rows_smem(W, capacity), s>>>(g, P);
        NL_CUDA_TRY(cudaGetLastError());
        *used_fast = 1;
    }
    if (W > 0) {
        ProfScope ps(ctx, PH_PAIRS_FALLBACK, s);
        k_pairs_listed<<<(unsigned)(ctx->sm_count * 4), 128, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, ctx->atom_cell, g, capacity,
            (g.nx + kTileCells - 1) / kTileCells, ctx->fb_list, ctx->fb_count, nbr, counts,
            ctx->flags);
        return cudaGetLastError();
    }
    ProfScope ps(ctx, PH_PAIRS_FALLBACK, s);
    int64_t blocks = (n + 127) / 128;
    const int64_t cap = (int64_t)ctx->sm_count * 16;
    if (blocks > cap) blocks = cap;
    if (g.literal)
        k_pairs_per_atom<true><<<(unsigned)blocks, 128, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, ctx->atom_cell, n, g, capacity, nbr, counts, ctx->flags);
    else
        k_pairs_per_atom<false><<<(unsigned)blocks, 128, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, ctx->atom_cell, n, g, capacity, nbr, counts, ctx->flags);
    return cudaGetLastError();
}

}  // namespace nl
