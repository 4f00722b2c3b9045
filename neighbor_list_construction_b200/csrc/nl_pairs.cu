// nl_pairs.cu -- pair search and padded-row output.
//
// Tessera abstract: neighbor topology is held fixed between rebuilds, so the
// list is a fixed-capacity tensor (rows padded with -1, overflow reported).
//
// Minimum image without division.  For wrapped coordinates d = w_j - w_i lies
// in (-L, L).  On an axis with n cells of width >= c*rl and a stencil of +-w
// cells (w = 1 for c = 1 and n >= 5; w = 2 for c = 1/2 and n >= 7), two atoms
// whose cells differ by at most w without crossing the periodic face have
// |d| <= (w+1) L/n < L/2 (plus rounding far below the margin), so
// rintf(d/L) == 0 and the literal formula leaves d unchanged; across the face
// |d| >= L - (w+1) L/n > L/2, so rintf(d/L) == -+1 and the literal formula
// gives exactly fl(d + L) or fl(d - L).  The shift S in {-L, 0, +L} is thus
// known per stencil cell and fl(fl(w_j - w_i) + S) equals
// d - L*rintf(d/L) bit for bit.  Smaller boxes use the literal formula.
#include "nl_internal.cuh"

namespace nl {
namespace {

// ---------------------------------------------------------------------------
// Per-atom search: one thread per atom, the stencil cells straight from
// global memory, hits stored directly into the atom's row.  Used for small
// boxes (literal minimum image), for tiles the staged kernel cannot take,
// and when the staged kernel's preconditions fail.
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
    for (int oz = -g.wz; oz <= g.wz; ++oz) {
        int z = cz + oz;
        float sz = 0.0f;
        if (z < 0) { z += g.nz; sz = -g.Lz; } else if (z >= g.nz) { z -= g.nz; sz = g.Lz; }
        for (int oy = -g.wy; oy <= g.wy; ++oy) {
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
// Staged column search (column grid only: cells rl wide in x, rl/2 in y, z).
//
// A tile is kTileCells consecutive cells along x of one (cy, cz) column.
// Its 25 neighbor rows (dy, dz in -2..2), each covering cells cx0-1 ..
// cx0+G along x (plus one periodic image cell at either end of the box), are
// contiguous ranges of the cell-ordered array; one warp lane per row issues
// their cp.async.bulk copies into shared memory, completing on one mbarrier.
// Atoms of a row are sorted by x, so the candidates of a home atom in a row
// lie in the index window of [x - h, x + h], h = sqrt(rl^2 - d_perp^2) from
// the atom's distance to the row's (y, z) cell face, plus a margin.  The
// window ends come from a per-row table of first indices at 1/16-cell steps
// in x (conservative: a window never loses a candidate).  Each lane owns one
// home atom of the tile (the tile's home atoms are x-sorted and share one
// narrow (y, z) column, so their windows have similar lengths); every lane
// walks the warp's longest window length from its own start, so a lane may
// test atoms beyond its window -- harmless, since every tested pair is
// decided by the exact predicate.  Hits are kept as 16-bit stage slots in a
// per-lane row in shared memory and written out as full 16-byte row vectors.
// ---------------------------------------------------------------------------
constexpr int kTileCells = 8;          // G: cells per tile along x
constexpr int kRows = 25;              // (dy, dz) in -2..2
constexpr int kCenterRow = 12;         // dy = dz = 0
constexpr int kBinsPerCell = 16;       // x sub-bins per cell (tables built by k_cell_sort)
constexpr int kRowCells = kTileCells + 2;
constexpr int kStageMin = 2048;        // fewest staged atoms worth a launch

struct ColTile {
    int row_off[kRows];
    int row_len[kRows];
    int row_lend[kRows];   // [0, lend): periodic image cell at the low x end (shift -Lx)
    int row_rbeg[kRows];   // [rbeg, len): periodic image cell at the high x end (shift +Lx)
    float row_sy[kRows];
    float row_sz[kRows];
    int row_cell[kRows][kRowCells + 1];   // staged start of each conceptual cell, then len
    int total;
    int home_begin, home_end;
    int fallback;
};

struct ColParams {
    const float4 *cell_pos;
    const int32_t *cell_start;
    int32_t *nbr;
    int32_t *counts;
    uint32_t *flags;
    const uint32_t *unsorted;
    uint32_t *fb_list;
    uint32_t *fb_count;
    const uint8_t *cell_tab;
    int tiles_x;
    int K;
    int B;              // row entries kept in shared memory (multiple of 4, <= K)
    int stage_max;      // staged atoms per tile
    float side_x, side_y, side_z;
    float inv_bin;      // kBinsPerCell / side_x (as in k_cell_sort)
    float eps;          // window margin (A)
    float rl2_margin;   // rl2 * (1 + 1e-4)
};

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts_u16(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"((unsigned short)v) : "memory");
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

// Waits for the phase with the given parity to complete; the thread is
// suspended (up to ~1 ms per call) instead of spinning.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}

// One contiguous global -> shared copy completing on `bar` (16-byte multiples).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Row output of one lane: the first B neighbor indices go to the lane's
// buffer in shared memory (bp = next free byte, bufend = its end); entries
// B .. K-1 of long rows go straight to the lane's global row (byte address of
// entry e = gmap + smem address of entry e); entries past K are only counted.
struct RowOut {
    uint32_t bp, bufend, rowend;
    uint64_t gmap;
};

// Appends `idx` when r2 < rl2 (and, for the home row, idx != self).  FAST:
// no lane can pass B in this row -- one predicated shared store and a
// predicated bump, no branch.  Otherwise also the global spill and the
// capacity cut-off.
template <bool SELF, bool FAST>
__device__ __forceinline__ void append_if_hit(float r2, float rl2, uint32_t idx, uint32_t self,
                                              RowOut &o)
{
    if (FAST) {
        if (SELF)
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.lt.f32 p, %1, %2;\n\t"
                "setp.ne.and.u32 p, %3, %4, p;\n\t"
                "@p st.shared.b32 [%0], %3;\n\t"
                "@p add.u32 %0, %0, 4;\n\t}"
                : "+r"(o.bp)
                : "f"(r2), "f"(rl2), "r"(idx), "r"(self));
        else
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.lt.f32 p, %1, %2;\n\t"
                "@p st.shared.b32 [%0], %3;\n\t"
                "@p add.u32 %0, %0, 4;\n\t}"
                : "+r"(o.bp)
                : "f"(r2), "f"(rl2), "r"(idx));
    } else {
        const uint64_t ga = o.gmap + (uint64_t)o.bp;
        asm volatile(
            "{\n\t.reg .pred p, ps, pg;\n\t"
            "setp.lt.f32 p, %1, %2;\n\t"
            "setp.ne.and.u32 p, %3, %4, p;\n\t"
            "setp.lt.and.u32 ps, %0, %5, p;\n\t"
            "setp.ge.and.u32 pg, %0, %5, p;\n\t"
            "setp.lt.and.u32 pg, %0, %6, pg;\n\t"
            "@ps st.shared.b32 [%0], %3;\n\t"
            "@pg st.global.b32 [%7], %3;\n\t"
            "@p add.u32 %0, %0, 4;\n\t}"
            : "+r"(o.bp)
            : "f"(r2), "f"(rl2), "r"(idx), "r"(SELF ? self : 0xffffffffu), "r"(o.bufend),
              "r"(o.rowend), "l"(ga));
    }
}

// One contiguous shared -> global copy (16-byte aligned, 16-byte multiple),
// tracked in this thread's bulk group.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until this thread's bulk copies have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// r2 of one candidate against this lane's atom, with the row's periodic
// shifts (XS: x image cells at the row ends; YZ: the row's y/z shift).
template <bool XS, bool YZ>
__device__ __forceinline__ float cand_r2(const float4 q, const float4 me, int s, float Lx,
                                         int lend_slot, int rbeg_slot, float sy, float sz)
{
    float dx = __fsub_rn(q.x, me.x);
    float dy = __fsub_rn(q.y, me.y);
    float dz = __fsub_rn(q.z, me.z);
    if (XS) dx = __fadd_rn(dx, s < lend_slot ? -Lx : (s >= rbeg_slot ? Lx : 0.0f));
    if (YZ) {
        dy = __fadd_rn(dy, sy);
        dz = __fadd_rn(dz, sz);
    }
    return r2_of(dx, dy, dz);
}

// One candidate, no periodic shift, as explicit PTX: three fp32
// differences, three products, two sums, all round-to-nearest with no
// contraction; on r2 < rl2 (and, for the home row, idx != self) append idx
// to the row buffer.  Only used with FAST (no lane can pass B).
template <bool SELF>
__device__ __forceinline__ void test_plain(const float4 c, const float4 me, float rl2,
                                           uint32_t self, uint32_t &bp)
{
    if (SELF)
        asm volatile(
            "{\n\t.reg .f32 dx, dy, dz, s;\n\t.reg .pred p;\n\t"
            "sub.rn.f32 dx, %1, %5;\n\t"
            "sub.rn.f32 dy, %2, %6;\n\t"
            "sub.rn.f32 dz, %3, %7;\n\t"
            "mul.rn.f32 dx, dx, dx;\n\t"
            "mul.rn.f32 dy, dy, dy;\n\t"
            "mul.rn.f32 dz, dz, dz;\n\t"
            "add.rn.f32 s, dx, dy;\n\t"
            "add.rn.f32 s, s, dz;\n\t"
            "setp.lt.f32 p, s, %8;\n\t"
            "setp.ne.and.u32 p, %4, %9, p;\n\t"
            "@p st.shared.b32 [%0], %4;\n\t"
            "@p add.u32 %0, %0, 4;\n\t}"
            : "+r"(bp)
            : "f"(c.x), "f"(c.y), "f"(c.z), "r"(__float_as_uint(c.w)), "f"(me.x), "f"(me.y),
              "f"(me.z), "f"(rl2), "r"(self));
    else
        asm volatile(
            "{\n\t.reg .f32 dx, dy, dz, s;\n\t.reg .pred p;\n\t"
            "sub.rn.f32 dx, %1, %5;\n\t"
            "sub.rn.f32 dy, %2, %6;\n\t"
            "sub.rn.f32 dz, %3, %7;\n\t"
            "mul.rn.f32 dx, dx, dx;\n\t"
            "mul.rn.f32 dy, dy, dy;\n\t"
            "mul.rn.f32 dz, dz, dz;\n\t"
            "add.rn.f32 s, dx, dy;\n\t"
            "add.rn.f32 s, s, dz;\n\t"
            "setp.lt.f32 p, s, %8;\n\t"
            "@p st.shared.b32 [%0], %4;\n\t"
            "@p add.u32 %0, %0, 4;\n\t}"
            : "+r"(bp)
            : "f"(c.x), "f"(c.y), "f"(c.z), "r"(__float_as_uint(c.w)), "f"(me.x), "f"(me.y),
              "f"(me.z), "f"(rl2));
}

// Tests L consecutive candidates q[0..L) of one row (stage slots slot0 ..)
// against this lane's atom: groups of 8, then of 4, then single ones.
template <bool XS, bool YZ, bool SELF, bool FAST>
__device__ __forceinline__ void scan_row(const float4 *__restrict__ q, int slot0, int L,
                                         const float4 me, float Lx, int lend_slot, int rbeg_slot,
                                         float sy, float sz, float rl2, RowOut &o)
{
    const uint32_t self = (uint32_t)__float_as_int(me.w);
    int k = 0;
    if (!XS && !YZ && FAST) {
        uint32_t bp = o.bp;
        for (; k + 8 <= L; k += 8) {
            float4 c[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) c[u] = q[k + u];
#pragma unroll
            for (int u = 0; u < 8; ++u) test_plain<SELF>(c[u], me, rl2, self, bp);
        }
        for (; k < L; ++k) test_plain<SELF>(q[k], me, rl2, self, bp);
        o.bp = bp;
        return;
    }
    for (; k + 8 <= L; k += 8) {
        float4 c[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) c[u] = q[k + u];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            append_if_hit<SELF, FAST>(
                cand_r2<XS, YZ>(c[u], me, slot0 + k + u, Lx, lend_slot, rbeg_slot, sy, sz), rl2,
                (uint32_t)__float_as_int(c[u].w), self, o);
    }
    if (k + 4 <= L) {
        float4 c[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) c[u] = q[k + u];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            append_if_hit<SELF, FAST>(
                cand_r2<XS, YZ>(c[u], me, slot0 + k + u, Lx, lend_slot, rbeg_slot, sy, sz), rl2,
                (uint32_t)__float_as_int(c[u].w), self, o);
        k += 4;
    }
    for (; k < L; ++k) {
        const float4 c = q[k];
        append_if_hit<SELF, FAST>(
            cand_r2<XS, YZ>(c, me, slot0 + k, Lx, lend_slot, rbeg_slot, sy, sz), rl2,
            (uint32_t)__float_as_int(c.w), self, o);
    }
}

__global__ void __launch_bounds__(64)
k_pairs_columns(const CellGrid g, const ColParams P)
{
    extern __shared__ __align__(16) unsigned char col_smem[];
    float4 *stage = reinterpret_cast<float4 *>(col_smem);
    uint8_t *tabs = col_smem + sizeof(float4) * P.stage_max;   // [kRows][kRowCells][16]
    int32_t *rows = reinterpret_cast<int32_t *>(tabs + kRows * kRowCells * kBinsPerCell);
    __shared__ ColTile ti;
    __shared__ __align__(8) uint64_t bar;

    const int W = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = P.B;        // neighbor indices kept in shared memory per row
    const int RS = B + 4;     // row stride in words (rows 16-byte aligned for bulk copies)
    int32_t *negs = rows + W * 32 * RS;   // P.K entries of -1, the padding source
    for (int e = threadIdx.x; e < P.K; e += blockDim.x) negs[e] = -1;
    const int tile = blockIdx.x;
    const int tx = tile % P.tiles_x;
    const int rest = tile / P.tiles_x;
    const int cy = rest % g.ny;
    const int cz = rest / g.ny;
    const int cx0 = tx * kTileCells;
    const int G = min(kTileCells, g.nx - cx0);
    const uint32_t stage_base = smem_u32(stage);

    // ---- row table: lane r of warp 0 describes row r (its atoms and the
    //      x tables of its G+2 conceptual cells cx0-1 .. cx0+G)
    if (warp == 0) {
        int seg_src[3] = {0, 0, 0}, seg_cnt[3] = {0, 0, 0};
        int64_t tab_src[3] = {0, 0, 0};
        int tab_cnt[3] = {0, 0, 0};
        int nseg = 0, len = 0;
        if (lane == 0) mbar_init(&bar, 1);
        if (lane < kRows) {
            const int dy = lane % 5 - 2, dz = lane / 5 - 2;
            int y = cy + dy, z = cz + dz;
            float sy = 0.0f, sz = 0.0f;
            if (y < 0) { y += g.ny; sy = -g.Ly; } else if (y >= g.ny) { y -= g.ny; sy = g.Ly; }
            if (z < 0) { z += g.nz; sz = -g.Lz; } else if (z >= g.nz) { z -= g.nz; sz = g.Lz; }
            const int64_t rowc = ((int64_t)z * g.ny + y) * g.nx;
            int k = 0;
            if (cx0 == 0) {  // conceptual cell -1 is cell nx-1
                const int a = P.cell_start[rowc + g.nx - 1], b = P.cell_start[rowc + g.nx];
                seg_src[nseg] = a;
                seg_cnt[nseg] = b - a;
                tab_src[nseg] = rowc + g.nx - 1;
                tab_cnt[nseg] = 1;
                ++nseg;
                ti.row_cell[lane][k++] = 0;
                len += b - a;
            }
            ti.row_lend[lane] = len;
            const int first = cx0 == 0 ? 0 : cx0 - 1;
            const int last = cx0 + G <= g.nx - 1 ? cx0 + G : g.nx - 1;
            const int a = P.cell_start[rowc + first];
            for (int cc = first; cc <= last; ++cc)
                ti.row_cell[lane][k++] = len + (P.cell_start[rowc + cc] - a);
            const int b = P.cell_start[rowc + last + 1];
            seg_src[nseg] = a;
            seg_cnt[nseg] = b - a;
            tab_src[nseg] = rowc + first;
            tab_cnt[nseg] = last - first + 1;
            ++nseg;
            if (lane == kCenterRow) {
                ti.home_begin = len + (P.cell_start[rowc + cx0] - a);
                ti.home_end = len + (P.cell_start[rowc + cx0 + G] - a);
            }
            len += b - a;
            ti.row_rbeg[lane] = len;
            if (cx0 + G == g.nx) {  // conceptual cell nx is cell 0
                const int a2 = P.cell_start[rowc], b2 = P.cell_start[rowc + 1];
                seg_src[nseg] = a2;
                seg_cnt[nseg] = b2 - a2;
                tab_src[nseg] = rowc;
                tab_cnt[nseg] = 1;
                ++nseg;
                ti.row_cell[lane][k++] = len;
                len += b2 - a2;
            }
            ti.row_cell[lane][k] = len;   // k == G + 2
            ti.row_len[lane] = len;
            ti.row_sy[lane] = sy;
            ti.row_sz[lane] = sz;
        }
        __syncwarp();
        // exclusive scan of the row lengths -> row offsets
        int x = len;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        const int off = x - len;
        const int total = __shfl_sync(0xffffffffu, x, 31);
        if (lane < kRows) ti.row_off[lane] = off;
        if (lane == kCenterRow) {
            ti.home_begin += off;
            ti.home_end += off;
        }
        const int fb = (total > P.stage_max || *P.unsorted != 0u) ? 1 : 0;
        if (lane == 0) {
            ti.total = total;
            ti.fallback = fb;
            if (fb) {
                const uint32_t slot = atomicAdd(P.fb_count, 1u);
                P.fb_list[slot] = (uint32_t)tile;
            } else {
                asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
                mbar_arrive_expect_tx(
                    &bar, (uint32_t)total * 16u + (uint32_t)(kRows * (G + 2) * kBinsPerCell));
            }
        }
        __syncwarp();
        if (!fb && lane < kRows) {
            uint32_t dst = stage_base + 16u * (uint32_t)off;
            uint32_t tdst = smem_u32(tabs) + (uint32_t)(lane * kRowCells * kBinsPerCell);
            for (int sg = 0; sg < nseg; ++sg) {
                if (seg_cnt[sg] > 0)
                    bulk_g2s(dst, P.cell_pos + seg_src[sg], (uint32_t)seg_cnt[sg] * 16u, &bar);
                dst += 16u * (uint32_t)seg_cnt[sg];
                bulk_g2s(tdst, P.cell_tab + tab_src[sg] * kBinsPerCell,
                         (uint32_t)(tab_cnt[sg] * kBinsPerCell), &bar);
                tdst += (uint32_t)(tab_cnt[sg] * kBinsPerCell);
            }
        }
    }
    __syncthreads();
    if (ti.fallback) return;
    {
        uint32_t spins = 0;
        while (!mbar_try_wait(&bar, 0)) {
            if (++spins >= 4096u) {   // ~4 s
                if (threadIdx.x == 0) atomicOr(P.flags, kFlagTimeout);
                return;
            }
        }
    }

    const float X0 = (float)(cx0 - 1) * P.side_x;   // low x face of conceptual cell 0
    const int nbins = (G + 2) * kBinsPerCell;
    const float rl2 = g.rl2;
    const int nhome = ti.home_end - ti.home_begin;
    const int nchunks = (nhome + 31) >> 5;
    const uint32_t mybuf = smem_u32(rows) + 4u * (uint32_t)((warp * 32 + lane) * RS);
    const float ylo = (float)cy * P.side_y, yhi = (float)(cy + 1) * P.side_y;
    const float zlo = (float)cz * P.side_z, zhi = (float)(cz + 1) * P.side_z;

    for (int c = warp; c < nchunks; c += W) {
        const int a = ti.home_begin + c * 32 + lane;
        const bool valid = a < ti.home_end;
        const float4 me =
            valid ? stage[a] : make_float4(-1e30f, -1e30f, -1e30f, __int_as_float(-1));
        const float dy_lo = me.y - ylo, dy_hi = yhi - me.y;
        const float dz_lo = me.z - zlo, dz_hi = zhi - me.z;
        const int myid = __float_as_int(me.w);
        bulk_wait_read();   // the previous chunk's rows have left this buffer
        RowOut o;
        o.bp = mybuf;
        o.bufend = mybuf + 4u * (uint32_t)B;
        o.rowend = mybuf + 4u * (uint32_t)P.K;
        o.gmap = (uint64_t)(uintptr_t)(P.nbr + (int64_t)(valid ? myid : 0) * P.K) - (uint64_t)mybuf;
        for (int r = 0; r < kRows; ++r) {
            const int dy = r % 5 - 2, dz = r / 5 - 2;
            const int off = ti.row_off[r], len = ti.row_len[r];
            if (len == 0) continue;
            float py = dy > 0 ? dy_hi + (float)(dy - 1) * P.side_y
                              : (dy < 0 ? dy_lo + (float)(-dy - 1) * P.side_y : 0.0f);
            float pz = dz > 0 ? dz_hi + (float)(dz - 1) * P.side_z
                              : (dz < 0 ? dz_lo + (float)(-dz - 1) * P.side_z : 0.0f);
            py = fmaxf(py - P.eps, 0.0f);
            pz = fmaxf(pz - P.eps, 0.0f);
            const float h2 = P.rl2_margin - (py * py + pz * pz);
            int lo = 0, hi = 0;
            if (valid && h2 > 0.0f) {
                // first index at or above bin b = start of b's cell + cell table entry
                // approximate root (relative error ~1e-6): the margin absorbs it
                const float h = h2 * rsqrtf(h2) + P.eps;
                const uint8_t *tb = tabs + r * (kRowCells * kBinsPerCell);
                const int *rc = ti.row_cell[r];
                const int b0 = max(0, min((int)floorf((me.x - h - X0) * P.inv_bin), nbins - 1));
                const int b1 = (int)floorf((me.x + h - X0) * P.inv_bin) + 1;
                lo = rc[b0 >> 4] + tb[b0];
                hi = b1 >= nbins ? len : (b1 <= 0 ? 0 : rc[b1 >> 4] + tb[b1]);
                if (hi < lo) hi = lo;
            }
            const int Lmax = __reduce_max_sync(0xffffffffu, hi - lo);
            if (Lmax == 0) continue;
            // whole groups of 4 when the row is long enough (extra tests are harmless)
            const int L = min((Lmax + 3) & ~3, len);
            const int st = lo < len - L ? lo : len - L;
            const int lend = ti.row_lend[r], rbeg = ti.row_rbeg[r];
            // image shifts are needed as soon as any lane's tested range
            // [st, st + L) reaches an image cell (not only its exact window):
            // an unshifted image copy of a cell could otherwise pair with a
            // home atom that also meets the cell's own copy
            const bool xs = __any_sync(0xffffffffu, st < lend || st + L > rbeg);
            const bool yz = ti.row_sy[r] != 0.0f || ti.row_sz[r] != 0.0f;
            const bool fast = !__any_sync(0xffffffffu, o.bp + 4u * (uint32_t)L > o.bufend);
            const float sy = ti.row_sy[r], sz = ti.row_sz[r];
            const float4 *a0 = stage + off + st;
            const int slot0 = off + st;
            const int ls = off + lend, rs = off + rbeg;
            const float Lx = g.Lx;
            if (r == kCenterRow) {
                if (xs) {
                    if (fast) scan_row<true, false, true, true>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                    else scan_row<true, false, true, false>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                } else {
                    if (fast) scan_row<false, false, true, true>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                    else scan_row<false, false, true, false>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                }
            } else if (!yz) {
                if (xs) {
                    if (fast) scan_row<true, false, false, true>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                    else scan_row<true, false, false, false>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                } else {
                    if (fast) scan_row<false, false, false, true>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                    else scan_row<false, false, false, false>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                }
            } else {
                if (xs) {
                    if (fast) scan_row<true, true, false, true>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                    else scan_row<true, true, false, false>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                } else {
                    if (fast) scan_row<false, true, false, true>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                    else scan_row<false, true, false, false>(a0, slot0, L, me, Lx, ls, rs, sy, sz, rl2, o);
                }
            }
        }
        const int cnt = (int)((o.bp - mybuf) >> 2);
        if (valid) {
            P.counts[myid] = cnt;
            if (cnt > P.K) atomicOr(P.flags, kFlagOverflow);
            // the lane's row leaves by bulk copies: buffered hits rounded up to a
            // whole 16-byte vector with -1, then -1 from `negs` up to K; entries
            // B .. min(cnt, K)-1 of a long row are already in global memory
            int32_t *rowbuf = rows + (warp * 32 + lane) * RS;
            int32_t *grow = P.nbr + (int64_t)myid * P.K;
            const int nsm = cnt < B ? cnt : B;
            const int n1 = (nsm + 3) & ~3;
            for (int e = nsm; e < n1; ++e) rowbuf[e] = -1;
            int npad_from = n1;
            if (cnt > B) {
                const int ntot = cnt < P.K ? cnt : P.K;
                npad_from = (ntot + 3) & ~3;
                for (int e = ntot; e < npad_from; ++e) grow[e] = -1;
            }
            fence_proxy_async_smem();
            if (n1 > 0) bulk_s2g(grow, mybuf, 4u * (uint32_t)n1);
            if (P.K > npad_from)
                bulk_s2g(grow + npad_from, smem_u32(negs), 4u * (uint32_t)(P.K - npad_from));
            bulk_commit();
        }
    }
    bulk_wait_all();
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

constexpr size_t kColSmemCap = 200 * 1024;
constexpr int kColWarps = 2;

constexpr int kRowBuffer = 128;   // row entries kept in shared memory

int row_buffer(int K) { return K < kRowBuffer ? K : kRowBuffer; }

size_t col_fixed_smem(int W, int K)
{
    const size_t tabs = (size_t)kRows * kRowCells * kBinsPerCell;
    const size_t rows = (size_t)W * 32 * (size_t)(row_buffer(K) + 4) * sizeof(int32_t);
    const size_t negs = (size_t)K * sizeof(int32_t);
    return tabs + rows + negs;
}

}  // namespace

cudaError_t pairs_set_attributes()
{
    return cudaFuncSetAttribute(k_pairs_columns, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kColSmemCap);
}

cudaError_t launch_pairs(nl_ctx *ctx, int64_t n, const CellGrid &g, int32_t capacity,
                         int32_t *nbr, int32_t *counts, cudaStream_t s, int *used_fast)
{
    *used_fast = 0;
    if (n <= 0) return cudaSuccess;
    // Staged kernel: column grid and rows of whole 16-byte vectors.  The
    // stage must hold a typical tile (25 rows x (G+2) cells at the mean cell
    // occupancy) with 25 % to spare; take the smallest shared-memory budget
    // (3, 2 or 1 CTAs per SM) that does.  Denser tiles fall back per atom.
    int stage_max = 0;
    const int W = kColWarps;
    if (g.wy == 2 && !g.literal && capacity % 4 == 0 &&
        (reinterpret_cast<uintptr_t>(nbr) & 15u) == 0 && n < (int64_t(1) << 31)) {
        const size_t fixed = col_fixed_smem(W, capacity);
        const double per_cell = (double)n / (double)g.ncell;
        const int want = (int)(1.1 * per_cell * kRows * (kTileCells + 2)) + 32;
        const int need = want > kStageMin ? want : kStageMin;
        // per-SM 228 KB less 1 KB per CTA and the static tile table
        for (size_t budget : {size_t(73) * 1024, size_t(110) * 1024, kColSmemCap}) {
            const int fit = budget > fixed ? (int)((budget - fixed) / sizeof(float4)) : 0;
            if (fit >= need || budget == kColSmemCap) {
                stage_max = fit < 8192 ? fit : 8192;
                break;
            }
        }
        if (stage_max < 256) stage_max = 0;
    }
    if (stage_max > 0) {
        ColParams P;
        P.cell_pos = ctx->cell_pos;
        P.cell_start = ctx->cell_start;
        P.nbr = nbr;
        P.counts = counts;
        P.flags = ctx->flags;
        P.unsorted = ctx->unsorted;
        P.fb_list = ctx->fb_list;
        P.fb_count = ctx->fb_count;
        P.cell_tab = ctx->cell_tab;
        P.tiles_x = (g.nx + kTileCells - 1) / kTileCells;
        P.K = capacity;
        P.B = row_buffer(capacity);
        P.stage_max = stage_max;
        P.side_x = g.Lx / (float)g.nx;
        P.side_y = g.Ly / (float)g.ny;
        P.side_z = g.Lz / (float)g.nz;
        P.inv_bin = (float)kBinsPerCell / P.side_x;
        const float rl = sqrtf(g.rl2);
        const float Lmax = fmaxf(g.Lx, fmaxf(g.Ly, g.Lz));
        P.eps = 1e-3f * rl + 4e-6f * Lmax;
        P.rl2_margin = g.rl2 * (1.0f + 1e-4f);
        const int64_t ntiles = (int64_t)P.tiles_x * g.ny * g.nz;
        const size_t smem = sizeof(float4) * (size_t)stage_max + col_fixed_smem(W, capacity);
        NL_CUDA_TRY(cudaMemsetAsync(ctx->fb_count, 0, sizeof(uint32_t), s));
        {
            ProfScope ps(ctx, PH_PAIRS, s);
            k_pairs_columns<<<(unsigned)ntiles, W * 32, smem, s>>>(g, P);
            NL_CUDA_TRY(cudaGetLastError());
        }
        *used_fast = 1;
        ProfScope ps(ctx, PH_PAIRS_FALLBACK, s);
        k_pairs_listed<<<(unsigned)(ctx->sm_count * 4), 128, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, ctx->atom_cell, g, capacity, P.tiles_x, ctx->fb_list,
            ctx->fb_count, nbr, counts, ctx->flags);
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
