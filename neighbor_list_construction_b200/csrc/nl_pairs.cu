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

// Close-pair accumulator of one thread: smallest r2 of its hits (+inf when
// none) and the number of hits with r2 < close_d2.
struct CloseAcc {
    float mn;
    uint32_t nc;
};

// Folds a warp's accumulators into the global minimum (r2 >= 0, so the
// float bits order like unsigned integers) and count.
__device__ __forceinline__ void close_publish(const CloseAcc &cl, uint32_t *min_bits,
                                              unsigned long long *n_close)
{
    const uint32_t mb = __reduce_min_sync(0xffffffffu, __float_as_uint(cl.mn));
    const uint32_t nc = __reduce_add_sync(0xffffffffu, cl.nc);
    if ((threadIdx.x & 31) == 0) {
        if (mb != 0x7f800000u) atomicMin(min_bits, mb);
        if (nc) atomicAdd(n_close, (unsigned long long)nc);
    }
}


// ---------------------------------------------------------------------------
// Per-atom search: one thread per atom, the stencil cells straight from
// global memory, hits stored directly into the atom's row.  Used for small
// boxes (literal minimum image), for tiles the staged kernel cannot take,
// and when the staged kernel's preconditions fail.
// ---------------------------------------------------------------------------
template <bool LITERAL, bool CLOSE>
__device__ __forceinline__ void pair_row_per_atom(int64_t k, const float4 *__restrict__ cell_pos,
                                                  const int32_t *__restrict__ cell_start,
                                                  const uint32_t *__restrict__ atom_cell,
                                                  const CellGrid &g, int32_t K,
                                                  int32_t *__restrict__ nbr,
                                                  int32_t *__restrict__ counts, uint32_t *flags,
                                                  float close_d2, CloseAcc &cl)
{
    const float4 p = cell_pos[k];
    const int i = __float_as_int(p.w);
    if (i >= g.n_rows) return;   // no row for this atom
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
                    const float r2 = r2_of(dx, dy, dz);
                    if (r2 < g.rl2) {
                        if (cnt < K) row[cnt] = jid;
                        ++cnt;
                        if (CLOSE) {
                            cl.mn = fminf(cl.mn, r2);
                            cl.nc += r2 < close_d2 ? 1u : 0u;
                        }
                    }
                }
            }
        }
    }
    counts[i] = cnt;
    for (int e = cnt < K ? cnt : K; e < K; ++e) row[e] = -1;
    if (cnt > K) atomicOr(flags, kFlagOverflow);
}

template <bool LITERAL, bool CLOSE>
__global__ void __launch_bounds__(128)
k_pairs_per_atom(const float4 *__restrict__ cell_pos, const int32_t *__restrict__ cell_start,
                 const uint32_t *__restrict__ atom_cell, int64_t n, CellGrid g, int32_t K,
                 int32_t *__restrict__ nbr, int32_t *__restrict__ counts, uint32_t *flags,
                 float close_d2, uint32_t *min_bits, unsigned long long *n_close)
{
    if (timed_out(flags)) return;   // cell starts may not be monotonic
    n = atoms_of(g, n);
    CloseAcc cl{__int_as_float(0x7f800000), 0u};
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
        pair_row_per_atom<LITERAL, CLOSE>(k, cell_pos, cell_start, atom_cell, g, K, nbr, counts,
                                          flags, close_d2, cl);
    if (CLOSE) close_publish(cl, min_bits, n_close);
}

// ---------------------------------------------------------------------------
// Staged tile search (column grid only: cells >= rl wide in x, >= rl/2 in y
// and z, so the stencil is +-1 cell in x and +-2 cells in y and z).
//
// A tile is kTX x kTY x kTZ home cells.  Its staged rows (y and z from
// two cells below to two cells above the home block) each cover the
// conceptual cells cx0-1 .. cx0+Gx along x, with a periodic image cell at
// either end of the box.  Every row is a contiguous range of the
// cell-ordered array; one lane per row issues its cp.async.bulk copies into
// shared memory, all completing on the stage's mbarrier.
//
// A home atom meets 25 rows (dy, dz in -2..2).  Atoms of a row are sorted by
// x, so its candidates in a row lie in the slot window of [x - h, x + h],
// h = sqrt(rl^2 - d_perp^2) from the atom's distance to the row's (y, z)
// cell face plus a margin; the window ends come from per-cell tables of
// first slots at 1/16-cell steps in x (conservative: no candidate is lost).
// A warp scans one row for all its lanes at once: the lanes are consecutive
// x-sorted home atoms, so at each step their windows sit on nearly
// consecutive slots; a lane past its own window loads nothing.  The home row
// is scanned in two ranges around the atom's own slot, so self never reaches
// the predicate.
//
// Hits go to a small per-lane buffer in shared memory, interleaved across
// the warp's lanes so that each per-slot store falls in the lane's own bank;
// when a lane holds kFlushAt entries the warp stores its whole 16-byte
// vectors to the rows.  Rows are finished with one cp.async.bulk copy from a
// shared block of -1.
// ---------------------------------------------------------------------------
constexpr int kTX = 3, kTY = 4, kTZ = 4;   // home cells per tile
constexpr int kSY = kTY + 4, kSZ = kTZ + 4;
constexpr int kSRows = kSY * kSZ;           // staged rows (64)
static_assert(kSRows <= 64, "a tile's rows are described two per lane of one warp");
constexpr int kHome = kTY * kTZ;            // home rows (16)
static_assert(kHome <= 32, "home rows are counted one per lane");
constexpr int kSCells = kTX + 2;            // conceptual cells per staged row
constexpr int kBinsPerCell = 16;            // x sub-bins per cell (tables built by k_cell_sort)
constexpr int kRowTab = kSCells * kBinsPerCell;
// A warp flush costs the same whatever it moves, so hits are flushed late:
// kFlushAt pending entries in some lane.  The buffer then holds at most
// kFlushAt - 1 pending plus one group of 4 new.  Measured on saltwater10m
// (pair search, ms): flush at 8 with 24 searching warps 5.11; at 16, 4.79;
// at 24 with 20 warps 4.45 (16 warps 4.73; larger buffers leave stages too
// small for the densest tiles).
constexpr int kFlushAt = 24;                // pending hits that make the warp flush
constexpr int kBuf = kFlushAt + 4;          // entries of a lane's hit buffer
constexpr uint32_t kHitStride = 128;        // bytes between a lane's buffer entries (32 lanes x 4)
constexpr int kPipeStages = 3;              // most staged tiles per CTA of the persistent launch
constexpr int kPipeMeta = kPipeStages + 1;  // tile descriptions: one ahead of the stages
constexpr int kPipeConsumers = 20;          // searching warps per CTA (plus one staging warp)
constexpr int kPipeThreads = 32 * (1 + kPipeConsumers);
constexpr int kQueue = 512;                 // chunk-queue entries
constexpr uint32_t kQueueEnd = 0xffffffffu;
constexpr uint32_t kEmptyCount = 1u << 16;  // arrivals that free a stage: the staging warp's
                                            // (kEmptyCount - chunks) plus one per chunk
constexpr int kListedWarps = 5;             // warps of a listed-tile CTA
constexpr int kListedCtas = 3;              // CTAs per SM the listed-tile launch may use
constexpr int kStageMin = 1024;             // fewest staged slots worth a launch

struct TileRows {
    int off[kSRows];                 // slot of the row's first atom
    int len[kSRows];
    int cell[kSRows][kSCells + 1];   // row-local start of conceptual cell k
    int home_begin[kHome];           // slot of the first home atom of home row h
    int home_pref[kHome + 1];        // home atoms before home row h
    int total;                       // staged slots, gaps included
    int fallback;
};

// Where a staged tile sits in the grid.
struct TileMeta {
    int cx0, cy0, cz0;     // first home cell
    int Gx, Gy, Gz;        // home cells (fewer at the high faces)
    int general;           // touches a periodic face: shifted scans where needed
};

struct TileParams {
    float close_d2;                 // close-pair threshold (CLOSE kernels)
    uint32_t *min_bits;             // float bits of the smallest pair r2 (CLOSE)
    unsigned long long *n_close;    // directed pairs with r2 < close_d2 (CLOSE)
    const float4 *cell_pos;
    const uint32_t *atom_cell;
    const int32_t *cell_start;
    const uint8_t *cell_tab;
    int32_t *nbr;
    int32_t *counts;
    uint32_t *flags;
    const uint32_t *unsorted;
    uint32_t *fb_list;
    uint32_t *fb_count;
    uint32_t *tile_ctr;             // next tile (or list entry) of the persistent launch
    const uint32_t *tile_list;      // the tiles to take, or NULL: every tile in order
    const uint32_t *tile_list_count;
    int stages;                     // shared-memory stages of a persistent CTA (1..kPipeStages)
    int tiles_x, tiles_y;
    int ntiles;
    int K;
    int stage_max;      // staged slots per tile, gaps included
    float side_x, side_y, side_z;
    float inv_bin;      // kBinsPerCell / side_x (as in k_cell_sort)
    float eps;          // window margin (A)
    float rl2_margin;   // rl2 * (1 + 1e-4)
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

// Arrival of this thread (release: its earlier shared-memory reads and
// writes are ordered before the phase completes), counting `count` arrivals.
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(count)
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

// Waits until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Four consecutive slots at shared address `addr` of which the first `act`
// (0..4 or more) belong to this lane's range: the active ones are loaded
// into c[0..3] (an inactive slot keeps a stale value), and each is tested:
// three fp32 differences (each followed by its periodic shift when GEN),
// three products and two sums, round-to-nearest with no contraction --
// (dx*dx + dy*dy) + dz*dz -- a hit requiring r2 < rl2 and the slot to be
// active.  A hit stores the candidate's index at bp and moves bp to the
// lane's next buffer entry, 128 bytes on (kHitStride).  GEN: x shifts
// sx0..sx3 per slot and the row's y, z shifts.  CLOSE: each hit also lowers
// cl.mn to its r2 and counts in cl.nc when r2 < close_d2.
template <bool GEN, bool CLOSE>
__device__ __forceinline__ void scan4(uint32_t addr, int act, float4 (&c)[4], const float4 me,
                                      float rl2, float sx0, float sx1, float sx2, float sx3,
                                      float sy, float sz, float close_d2, CloseAcc &cl,
                                      uint32_t &bp)
{
    // (me.x, me.y) as one packed pair for the f32x2 forms: x in the low half
    const unsigned long long mxy =
        ((unsigned long long)__float_as_uint(me.y) << 32) | __float_as_uint(me.x);
    if (GEN && CLOSE)
        asm volatile("{\n\t.reg .f32 dx, dy, dz;\n\t.reg .pred q0, q1, q2, q3, qc;\n\t"
                     "setp.gt.s32 q0, %19, 0;\n\t"
                     "setp.gt.s32 q1, %19, 1;\n\t"
                     "setp.gt.s32 q2, %19, 2;\n\t"
                     "setp.gt.s32 q3, %19, 3;\n\t"
                     "@q0 ld.shared.v4.f32 {%1, %2, %3, %4}, [%20];\n\t"
                     "@q1 ld.shared.v4.f32 {%5, %6, %7, %8}, [%20+16];\n\t"
                     "@q2 ld.shared.v4.f32 {%9, %10, %11, %12}, [%20+32];\n\t"
                     "@q3 ld.shared.v4.f32 {%13, %14, %15, %16}, [%20+48];\n\t"
                     "sub.rn.f32 dx, %1, %21;\n\t"
                     "sub.rn.f32 dy, %2, %22;\n\t"
                     "sub.rn.f32 dz, %3, %23;\n\t"
                     "add.rn.f32 dx, dx, %26;\n\t"
                     "add.rn.f32 dy, dy, %30;\n\t"
                     "add.rn.f32 dz, dz, %31;\n\t"
                     "mul.rn.f32 dx, dx, dx;\n\t"
                     "mul.rn.f32 dy, dy, dy;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q0, dx, %24, q0;\n\t"
                     "@q0 st.shared.b32 [%0], %4;\n\t"
                     "@q0 add.u32 %0, %0, 128;\n\t"
                     "@q0 min.f32 %17, %17, dx;\n\t"
                     "setp.lt.and.f32 qc, dx, %25, q0;\n\t"
                     "@qc add.u32 %18, %18, 1;\n\t"
                     "sub.rn.f32 dx, %5, %21;\n\t"
                     "sub.rn.f32 dy, %6, %22;\n\t"
                     "sub.rn.f32 dz, %7, %23;\n\t"
                     "add.rn.f32 dx, dx, %27;\n\t"
                     "add.rn.f32 dy, dy, %30;\n\t"
                     "add.rn.f32 dz, dz, %31;\n\t"
                     "mul.rn.f32 dx, dx, dx;\n\t"
                     "mul.rn.f32 dy, dy, dy;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q1, dx, %24, q1;\n\t"
                     "@q1 st.shared.b32 [%0], %8;\n\t"
                     "@q1 add.u32 %0, %0, 128;\n\t"
                     "@q1 min.f32 %17, %17, dx;\n\t"
                     "setp.lt.and.f32 qc, dx, %25, q1;\n\t"
                     "@qc add.u32 %18, %18, 1;\n\t"
                     "sub.rn.f32 dx, %9, %21;\n\t"
                     "sub.rn.f32 dy, %10, %22;\n\t"
                     "sub.rn.f32 dz, %11, %23;\n\t"
                     "add.rn.f32 dx, dx, %28;\n\t"
                     "add.rn.f32 dy, dy, %30;\n\t"
                     "add.rn.f32 dz, dz, %31;\n\t"
                     "mul.rn.f32 dx, dx, dx;\n\t"
                     "mul.rn.f32 dy, dy, dy;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q2, dx, %24, q2;\n\t"
                     "@q2 st.shared.b32 [%0], %12;\n\t"
                     "@q2 add.u32 %0, %0, 128;\n\t"
                     "@q2 min.f32 %17, %17, dx;\n\t"
                     "setp.lt.and.f32 qc, dx, %25, q2;\n\t"
                     "@qc add.u32 %18, %18, 1;\n\t"
                     "sub.rn.f32 dx, %13, %21;\n\t"
                     "sub.rn.f32 dy, %14, %22;\n\t"
                     "sub.rn.f32 dz, %15, %23;\n\t"
                     "add.rn.f32 dx, dx, %29;\n\t"
                     "add.rn.f32 dy, dy, %30;\n\t"
                     "add.rn.f32 dz, dz, %31;\n\t"
                     "mul.rn.f32 dx, dx, dx;\n\t"
                     "mul.rn.f32 dy, dy, dy;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q3, dx, %24, q3;\n\t"
                     "@q3 st.shared.b32 [%0], %16;\n\t"
                     "@q3 add.u32 %0, %0, 128;\n\t"
                     "@q3 min.f32 %17, %17, dx;\n\t"
                     "setp.lt.and.f32 qc, dx, %25, q3;\n\t"
                     "@qc add.u32 %18, %18, 1;\n\t"
                     "}"
                     : "+r"(bp), "+f"(c[0].x), "+f"(c[0].y), "+f"(c[0].z), "+f"(c[0].w), "+f"(c[1].x), "+f"(c[1].y), "+f"(c[1].z), "+f"(c[1].w), "+f"(c[2].x), "+f"(c[2].y), "+f"(c[2].z), "+f"(c[2].w), "+f"(c[3].x), "+f"(c[3].y), "+f"(c[3].z), "+f"(c[3].w), "+f"(cl.mn), "+r"(cl.nc)
                     : "r"(act), "r"(addr), "f"(me.x), "f"(me.y), "f"(me.z), "f"(rl2), "f"(close_d2), "f"(sx0), "f"(sx1), "f"(sx2), "f"(sx3), "f"(sy), "f"(sz));
    if (GEN && !CLOSE)
        asm volatile("{\n\t.reg .f32 dx, dy, dz;\n\t.reg .pred q0, q1, q2, q3;\n\t"
                     "setp.gt.s32 q0, %17, 0;\n\t"
                     "setp.gt.s32 q1, %17, 1;\n\t"
                     "setp.gt.s32 q2, %17, 2;\n\t"
                     "setp.gt.s32 q3, %17, 3;\n\t"
                     "@q0 ld.shared.v4.f32 {%1, %2, %3, %4}, [%18];\n\t"
                     "@q1 ld.shared.v4.f32 {%5, %6, %7, %8}, [%18+16];\n\t"
                     "@q2 ld.shared.v4.f32 {%9, %10, %11, %12}, [%18+32];\n\t"
                     "@q3 ld.shared.v4.f32 {%13, %14, %15, %16}, [%18+48];\n\t"
                     "sub.rn.f32 dx, %1, %19;\n\t"
                     "sub.rn.f32 dy, %2, %20;\n\t"
                     "sub.rn.f32 dz, %3, %21;\n\t"
                     "add.rn.f32 dx, dx, %23;\n\t"
                     "add.rn.f32 dy, dy, %27;\n\t"
                     "add.rn.f32 dz, dz, %28;\n\t"
                     "mul.rn.f32 dx, dx, dx;\n\t"
                     "mul.rn.f32 dy, dy, dy;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q0, dx, %22, q0;\n\t"
                     "@q0 st.shared.b32 [%0], %4;\n\t"
                     "@q0 add.u32 %0, %0, 128;\n\t"
                     "sub.rn.f32 dx, %5, %19;\n\t"
                     "sub.rn.f32 dy, %6, %20;\n\t"
                     "sub.rn.f32 dz, %7, %21;\n\t"
                     "add.rn.f32 dx, dx, %24;\n\t"
                     "add.rn.f32 dy, dy, %27;\n\t"
                     "add.rn.f32 dz, dz, %28;\n\t"
                     "mul.rn.f32 dx, dx, dx;\n\t"
                     "mul.rn.f32 dy, dy, dy;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q1, dx, %22, q1;\n\t"
                     "@q1 st.shared.b32 [%0], %8;\n\t"
                     "@q1 add.u32 %0, %0, 128;\n\t"
                     "sub.rn.f32 dx, %9, %19;\n\t"
                     "sub.rn.f32 dy, %10, %20;\n\t"
                     "sub.rn.f32 dz, %11, %21;\n\t"
                     "add.rn.f32 dx, dx, %25;\n\t"
                     "add.rn.f32 dy, dy, %27;\n\t"
                     "add.rn.f32 dz, dz, %28;\n\t"
                     "mul.rn.f32 dx, dx, dx;\n\t"
                     "mul.rn.f32 dy, dy, dy;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q2, dx, %22, q2;\n\t"
                     "@q2 st.shared.b32 [%0], %12;\n\t"
                     "@q2 add.u32 %0, %0, 128;\n\t"
                     "sub.rn.f32 dx, %13, %19;\n\t"
                     "sub.rn.f32 dy, %14, %20;\n\t"
                     "sub.rn.f32 dz, %15, %21;\n\t"
                     "add.rn.f32 dx, dx, %26;\n\t"
                     "add.rn.f32 dy, dy, %27;\n\t"
                     "add.rn.f32 dz, dz, %28;\n\t"
                     "mul.rn.f32 dx, dx, dx;\n\t"
                     "mul.rn.f32 dy, dy, dy;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q3, dx, %22, q3;\n\t"
                     "@q3 st.shared.b32 [%0], %16;\n\t"
                     "@q3 add.u32 %0, %0, 128;\n\t"
                     "}"
                     : "+r"(bp), "+f"(c[0].x), "+f"(c[0].y), "+f"(c[0].z), "+f"(c[0].w), "+f"(c[1].x), "+f"(c[1].y), "+f"(c[1].z), "+f"(c[1].w), "+f"(c[2].x), "+f"(c[2].y), "+f"(c[2].z), "+f"(c[2].w), "+f"(c[3].x), "+f"(c[3].y), "+f"(c[3].z), "+f"(c[3].w)
                     : "r"(act), "r"(addr), "f"(me.x), "f"(me.y), "f"(me.z), "f"(rl2), "f"(sx0), "f"(sx1), "f"(sx2), "f"(sx3), "f"(sy), "f"(sz));
    if (!GEN && CLOSE)
        asm volatile("{\n\t.reg .f32 dx, dy, dz;\n\t.reg .b64 cxy, dxy;\n\t.reg .pred q0, q1, q2, q3, qc;\n\t"
                     "setp.gt.s32 q0, %19, 0;\n\t"
                     "setp.gt.s32 q1, %19, 1;\n\t"
                     "setp.gt.s32 q2, %19, 2;\n\t"
                     "setp.gt.s32 q3, %19, 3;\n\t"
                     "@q0 ld.shared.v4.f32 {%1, %2, %3, %4}, [%20];\n\t"
                     "@q1 ld.shared.v4.f32 {%5, %6, %7, %8}, [%20+16];\n\t"
                     "@q2 ld.shared.v4.f32 {%9, %10, %11, %12}, [%20+32];\n\t"
                     "@q3 ld.shared.v4.f32 {%13, %14, %15, %16}, [%20+48];\n\t"
                     "mov.b64 cxy, {%1, %2};\n\t"
                     "sub.rn.f32x2 dxy, cxy, %26;\n\t"
                     "mul.rn.f32x2 dxy, dxy, dxy;\n\t"
                     "mov.b64 {dx, dy}, dxy;\n\t"
                     "sub.rn.f32 dz, %3, %23;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q0, dx, %24, q0;\n\t"
                     "@q0 st.shared.b32 [%0], %4;\n\t"
                     "@q0 add.u32 %0, %0, 128;\n\t"
                     "@q0 min.f32 %17, %17, dx;\n\t"
                     "setp.lt.and.f32 qc, dx, %25, q0;\n\t"
                     "@qc add.u32 %18, %18, 1;\n\t"
                     "mov.b64 cxy, {%5, %6};\n\t"
                     "sub.rn.f32x2 dxy, cxy, %26;\n\t"
                     "mul.rn.f32x2 dxy, dxy, dxy;\n\t"
                     "mov.b64 {dx, dy}, dxy;\n\t"
                     "sub.rn.f32 dz, %7, %23;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q1, dx, %24, q1;\n\t"
                     "@q1 st.shared.b32 [%0], %8;\n\t"
                     "@q1 add.u32 %0, %0, 128;\n\t"
                     "@q1 min.f32 %17, %17, dx;\n\t"
                     "setp.lt.and.f32 qc, dx, %25, q1;\n\t"
                     "@qc add.u32 %18, %18, 1;\n\t"
                     "mov.b64 cxy, {%9, %10};\n\t"
                     "sub.rn.f32x2 dxy, cxy, %26;\n\t"
                     "mul.rn.f32x2 dxy, dxy, dxy;\n\t"
                     "mov.b64 {dx, dy}, dxy;\n\t"
                     "sub.rn.f32 dz, %11, %23;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q2, dx, %24, q2;\n\t"
                     "@q2 st.shared.b32 [%0], %12;\n\t"
                     "@q2 add.u32 %0, %0, 128;\n\t"
                     "@q2 min.f32 %17, %17, dx;\n\t"
                     "setp.lt.and.f32 qc, dx, %25, q2;\n\t"
                     "@qc add.u32 %18, %18, 1;\n\t"
                     "mov.b64 cxy, {%13, %14};\n\t"
                     "sub.rn.f32x2 dxy, cxy, %26;\n\t"
                     "mul.rn.f32x2 dxy, dxy, dxy;\n\t"
                     "mov.b64 {dx, dy}, dxy;\n\t"
                     "sub.rn.f32 dz, %15, %23;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q3, dx, %24, q3;\n\t"
                     "@q3 st.shared.b32 [%0], %16;\n\t"
                     "@q3 add.u32 %0, %0, 128;\n\t"
                     "@q3 min.f32 %17, %17, dx;\n\t"
                     "setp.lt.and.f32 qc, dx, %25, q3;\n\t"
                     "@qc add.u32 %18, %18, 1;\n\t"
                     "}"
                     : "+r"(bp), "+f"(c[0].x), "+f"(c[0].y), "+f"(c[0].z), "+f"(c[0].w), "+f"(c[1].x), "+f"(c[1].y), "+f"(c[1].z), "+f"(c[1].w), "+f"(c[2].x), "+f"(c[2].y), "+f"(c[2].z), "+f"(c[2].w), "+f"(c[3].x), "+f"(c[3].y), "+f"(c[3].z), "+f"(c[3].w), "+f"(cl.mn), "+r"(cl.nc)
                     : "r"(act), "r"(addr), "f"(me.x), "f"(me.y), "f"(me.z), "f"(rl2), "f"(close_d2),
                       "l"(mxy));
    if (!GEN && !CLOSE)
        asm volatile("{\n\t.reg .f32 dx, dy, dz;\n\t.reg .b64 cxy, dxy;\n\t.reg .pred q0, q1, q2, q3;\n\t"
                     "setp.gt.s32 q0, %17, 0;\n\t"
                     "setp.gt.s32 q1, %17, 1;\n\t"
                     "setp.gt.s32 q2, %17, 2;\n\t"
                     "setp.gt.s32 q3, %17, 3;\n\t"
                     "@q0 ld.shared.v4.f32 {%1, %2, %3, %4}, [%18];\n\t"
                     "@q1 ld.shared.v4.f32 {%5, %6, %7, %8}, [%18+16];\n\t"
                     "@q2 ld.shared.v4.f32 {%9, %10, %11, %12}, [%18+32];\n\t"
                     "@q3 ld.shared.v4.f32 {%13, %14, %15, %16}, [%18+48];\n\t"
                     "mov.b64 cxy, {%1, %2};\n\t"
                     "sub.rn.f32x2 dxy, cxy, %23;\n\t"
                     "mul.rn.f32x2 dxy, dxy, dxy;\n\t"
                     "mov.b64 {dx, dy}, dxy;\n\t"
                     "sub.rn.f32 dz, %3, %21;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q0, dx, %22, q0;\n\t"
                     "@q0 st.shared.b32 [%0], %4;\n\t"
                     "@q0 add.u32 %0, %0, 128;\n\t"
                     "mov.b64 cxy, {%5, %6};\n\t"
                     "sub.rn.f32x2 dxy, cxy, %23;\n\t"
                     "mul.rn.f32x2 dxy, dxy, dxy;\n\t"
                     "mov.b64 {dx, dy}, dxy;\n\t"
                     "sub.rn.f32 dz, %7, %21;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q1, dx, %22, q1;\n\t"
                     "@q1 st.shared.b32 [%0], %8;\n\t"
                     "@q1 add.u32 %0, %0, 128;\n\t"
                     "mov.b64 cxy, {%9, %10};\n\t"
                     "sub.rn.f32x2 dxy, cxy, %23;\n\t"
                     "mul.rn.f32x2 dxy, dxy, dxy;\n\t"
                     "mov.b64 {dx, dy}, dxy;\n\t"
                     "sub.rn.f32 dz, %11, %21;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q2, dx, %22, q2;\n\t"
                     "@q2 st.shared.b32 [%0], %12;\n\t"
                     "@q2 add.u32 %0, %0, 128;\n\t"
                     "mov.b64 cxy, {%13, %14};\n\t"
                     "sub.rn.f32x2 dxy, cxy, %23;\n\t"
                     "mul.rn.f32x2 dxy, dxy, dxy;\n\t"
                     "mov.b64 {dx, dy}, dxy;\n\t"
                     "sub.rn.f32 dz, %15, %21;\n\t"
                     "mul.rn.f32 dz, dz, dz;\n\t"
                     "add.rn.f32 dx, dx, dy;\n\t"
                     "add.rn.f32 dx, dx, dz;\n\t"
                     "setp.lt.and.f32 q3, dx, %22, q3;\n\t"
                     "@q3 st.shared.b32 [%0], %16;\n\t"
                     "@q3 add.u32 %0, %0, 128;\n\t"
                     "}"
                     : "+r"(bp), "+f"(c[0].x), "+f"(c[0].y), "+f"(c[0].z), "+f"(c[0].w), "+f"(c[1].x), "+f"(c[1].y), "+f"(c[1].z), "+f"(c[1].w), "+f"(c[2].x), "+f"(c[2].y), "+f"(c[2].z), "+f"(c[2].w), "+f"(c[3].x), "+f"(c[3].y), "+f"(c[3].z), "+f"(c[3].w)
                     : "r"(act), "r"(addr), "f"(me.x), "f"(me.y), "f"(me.z), "f"(rl2), "l"(mxy));
    (void)close_d2;
    (void)cl;
    (void)sx0;
    (void)sx1;
    (void)sx2;
    (void)sx3;
    (void)sy;
    (void)sz;
}

__device__ __forceinline__ void stg_u4(char *p, uint4 v)
{
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Output state of one lane.  Its hit buffer is interleaved with the other
// lanes of the warp: entry e sits at base + e * kHitStride (base = the
// warp's buffer + 4 * lane), so the per-slot hit stores of a warp always fall
// in 32 different banks.  bp = the next free entry; the first gfl bytes of
// the atom's row are stored; Kb = capacity in bytes.
struct LaneOut {
    uint32_t bp, base, gfl, Kb;
    char *grow;
};

__device__ __forceinline__ uint4 buffer_vector(uint32_t base, uint32_t e)
{
    return make_uint4(lds_u32(base + (e + 0u) * kHitStride), lds_u32(base + (e + 1u) * kHitStride),
                      lds_u32(base + (e + 2u) * kHitStride), lds_u32(base + (e + 3u) * kHitStride));
}

// Store the lane's whole 16-byte vectors (4 entries each) to its row
// (entries past the capacity are only counted) and move the remaining
// entries (at most 3) to the buffer's start; called when some lane of the
// warp holds kFlushAt entries, so at most kBuf - 1 are pending.
__device__ __forceinline__ void flush_check(LaneOut &o)
{
    const uint32_t u = (o.bp - o.base) / kHitStride;
    const uint32_t nv = u & ~3u;
    if (nv != 0u) {
#pragma unroll
        for (uint32_t v = 0; v < (uint32_t)(kBuf / 4 - 1); ++v)
            if (4u * v < nv && o.gfl + 16u * v < o.Kb)
                stg_u4(o.grow + o.gfl + 16u * v, buffer_vector(o.base, 4u * v));
#pragma unroll
        for (uint32_t k = 0; k < 3u; ++k)
            if (nv + k < u) sts_u32(o.base + k * kHitStride, lds_u32(o.base + (nv + k) * kHitStride));
        o.gfl += 4u * nv;
        o.bp -= nv * kHitStride;
    }
}

// Tests this lane's slots lo .. lo+len-1 of one staged row.  The warp runs
// its longest range in groups of 4; a lane past its own range loads nothing,
// so no shared-memory traffic is spent on it.  The lanes are consecutive
// x-sorted home atoms and scan the same row at the same step, so their
// 16-byte loads fall on nearly consecutive slots.  When a lane of the warp
// holds kFlushAt pending hits, the lanes' whole hit vectors are flushed.
// GEN: periodic shifts, per slot in x (slots below ri.x are the low image
// cell, at or above ri.y the high one) and per row in y, z (ri.z, ri.w).
template <bool GEN, bool CLOSE>
__device__ __forceinline__ void scan_range(const float4 *__restrict__ stage, int lo, int len,
                                           const float4 me, float rl2, int4 ri, float Lx,
                                           float4 (&c)[4], float close_d2, CloseAcc &cl,
                                           LaneOut &o)
{
    const int Lmax = __reduce_max_sync(0xffffffffu, len);
    const float sy = __int_as_float(ri.z), sz = __int_as_float(ri.w);
    const uint32_t a0 = smem_u32(stage) + 16u * (uint32_t)lo;
#pragma unroll 1
    for (int j = 0; j < Lmax; j += 4) {
        float sxv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (GEN) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                sxv[u] = lo + j + u < ri.x ? -Lx : (lo + j + u >= ri.y ? Lx : 0.0f);
        }
        scan4<GEN, CLOSE>(a0 + 16u * (uint32_t)j, len - j, c, me, rl2, sxv[0], sxv[1], sxv[2],
                          sxv[3], sy, sz, close_d2, cl, o.bp);
        // flush when some lane holds kFlushAt entries (at most kFlushAt - 1 + 4 pending)
        if (__any_sync(0xffffffffu, o.bp - o.base >= kHitStride * kFlushAt)) flush_check(o);
    }
}

// A range of a tile that touches the periodic faces takes the shifted scan
// only when some lane's range needs it: the row has a y or z shift, or the
// range reaches one of the row's x image cells.  Otherwise every shift is 0
// and the plain scan gives the same bits.
template <bool GEN, bool CLOSE>
__device__ __forceinline__ void scan_checked(const float4 *__restrict__ stage, int lo, int len,
                                             const float4 me, float rl2, int4 ri, float Lx,
                                             float4 (&c)[4], float close_d2,
                                             CloseAcc &cl, LaneOut &o)
{
    if (GEN) {
        const bool need = (ri.z != 0 || ri.w != 0 || lo < ri.x || lo + len > ri.y) && len > 0;
        if (__any_sync(0xffffffffu, need)) {
            scan_range<true, CLOSE>(stage, lo, len, me, rl2, ri, Lx, c, close_d2, cl, o);
            return;
        }
    }
    scan_range<false, CLOSE>(stage, lo, len, me, rl2, ri, Lx, c, close_d2, cl, o);
}

// All 25 rows of one lane's atom: per row, the x half-width h of the window
// from the squared distance (less the margin) between the atom and the row's
// (y, z) cell column, its bins, and from the slot table its slots.  The home
// row is scanned in two ranges around the atom's own slot, so self never
// reaches the predicate.
template <bool GEN, bool CLOSE>
__device__ __forceinline__ void scan_rows(const float4 *__restrict__ stage,
                                          const uint8_t *__restrict__ tabs,
                                          const TileRows &tr, const int4 *rinfo,
                                          const TileParams &P, float rl2, float Lx, int nbins,
                                          const float4 me, bool valid, int slot, int Rh,
                                          float dy_lo, float dy_hi, float dz_lo, float dz_hi,
                                          float mxr, float close_d2, CloseAcc &cl, LaneOut &o)
{
    // candidate registers, carried across groups (an inactive slot's stale
    // value is never taken: its hit predicate is false)
    float4 c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) c[k] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    // rows by dz, then dy: the z distance to a row's column once per dz
#pragma unroll 1
    for (int dz = -2; dz <= 2; ++dz) {
        float pz = dz > 0 ? dz_hi + (float)(dz - 1) * P.side_z
                          : (dz < 0 ? dz_lo + (float)(-dz - 1) * P.side_z : 0.0f);
        pz = fmaxf(pz - P.eps, 0.0f);
        const float pz2 = pz * pz;
#pragma unroll 1
        for (int dy = -2; dy <= 2; ++dy) {
            const int R = Rh + dy + kSY * dz;
            float py = dy > 0 ? dy_hi + (float)(dy - 1) * P.side_y
                              : (dy < 0 ? dy_lo + (float)(-dy - 1) * P.side_y : 0.0f);
            py = fmaxf(py - P.eps, 0.0f);
            const float h2 = P.rl2_margin - (py * py + pz2);
            const bool ok = valid && h2 > 0.0f;
            // approximate root (relative error ~1e-6): the margin absorbs it
            const float hc = fmaxf(h2, 1e-20f);
            const float hw = hc * rsqrtf(hc) + P.eps;
            const int b0 = min(max(__float2int_rd((mxr - hw) * P.inv_bin), 0), nbins - 1);
            const int b1 = min(max(__float2int_rd((mxr + hw) * P.inv_bin) + 1, 0), nbins);
            // first staged slot at or above a bin: start of its cell + the cell's
            // table entry; past the last bin, the row end
            const uint8_t *tb = tabs + R * kRowTab;
            const int off = tr.off[R];
            const int lo = off + tr.cell[R][b0 >> 4] + tb[b0];
            const int hi = off + (b1 < nbins ? tr.cell[R][b1 >> 4] + tb[b1] : tr.len[R]);
            const int4 ri = GEN ? rinfo[R] : make_int4(0, 0, 0, 0);
            if (dy == 0 && dz == 0) {   // the home row
                const int e1 = min(hi, slot);
                scan_checked<GEN, CLOSE>(stage, lo, ok && e1 > lo ? e1 - lo : 0, me, rl2, ri, Lx, c,
                                         close_d2, cl, o);
                const int s1 = max(lo, slot + 1);
                scan_checked<GEN, CLOSE>(stage, s1, ok && hi > s1 ? hi - s1 : 0, me, rl2, ri, Lx, c,
                                         close_d2, cl, o);
            } else {
                scan_checked<GEN, CLOSE>(stage, lo, ok && hi > lo ? hi - lo : 0, me, rl2, ri, Lx, c,
                                         close_d2, cl, o);
            }
        }
    }
    flush_check(o);
}

// Staged row R of a tile: conceptual cells cx0-1 .. cx0+Gx of the (y, z)
// column two cells below .. above the home block, as up to three
// contiguous pieces of the cell-ordered array (the low periodic image cell
// nx-1, the in-box cells, the high periodic image cell 0).
struct RowSrc {
    int need;
    int has_lo, has_hi;         // image cells present (cx0 == 0; cx0 + Gx == nx)
    int lo_src, lo_cnt;
    int mid_src, mid_cnt;
    int mid_cells;
    int hi_src, hi_cnt;
    int64_t rowc;               // cell index of x = 0 in this (y, z) column
    int first;                  // first in-box cell
    int len, lend, rbeg;        // slots; [0, lend) low image, [rbeg, len) high image
    float sy, sz;               // periodic shifts of the row
};

__device__ __forceinline__ void describe_row(const CellGrid &g, const int32_t *__restrict__ cs,
                                             int R, int cx0, int cy0, int cz0, int Gx, int Gy,
                                             int Gz, RowSrc &rs, int *cell)
{
    const int ry = R % kSY, rz = R / kSY;
    rs.need = R < kSRows && ry < Gy + 4 && rz < Gz + 4;
    rs.has_lo = rs.has_hi = 0;
    rs.lo_cnt = rs.mid_cnt = rs.hi_cnt = 0;
    rs.lo_src = rs.mid_src = rs.hi_src = 0;
    rs.mid_cells = 0;
    rs.rowc = 0;
    rs.first = 0;
    rs.len = rs.lend = rs.rbeg = 0;
    rs.sy = rs.sz = 0.0f;
    if (!rs.need) return;
    int y = cy0 - 2 + ry, z = cz0 - 2 + rz;
    if (y < 0) { y += g.ny; rs.sy = -g.Ly; } else if (y >= g.ny) { y -= g.ny; rs.sy = g.Ly; }
    if (z < 0) { z += g.nz; rs.sz = -g.Lz; } else if (z >= g.nz) { z -= g.nz; rs.sz = g.Lz; }
    const int64_t rowc = ((int64_t)z * g.ny + y) * g.nx;
    rs.rowc = rowc;
    int k = 0, len = 0;
    if (cx0 == 0) {   // conceptual cell -1 is cell nx-1
        const int a = cs[rowc + g.nx - 1], b = cs[rowc + g.nx];
        rs.has_lo = 1;
        rs.lo_src = a;
        rs.lo_cnt = b - a;
        cell[k++] = 0;
        len = b - a;
    }
    rs.lend = len;
    const int first = cx0 == 0 ? 0 : cx0 - 1;
    const int last = cx0 + Gx <= g.nx - 1 ? cx0 + Gx : g.nx - 1;
    const int a = cs[rowc + first];
    for (int cc = first; cc <= last; ++cc) cell[k++] = len + (cs[rowc + cc] - a);
    const int b = cs[rowc + last + 1];
    rs.first = first;
    rs.mid_src = a;
    rs.mid_cnt = b - a;
    rs.mid_cells = last - first + 1;
    len += b - a;
    rs.rbeg = len;
    if (cx0 + Gx == g.nx) {   // conceptual cell nx is cell 0
        const int a2 = cs[rowc], b2 = cs[rowc + 1];
        rs.has_hi = 1;
        rs.hi_src = a2;
        rs.hi_cnt = b2 - a2;
        cell[k++] = len;
        len += b2 - a2;
    }
    cell[k] = len;   // k == Gx + 2
    rs.len = len;
}

// Issues the copies of one staged row: its atoms to stage slot `off`, the x
// tables of its Gx + 2 conceptual cells to `tdst`; all complete on `bar`.
__device__ __forceinline__ void copy_row(const RowSrc &rs, const TileParams &P, const CellGrid &g,
                                         uint32_t stage_base, int off, uint32_t tdst, uint64_t *bar)
{
    if (!rs.need) return;
    uint32_t dst = stage_base + 16u * (uint32_t)off;
    if (rs.lo_cnt > 0) bulk_g2s(dst, P.cell_pos + rs.lo_src, 16u * (uint32_t)rs.lo_cnt, bar);
    dst += 16u * (uint32_t)rs.lo_cnt;
    if (rs.mid_cnt > 0) bulk_g2s(dst, P.cell_pos + rs.mid_src, 16u * (uint32_t)rs.mid_cnt, bar);
    dst += 16u * (uint32_t)rs.mid_cnt;
    if (rs.hi_cnt > 0) bulk_g2s(dst, P.cell_pos + rs.hi_src, 16u * (uint32_t)rs.hi_cnt, bar);
    const uint32_t tb = (uint32_t)kBinsPerCell;
    if (rs.has_lo) {
        bulk_g2s(tdst, P.cell_tab + (rs.rowc + g.nx - 1) * kBinsPerCell, tb, bar);
        tdst += tb;
    }
    bulk_g2s(tdst, P.cell_tab + (rs.rowc + rs.first) * kBinsPerCell, tb * (uint32_t)rs.mid_cells,
             bar);
    tdst += tb * (uint32_t)rs.mid_cells;
    if (rs.has_hi) bulk_g2s(tdst, P.cell_tab + rs.rowc * kBinsPerCell, tb, bar);
}

// Bytes copy_row moves for a row.
__device__ __forceinline__ uint32_t row_bytes(const RowSrc &rs)
{
    if (!rs.need) return 0u;
    return 16u * (uint32_t)rs.len +
           (uint32_t)kBinsPerCell * (uint32_t)(rs.has_lo + rs.mid_cells + rs.has_hi);
}

// Describes tile `t` (rows, their offsets in the stage, home rows) into `tr`
// and `m` with the 32 lanes of one warp.  Returns, in every lane, the bytes
// the row copies will carry; tr.fallback is set when the rows do not fit a
// stage of P.stage_max slots (or the cells are not x-sorted).  ra, rb: the
// lane's two rows (lane and lane + 32).
__device__ __forceinline__ uint32_t describe_tile(int t, const CellGrid &g, const TileParams &P,
                                                  TileRows &tr, int4 *rinfo, TileMeta &m,
                                                  RowSrc &ra, RowSrc &rb)
{
    const int lane = threadIdx.x & 31;
    const int tx = t % P.tiles_x;
    t /= P.tiles_x;
    const int ty = t % P.tiles_y, tz = t / P.tiles_y;
    const int cx0 = tx * kTX, cy0 = ty * kTY, cz0 = tz * kTZ;
    const int Gx = min(kTX, g.nx - cx0), Gy = min(kTY, g.ny - cy0), Gz = min(kTZ, g.nz - cz0);
    int cell_scratch[kSCells + 1];
    describe_row(g, P.cell_start, lane, cx0, cy0, cz0, Gx, Gy, Gz, ra, tr.cell[lane]);
    describe_row(g, P.cell_start, lane + 32, cx0, cy0, cz0, Gx, Gy, Gz, rb,
                 lane + 32 < kSRows ? tr.cell[lane + 32] : cell_scratch);
    // offsets: rows back to back in staged order
    const int va = ra.len, vb = lane + 32 < kSRows ? rb.len : 0;
    int xa = va, xb = vb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, xa, o);
        const int yb = __shfl_up_sync(0xffffffffu, xb, o);
        if (lane >= o) {
            xa += ya;
            xb += yb;
        }
    }
    const int suma = __shfl_sync(0xffffffffu, xa, 31);
    const int sumb = __shfl_sync(0xffffffffu, xb, 31);
    const int offa = xa - va;
    const int offb = suma + xb - vb;
    const int total = suma + sumb;
    tr.off[lane] = offa;
    tr.len[lane] = ra.len;
    rinfo[lane] = make_int4(offa + ra.lend, offa + ra.rbeg, __float_as_int(ra.sy),
                            __float_as_int(ra.sz));
    if (lane + 32 < kSRows) {
        tr.off[lane + 32] = offb;
        tr.len[lane + 32] = rb.len;
        rinfo[lane + 32] = make_int4(offb + rb.lend, offb + rb.rbeg, __float_as_int(rb.sy),
                                     __float_as_int(rb.sz));
    }
    // home rows h = hy + kTY hz are staged rows (hy + 2) + kSY (hz + 2)
    __syncwarp();
    int hcnt = 0;
    if (lane < kHome) {
        const int hy = lane % kTY, hz = lane / kTY;
        const int R = (hy + 2) + kSY * (hz + 2);
        tr.home_begin[lane] = tr.off[R] + tr.cell[R][1];
        hcnt = hy < Gy && hz < Gz ? tr.cell[R][Gx + 1] - tr.cell[R][1] : 0;
    }
    int hx = hcnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, hx, o);
        if (lane >= o) hx += y;
    }
    if (lane < kHome) tr.home_pref[lane] = hx - hcnt;
    if (lane == kHome - 1) tr.home_pref[kHome] = hx;
    const uint32_t bytes = __reduce_add_sync(0xffffffffu, row_bytes(ra) + row_bytes(rb));
    if (lane == 0) {
        tr.total = total;
        tr.fallback = (total > P.stage_max || *P.unsorted != 0u) ? 1 : 0;
        m.cx0 = cx0;
        m.cy0 = cy0;
        m.cz0 = cz0;
        m.Gx = Gx;
        m.Gy = Gy;
        m.Gz = Gz;
        m.general = cx0 == 0 || cx0 + Gx == g.nx || cy0 < 2 || cy0 + Gy + 2 > g.ny || cz0 < 2 ||
                    cz0 + Gz + 2 > g.nz;
    }
    __syncwarp();
    return bytes;
}

// Chunk c (home atoms 32c .. 32c + 31 in home-row order) of a staged tile:
// each lane searches the 25 rows of its atom and writes the atom's row and
// count.  hb: the warp's interleaved hit buffer; negs_addr: a shared block of
// -1.
template <bool CLOSE>
__device__ __forceinline__ void search_chunk(int c, const float4 *__restrict__ stage,
                                             const uint8_t *__restrict__ tabs,
                                             const TileRows &tr, const int4 *rinfo,
                                             const TileMeta &m, const CellGrid &g,
                                             const TileParams &P, uint32_t hb,
                                             uint32_t negs_addr, CloseAcc &cl)
{
    const int lane = threadIdx.x & 31;
    const int nbins = (m.Gx + 2) * kBinsPerCell;
    const float X0 = (float)(m.cx0 - 1) * P.side_x;   // low x face of conceptual cell 0
    const float rl2 = g.rl2;
    const int nhome = tr.home_pref[kHome];
    const int a = c * 32 + lane;
    int h = 0;
    while (h < kHome - 1 && a >= tr.home_pref[h + 1]) ++h;
    const int slot = tr.home_begin[h] + (a - tr.home_pref[h]);
    const float qn = __int_as_float(0x7fc00000);
    float4 me = a < nhome ? stage[slot] : make_float4(qn, qn, qn, qn);
    // a lane has a row to build when its atom exists and is below n_rows
    const bool valid = a < nhome && __float_as_int(me.w) < g.n_rows;
    if (!valid) me = make_float4(qn, qn, qn, qn);
    const int hy = h % kTY, hz = h / kTY;
    const float ylo = (float)(m.cy0 + hy) * P.side_y, yhi = (float)(m.cy0 + hy + 1) * P.side_y;
    const float zlo = (float)(m.cz0 + hz) * P.side_z, zhi = (float)(m.cz0 + hz + 1) * P.side_z;
    const float dy_lo = me.y - ylo, dy_hi = yhi - me.y;
    const float dz_lo = me.z - zlo, dz_hi = zhi - me.z;

    LaneOut o;
    o.base = hb + 4u * (uint32_t)lane;
    o.bp = o.base;
    o.gfl = 0u;
    o.Kb = 4u * (uint32_t)P.K;
    const int myid = __float_as_int(me.w);
    o.grow = reinterpret_cast<char *>(P.nbr + (int64_t)(valid ? myid : 0) * P.K);
    const float mxr = me.x - X0;
    const int Rh = (hy + 2) + kSY * (hz + 2);
    if (m.general)
        scan_rows<true, CLOSE>(stage, tabs, tr, rinfo, P, rl2, g.Lx, nbins, me, valid, slot, Rh,
                               dy_lo, dy_hi, dz_lo, dz_hi, mxr, P.close_d2, cl, o);
    else
        scan_rows<false, CLOSE>(stage, tabs, tr, rinfo, P, rl2, g.Lx, nbins, me, valid, slot, Rh,
                                dy_lo, dy_hi, dz_lo, dz_hi, mxr, P.close_d2, cl, o);

    // ---- finish the row (the scan ends with a flush: at most 3 entries
    //      pending): the partial vector completed with -1, then -1 from the
    //      shared block up to the capacity
    if (valid) {
        const uint32_t u = (o.bp - o.base) / kHitStride;
        uint32_t pf = o.gfl;
        if (u != 0u) {
            uint4 v;
            v.x = lds_u32(o.base);
            v.y = u > 1u ? lds_u32(o.base + kHitStride) : 0xffffffffu;
            v.z = u > 2u ? lds_u32(o.base + 2u * kHitStride) : 0xffffffffu;
            v.w = 0xffffffffu;
            if (o.gfl < o.Kb) stg_u4(o.grow + o.gfl, v);
            pf += 16u;
        }
        if (pf < o.Kb) bulk_s2g(o.grow + pf, negs_addr, o.Kb - pf);
        bulk_commit();
        const int cnt = (int)((o.gfl >> 2) + u);
        P.counts[myid] = cnt;
        if (cnt > P.K) atomicOr(P.flags, kFlagOverflow);
    }
}

// Shared state of the persistent launch (static part).
struct PipeShared {
    uint64_t full[kPipeStages];      // a stage's rows have landed (tx-count phase)
    uint64_t empty[kPipeStages];     // every chunk of a stage's tile is done
    uint32_t queue[kQueue];          // chunks, in the order the staging warp filled them
    uint32_t q_tail;                 // entries published
    uint32_t q_head;                 // entries taken
    TileRows tr[kPipeMeta];
    int4 rinfo[kPipeMeta][kSRows];   // x image bounds (slots) and y, z shifts per row
    TileMeta meta[kPipeMeta];
};

// Persistent pair search, one CTA per SM.  Warp 0 stages: it takes tiles from
// a global counter, describes each (ahead of time, into one of kPipeMeta
// description slots), waits for one of kPipeStages shared-memory stages to be
// free, issues the rows' cp.async.bulk copies against the stage's `full`
// barrier, and publishes the tile's chunks (32 home atoms each) on a queue.
// Warps 1..kPipeConsumers each take the next chunk from the queue, wait for
// its stage's rows, search it, and arrive on the stage's `empty` barrier; the
// staging warp's own arrival at fill time counts kEmptyCount - chunks, so the
// stage frees when its last chunk is done.  No warp waits for another at a
// CTA barrier: a warp that finishes a chunk moves to the next one, in this
// tile or the next, while warp 0 stages ahead.  A tile whose rows exceed a
// stage is listed for k_pairs_listed.  Every wait is bounded: one that gives
// up records kFlagTimeout and the warp leaves (the staging warp first
// publishes an end entry per searching warp).
template <bool CLOSE>
__global__ void __launch_bounds__(kPipeThreads, 1)
k_pairs_pipe(const CellGrid g, const TileParams P)
{
    // cell starts may not be monotonic; one decision for the whole CTA
    if (__syncthreads_or(timed_out(P.flags))) return;
    extern __shared__ __align__(16) unsigned char pipe_smem[];
    __shared__ PipeShared sh;
    const int S = P.stages;
    float4 *stages = reinterpret_cast<float4 *>(pipe_smem);                       // [S][stage_max]
    uint8_t *tabs = pipe_smem + sizeof(float4) * (size_t)S * P.stage_max;          // [S][kSRows][kRowTab]
    int32_t *hits = reinterpret_cast<int32_t *>(tabs + S * kSRows * kRowTab);
    int32_t *negs = hits + kPipeConsumers * 32 * kBuf;                           // P.K entries of -1

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < P.K; e += blockDim.x) negs[e] = -1;
    fence_proxy_async_smem();   // -1 block is read by bulk copies of any thread
    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(&sh.full[st], 1);
            mbar_init(&sh.empty[st], kEmptyCount);
        }
        sh.q_tail = 0u;
        sh.q_head = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------ staging warp
        uint32_t fpar = 0u, used = 0u;   // per stage: parity of its next fill, filled before
        uint32_t tail = 0u;
        int k = 0, mi = 0;               // fills issued; description slot of the next fill
        bool gave_up = false;
        // the next tile: in order, or the next entry of the list; -1 when done
        auto next_tile = [&]() {
            int tt = -1;
            if (lane == 0) {
                const uint32_t e = atomicAdd(P.tile_ctr, 1u);
                if (P.tile_list)
                    tt = e < ld_volatile_u32(P.tile_list_count) ? (int)P.tile_list[e] : -1;
                else
                    tt = e < (uint32_t)P.ntiles ? (int)e : -1;
            }
            return __shfl_sync(0xffffffffu, tt, 0);
        };
        int t = next_tile();
        while (t >= 0) {
            RowSrc ra, rb;
            const uint32_t bytes = describe_tile(t, g, P, sh.tr[mi], sh.rinfo[mi], sh.meta[mi], ra, rb);
            const int tile = t;
            t = next_tile();
            const int nhome = sh.tr[mi].home_pref[kHome];
            if (sh.tr[mi].fallback) {
                if (lane == 0) P.fb_list[atomicAdd(P.fb_count, 1u)] = (uint32_t)tile;   // out list
                continue;
            }
            if (nhome == 0) continue;
            const int st = k % S;
            if (used >> st & 1u) {   // the stage's previous tile must be searched out
                bool done = false;
                for (uint32_t spins = 0; spins < 4096u && !done; ++spins)
                    done = mbar_try_wait(&sh.empty[st], ((fpar >> st) & 1u) ^ 1u);
                if (!done) {
                    gave_up = true;
                    break;
                }
            }
            const uint32_t stage_base = smem_u32(stages + (size_t)st * P.stage_max);
            const uint32_t tab_base = smem_u32(tabs + st * kSRows * kRowTab);
            if (lane == 0) mbar_arrive_expect_tx(&sh.full[st], bytes);
            __syncwarp();
            copy_row(ra, P, g, stage_base, sh.tr[mi].off[lane], tab_base + (uint32_t)(lane * kRowTab),
                     &sh.full[st]);
            if (lane + 32 < kSRows)
                copy_row(rb, P, g, stage_base, sh.tr[mi].off[lane + 32],
                         tab_base + (uint32_t)((lane + 32) * kRowTab), &sh.full[st]);
            const uint32_t nchunks = (uint32_t)(nhome + 31) >> 5;
            if (lane == 0) {
                mbar_arrive_cnt(&sh.empty[st], kEmptyCount - nchunks);
                const uint32_t head = (uint32_t)st | ((uint32_t)mi << 2) |
                                      (((fpar >> st) & 1u) << 5);
                for (uint32_t c = 0; c < nchunks; ++c)
                    sh.queue[(tail + c) % kQueue] = head | (c << 8);
                __threadfence_block();
                st_volatile_u32(&sh.q_tail, tail + nchunks);
            }
            tail += nchunks;
            fpar ^= 1u << st;
            used |= 1u << st;
            ++k;
            mi = (mi + 1) % kPipeMeta;
        }
        if (lane == 0) {
            if (gave_up) atomicOr(P.flags, kFlagTimeout);
            for (uint32_t c = 0; c < (uint32_t)kPipeConsumers; ++c)
                sh.queue[(tail + c) % kQueue] = kQueueEnd;
            __threadfence_block();
            st_volatile_u32(&sh.q_tail, tail + (uint32_t)kPipeConsumers);
        }
        return;
    }

    // --------------------------------------------------------- searching warps
    CloseAcc cl{__int_as_float(0x7f800000), 0u};
    const uint32_t hb = smem_u32(hits) + (uint32_t)((warp - 1) * 32 * kBuf * 4);   // the warp's buffer
    const uint32_t negs_addr = smem_u32(negs);
    for (;;) {
        uint32_t e = kQueueEnd;
        if (lane == 0) {
            const uint32_t tk = atomicAdd(&sh.q_head, 1u);
            uint32_t spins = 0u;
            bool ok = true;
            while (ld_volatile_u32(&sh.q_tail) <= tk) {
                if (++spins >= kSpinLimit) {
                    ok = false;
                    break;
                }
                __nanosleep(128);
            }
            if (ok) {
                __threadfence_block();
                e = ld_volatile_u32(&sh.queue[tk % kQueue]);
            } else {
                atomicOr(P.flags, kFlagTimeout);
            }
        }
        e = __shfl_sync(0xffffffffu, e, 0);
        if (e == kQueueEnd) break;
        const int st = (int)(e & 3u), mslot = (int)((e >> 2) & 7u);
        const uint32_t par = (e >> 5) & 1u;
        const int c = (int)(e >> 8);
        bool done = false;
        for (uint32_t spins = 0; spins < 4096u && !done; ++spins)   // ~4 s
            done = mbar_try_wait(&sh.full[st], par);
        if (!__all_sync(0xffffffffu, done)) {
            // the stage's copies carry exactly the announced bytes, so the
            // phase completes when they land: record the timeout, wait once
            // more (bounded) so no copy is left writing into shared memory,
            // and leave
            if (lane == 0) atomicOr(P.flags, kFlagTimeout);
            for (uint32_t spins = 0; spins < 4096u && !done; ++spins)
                done = mbar_try_wait(&sh.full[st], par);
            break;
        }
        search_chunk<CLOSE>(c, stages + (size_t)st * P.stage_max, tabs + st * kSRows * kRowTab,
                            sh.tr[mslot], sh.rinfo[mslot], sh.meta[mslot], g, P, hb, negs_addr, cl);
        __syncwarp();
        if (lane == 0) mbar_arrive_cnt(&sh.empty[st], 1u);
    }
    if (CLOSE) close_publish(cl, P.min_bits, P.n_close);
    bulk_wait_read<0>();   // the -1 block stays readable until the copies are done
}

// The listed tiles (rows beyond the persistent launch's stages): persistent
// CTAs over the list, up to kListedCtas per SM with larger stages, one tile
// at a time.  A tile that still does not fit is searched per atom from
// global memory.
template <bool CLOSE>
__global__ void __launch_bounds__(kListedWarps * 32, 1)
k_pairs_listed(const CellGrid g, const TileParams P)
{
    // cell starts may not be monotonic; one decision for the whole CTA
    if (__syncthreads_or(timed_out(P.flags))) return;
    extern __shared__ __align__(16) unsigned char tile_smem[];
    float4 *stage = reinterpret_cast<float4 *>(tile_smem);
    uint8_t *tabs = tile_smem + sizeof(float4) * P.stage_max;                   // [kSRows][kRowTab]
    int32_t *hits = reinterpret_cast<int32_t *>(tabs + kSRows * kRowTab);       // [W][kBuf][32]
    int32_t *negs = hits + kListedWarps * 32 * kBuf;                           // P.K entries of -1
    __shared__ TileRows tr;
    __shared__ int4 rinfo[kSRows];
    __shared__ TileMeta meta;
    __shared__ __align__(8) uint64_t bar;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < P.K; e += blockDim.x) negs[e] = -1;
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    uint32_t phase = 0;   // parity of the mbarrier phase the next staging completes
    CloseAcc cl{__int_as_float(0x7f800000), 0u};
    const uint32_t hb = smem_u32(hits) + (uint32_t)(warp * 32 * kBuf * 4);   // the warp's buffer
    const uint32_t negs_addr = smem_u32(negs);

    for (uint32_t e = blockIdx.x; e < *P.fb_count; e += gridDim.x) {
        const int t = (int)P.fb_list[e];
        if (warp == 0) {
            RowSrc ra, rb;
            const uint32_t bytes = describe_tile(t, g, P, tr, rinfo, meta, ra, rb);
            if (!tr.fallback) {
                if (lane == 0) mbar_arrive_expect_tx(&bar, bytes);
                __syncwarp();
                const uint32_t stage_base = smem_u32(stage);
                copy_row(ra, P, g, stage_base, tr.off[lane], smem_u32(tabs) + (uint32_t)(lane * kRowTab),
                         &bar);
                if (lane + 32 < kSRows)
                    copy_row(rb, P, g, stage_base, tr.off[lane + 32],
                             smem_u32(tabs) + (uint32_t)((lane + 32) * kRowTab), &bar);
            }
        }
        __syncthreads();
        if (tr.fallback) {   // per atom, straight from global memory
            for (int hz = 0; hz < meta.Gz; ++hz)
                for (int hy = 0; hy < meta.Gy; ++hy) {
                    const int64_t rowc = ((int64_t)(meta.cz0 + hz) * g.ny + (meta.cy0 + hy)) * g.nx;
                    const int32_t k0 = P.cell_start[rowc + meta.cx0];
                    const int32_t k1 = P.cell_start[rowc + meta.cx0 + meta.Gx];
                    for (int32_t k = k0 + threadIdx.x; k < k1; k += blockDim.x)
                        pair_row_per_atom<false, CLOSE>(k, P.cell_pos, P.cell_start, P.atom_cell,
                                                        g, P.K, P.nbr, P.counts, P.flags,
                                                        P.close_d2, cl);
                }
            __syncthreads();
            continue;
        }
        {
            bool done = false;
            for (uint32_t spins = 0; spins < 4096u && !done; ++spins)   // ~4 s
                done = mbar_try_wait(&bar, phase);
            if (__syncthreads_or(!done)) {
                // see k_pairs_pipe: record, wait once more (bounded), leave
                if (threadIdx.x == 0) atomicOr(P.flags, kFlagTimeout);
                for (uint32_t spins = 0; spins < 4096u && !done; ++spins)
                    done = mbar_try_wait(&bar, phase);
                break;
            }
            phase ^= 1u;
        }
        const int nhome = tr.home_pref[kHome];
        for (int c = warp; c * 32 < nhome; c += kListedWarps)
            search_chunk<CLOSE>(c, stage, tabs, tr, rinfo, meta, g, P, hb, negs_addr, cl);
        __syncthreads();   // the tile's shared data is reused by the next one
    }
    if (CLOSE) close_publish(cl, P.min_bits, P.n_close);
    bulk_wait_read<0>();   // the -1 block stays readable until the copies are done
}

constexpr int kSlotLimit = 65000;   // slot-table entries are 16 bits

// Dynamic shared memory of the persistent launch with S stages of
// stage_max slots: the stages, their row tables, the hit buffers, the -1
// block.
size_t pipe_smem_bytes(int K, int S, int stage_max)
{
    return (size_t)S * ((size_t)stage_max * sizeof(float4) + (size_t)kSRows * kRowTab) +
           (size_t)kPipeConsumers * 32 * kBuf * sizeof(int32_t) + (size_t)K * sizeof(int32_t);
}

// Stage slots of the persistent launch with S stages, from what shared
// memory leaves after its static part; also bounded by the chunk queue
// (every chunk of S tiles plus the end entries) and the 16-bit slot tables.
// 0 when too small to be worth a launch.
int pipe_stage_slots(int optin, int static_smem, int K, int S)
{
    const long budget = (long)optin - static_smem - (long)pipe_smem_bytes(K, S, 0);
    long fit = budget > 0 ? budget / ((long)sizeof(float4) * S) : 0;
    const long qcap = (long)(kQueue - kPipeConsumers - 8) / S * 32;
    if (fit > qcap) fit = qcap;
    if (fit > kSlotLimit) fit = kSlotLimit;
    return fit >= 256 ? (int)(fit & ~31L) : 0;
}

size_t listed_fixed_smem(int K)
{
    return (size_t)kSRows * kRowTab + (size_t)kListedWarps * 32 * kBuf * sizeof(int32_t) +
           (size_t)K * sizeof(int32_t);
}

template <class Kernel>
cudaError_t allow_smem(Kernel kernel, int optin)
{
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                optin - (int)fa.sharedSizeBytes);
}

}  // namespace

cudaError_t pairs_set_attributes()
{
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    if ((e = allow_smem(k_pairs_pipe<false>, optin)) != cudaSuccess) return e;
    if ((e = allow_smem(k_pairs_pipe<true>, optin)) != cudaSuccess) return e;
    if ((e = allow_smem(k_pairs_listed<false>, optin)) != cudaSuccess) return e;
    return allow_smem(k_pairs_listed<true>, optin);
}

namespace {

template <bool CLOSE>
cudaError_t launch_pairs_t(nl_ctx *ctx, int64_t n, const CellGrid &g, int32_t capacity,
                           int32_t *nbr, int32_t *counts, cudaStream_t s, int *used_fast,
                           const CloseOut *close)
{
    *used_fast = 0;
    if (n <= 0) return cudaSuccess;
    // Persistent staged kernel: column grid and rows of whole 16-byte
    // vectors.  Its kPipeStages stages share what is left of the SM's
    // shared memory; a stage should hold a typical tile (kSRows rows x
    // (kTX + 2) cells at the mean cell occupancy) with 10 % to spare.  Denser
    // tiles are listed for a second launch with larger stages.
    int stage3 = 0, stage2 = 0;   // stage slots with three and with two stages per CTA
    int need = 0, per_sm = 0, reserved = 0, optin = 0;
    if (g.wy == 2 && g.wz == 2 && !g.literal && capacity % 4 == 0 &&
        (reinterpret_cast<uintptr_t>(nbr) & 15u) == 0 && n < (int64_t(1) << 31)) {
        int dev = 0;
        NL_CUDA_TRY(cudaGetDevice(&dev));
        NL_CUDA_TRY(cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev));
        NL_CUDA_TRY(cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev));
        NL_CUDA_TRY(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
        cudaFuncAttributes fa;
        NL_CUDA_TRY(cudaFuncGetAttributes(&fa, k_pairs_pipe<CLOSE>));
        const double per_cell = (double)n / (double)g.ncell;
        const int want = (int)(1.1 * per_cell * kSRows * kSCells) + 32;
        need = want > kStageMin ? want : kStageMin;
        stage3 = pipe_stage_slots(optin, (int)fa.sharedSizeBytes, capacity, 3);
        stage2 = pipe_stage_slots(optin, (int)fa.sharedSizeBytes, capacity, 2);
    }
    if (stage2 > 0) {
        TileParams P;
        P.close_d2 = CLOSE ? close->close_d2 : 0.0f;
        P.min_bits = CLOSE ? reinterpret_cast<uint32_t *>(close->min_d2) : nullptr;
        P.n_close = CLOSE ? reinterpret_cast<unsigned long long *>(close->n_close) : nullptr;
        P.cell_pos = ctx->cell_pos;
        P.atom_cell = ctx->atom_cell;
        P.cell_start = ctx->cell_start;
        P.cell_tab = ctx->cell_tab;
        P.nbr = nbr;
        P.counts = counts;
        P.flags = ctx->flags;
        P.unsorted = ctx->unsorted;
        P.tiles_x = (g.nx + kTX - 1) / kTX;
        P.tiles_y = (g.ny + kTY - 1) / kTY;
        const int tiles_z = (g.nz + kTZ - 1) / kTZ;
        P.ntiles = P.tiles_x * P.tiles_y * tiles_z;
        P.K = capacity;
        P.side_x = g.Lx / (float)g.nx;
        P.side_y = g.Ly / (float)g.ny;
        P.side_z = g.Lz / (float)g.nz;
        P.inv_bin = (float)kBinsPerCell / P.side_x;
        const float rl = sqrtf(g.rl2);
        const float Lmax = fmaxf(g.Lx, fmaxf(g.Ly, g.Lz));
        P.eps = 1e-3f * rl + 4e-6f * Lmax;
        P.rl2_margin = g.rl2 * (1.0f + 1e-4f);
        // fb_count, tile_ctr, fb_count2, tile_ctr2
        NL_CUDA_TRY(cudaMemsetAsync(ctx->fb_count, 0, 4 * sizeof(uint32_t), s));
        // Three stages when a typical tile fits them: every tile is taken in
        // order and a tile beyond the stage is listed; a second persistent
        // launch with two larger stages takes the listed tiles.  Systems
        // denser than that start with the two-stage launch over every tile.
        // Tiles beyond even those stages go to k_pairs_listed.
        TileParams P2 = P;
        P2.stages = 2;
        P2.stage_max = stage2;
        P2.tile_ctr = ctx->tile_ctr2;
        P2.fb_list = ctx->fb_list2;
        P2.fb_count = ctx->fb_count2;
        if (stage3 > 0 && (double)need <= 1.1 * stage3) {
            TileParams P3 = P;
            P3.stages = 3;
            P3.stage_max = stage3;
            P3.tile_ctr = ctx->tile_ctr;
            P3.tile_list = nullptr;
            P3.tile_list_count = nullptr;
            P3.fb_list = ctx->fb_list;
            P3.fb_count = ctx->fb_count;
            {
                ProfScope ps(ctx, PH_PAIRS, s);
                k_pairs_pipe<CLOSE><<<(unsigned)ctx->sm_count, kPipeThreads,
                                      pipe_smem_bytes(capacity, 3, stage3), s>>>(g, P3);
                NL_CUDA_TRY(cudaGetLastError());
            }
            P2.tile_list = ctx->fb_list;
            P2.tile_list_count = ctx->fb_count;
            ProfScope ps(ctx, PH_PAIRS_LISTED, s);
            k_pairs_pipe<CLOSE><<<(unsigned)ctx->sm_count, kPipeThreads,
                                  pipe_smem_bytes(capacity, 2, stage2), s>>>(g, P2);
            NL_CUDA_TRY(cudaGetLastError());
        } else {
            P2.tile_list = nullptr;
            P2.tile_list_count = nullptr;
            ProfScope ps(ctx, PH_PAIRS, s);
            k_pairs_pipe<CLOSE><<<(unsigned)ctx->sm_count, kPipeThreads,
                                  pipe_smem_bytes(capacity, 2, stage2), s>>>(g, P2);
            NL_CUDA_TRY(cudaGetLastError());
        }
        *used_fast = 1;
        // tiles beyond the two-stage launch: as many CTAs per SM (up to
        // kListedCtas) as still give each a stage of twice a typical tile;
        // one CTA with the largest stage when none does.  A tile beyond its
        // stage is searched per atom from global memory in the same kernel.
        cudaFuncAttributes fl;
        NL_CUDA_TRY(cudaFuncGetAttributes(&fl, k_pairs_listed<CLOSE>));
        const long lfixed = (long)listed_fixed_smem(capacity);
        const long big = ((long)optin - (long)fl.sharedSizeBytes - lfixed) / (long)sizeof(float4);
        long lfit = big;
        int lctas = 1;
        for (int c = kListedCtas; c >= 2; --c) {
            const long b = (long)per_sm / c - reserved - (long)fl.sharedSizeBytes;
            long f = b > lfixed ? (b - lfixed) / (long)sizeof(float4) : 0;
            if (f > big) f = big;
            while (f >= 2L * need) {
                int nb = 0;
                NL_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                    &nb, k_pairs_listed<CLOSE>, kListedWarps * 32,
                    sizeof(float4) * (size_t)f + (size_t)lfixed));
                if (nb >= c) break;
                f -= 32;
            }
            if (f >= 2L * need) {
                lfit = f;
                lctas = c;
                break;
            }
        }
        TileParams PL = P;
        PL.stage_max = (int)(lfit < kSlotLimit ? lfit : kSlotLimit);
        PL.fb_list = ctx->fb_list2;
        PL.fb_count = ctx->fb_count2;
        ProfScope ps(ctx, PH_PAIRS_LISTED, s);
        k_pairs_listed<CLOSE><<<(unsigned)(ctx->sm_count * lctas), kListedWarps * 32,
                                sizeof(float4) * (size_t)PL.stage_max + (size_t)lfixed, s>>>(g, PL);
        return cudaGetLastError();
    }
    ProfScope ps(ctx, PH_PAIRS_LISTED, s);
    const unsigned blocks =
        g.literal ? resident_grid(ctx, k_pairs_per_atom<true, CLOSE>, 128, 0, (n + 127) / 128)
                  : resident_grid(ctx, k_pairs_per_atom<false, CLOSE>, 128, 0, (n + 127) / 128);
    const float cd2 = CLOSE ? close->close_d2 : 0.0f;
    uint32_t *mb = CLOSE ? reinterpret_cast<uint32_t *>(close->min_d2) : nullptr;
    unsigned long long *nc = CLOSE ? reinterpret_cast<unsigned long long *>(close->n_close) : nullptr;
    if (g.literal)
        k_pairs_per_atom<true, CLOSE><<<(unsigned)blocks, 128, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, ctx->atom_cell, n, g, capacity, nbr, counts, ctx->flags,
            cd2, mb, nc);
    else
        k_pairs_per_atom<false, CLOSE><<<(unsigned)blocks, 128, 0, s>>>(
            ctx->cell_pos, ctx->cell_start, ctx->atom_cell, n, g, capacity, nbr, counts, ctx->flags,
            cd2, mb, nc);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pairs(nl_ctx *ctx, int64_t n, const CellGrid &g, int32_t capacity,
                         int32_t *nbr, int32_t *counts, cudaStream_t s, int *used_fast,
                         const CloseOut *close)
{
    if (close)
        return launch_pairs_t<true>(ctx, n, g, capacity, nbr, counts, s, used_fast, close);
    return launch_pairs_t<false>(ctx, n, g, capacity, nbr, counts, s, used_fast, nullptr);
}

}  // namespace nl
