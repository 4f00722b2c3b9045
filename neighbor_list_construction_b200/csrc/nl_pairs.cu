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

template <bool LITERAL>
__global__ void __launch_bounds__(128)
k_pairs_per_atom(const float4 *__restrict__ cell_pos, const int32_t *__restrict__ cell_start,
                 const uint32_t *__restrict__ atom_cell, int64_t n, CellGrid g, int32_t K,
                 int32_t *__restrict__ nbr, int32_t *__restrict__ counts, uint32_t *flags)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride) {
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
}

}  // namespace

cudaError_t launch_pairs(nl_ctx *ctx, int64_t n, const CellGrid &g, int32_t capacity,
                         int32_t *nbr, int32_t *counts, cudaStream_t s, int *used_fast)
{
    *used_fast = 0;
    if (n <= 0) return cudaSuccess;
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
