// nl_internal.cuh -- shared declarations of the libnl CUDA sources.
//
// Everything here is internal to libnl.so; the public C ABI is include/nl.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "nl.h"
#include "nl_device.cuh"


// ------------------------------------------------------------------ context
struct nl_ctx {
    int device = 0;
    int sm_count = 148;
    int edge_blocks_per_sm = 0;   // resident CTAs of the edge-feature kernel (0: not asked yet)
    int64_t max_atoms = 0;
    int32_t max_capacity = 0;
    int64_t max_cells = 0;

    // radix sort
    uint64_t *keys[2] = {nullptr, nullptr};
    uint32_t *vals[2] = {nullptr, nullptr};
    uint32_t *hist = nullptr;          // [8][256] counts, then exclusive starts
    uint32_t *sort_status = nullptr;   // [8][max_sort_tiles][256] look-back
    uint32_t *sort_ctr = nullptr;      // [8] tile tickets
    int64_t max_sort_tiles = 0;

    // cells
    int32_t *cell_count = nullptr;     // [max_cells]
    int32_t *cell_start = nullptr;     // [max_cells + 1]
    uint32_t *scan_status = nullptr;   // [max_scan_tiles]
    uint32_t *scan_ctr = nullptr;      // [1]
    int64_t max_scan_tiles = 0;
    uint32_t *atom_cell = nullptr;     // [max_atoms]
    uint32_t *atom_rank = nullptr;     // [max_atoms]
    float4 *cell_pos = nullptr;        // [max_atoms] wrapped xyz + index bits
    uint8_t *cell_tab = nullptr;       // [max_cells][16] x sub-bin tables
    float4 *ref = nullptr;             // [max_atoms] reference positions

    // status and small state
    uint32_t *flags = nullptr;         // [1]
    uint32_t *skin_acc = nullptr;      // [2]: max bits, block ticket
    int32_t *step = nullptr;           // [1] replay iteration index
    int32_t *rebuild_tmp = nullptr;    // [1]
    uint32_t *unsorted = nullptr;      // [1] 1 if a cell was too large for the in-cell sort
    uint32_t *fb_count = nullptr;      // [1] tiles listed for the larger-stage launch
    uint32_t *tile_ctr = nullptr;      // [1] next tile of the persistent pair search (after fb_count)
    uint32_t *fb_count2 = nullptr;     // [1] tiles listed by the two-stage pass (after tile_ctr)
    uint32_t *tile_ctr2 = nullptr;     // [1] next list entry of the two-stage pass
    uint32_t *fb_list2 = nullptr;      // [max_cells] their ids
    uint32_t *probe_word = nullptr;    // [1] a word nothing writes (bounded-wait self-test)
    uint32_t *sort_gate = nullptr;     // [1] set when the sort needs its full path
    uint32_t *fb_list = nullptr;       // [max_cells] their ids
    uint32_t *zero_block = nullptr;    // one allocation holding the small state

    // last build
    int64_t last_n = -1;
    nl::CellGrid last_grid{};
    int last_fast = 0;

    // replay cache
    cudaGraph_t replay_graph = nullptr;
    cudaGraphExec_t replay_exec = nullptr;
    unsigned char replay_key[128] = {0};
    int replay_key_len = 0;

    // profiling
    int prof_on = 0;
    static const int kProfSlots = 8192;
    cudaEvent_t *prof_ev = nullptr;    // [2 * kProfSlots]
    int *prof_phase = nullptr;         // [kProfSlots]
    int prof_used = 0;
    int prof_dropped = 0;
    double prof_ms[nl::PH_COUNT] = {0};
    int64_t prof_launches[nl::PH_COUNT] = {0};
};

namespace nl {

// -------------------------------------------------------------- profiling
// Returns a slot (or -1) and records its start event on `s`.
int prof_begin(nl_ctx *ctx, int phase, cudaStream_t s);
void prof_end(nl_ctx *ctx, int slot, cudaStream_t s);

struct ProfScope {
    nl_ctx *ctx;
    cudaStream_t s;
    int slot;
    ProfScope(nl_ctx *c, int phase, cudaStream_t st) : ctx(c), s(st), slot(prof_begin(c, phase, st)) {}
    ~ProfScope() { prof_end(ctx, slot, s); }
};

// ------------------------------------------------------------- launchers
// Curve keys of all atoms into ctx->keys[0]/vals[0] and the histograms of
// the top kTopPasses digits into ctx->hist (which must be zero); curve 0
// Hilbert, 1 Morton.  With a gate: only when *gate != 0, and the histograms
// of the other digits, and then it also clears zero[0, zero_words).
cudaError_t launch_keys(nl_ctx *ctx, int64_t n, const float4 *pos, float Lx, float Ly,
                        float Lz, float Sx, float Sy, float Sz, int curve, cudaStream_t s,
                        const uint32_t *gate = nullptr, uint32_t *zero = nullptr,
                        int64_t zero_words = 0);
// Exclusive scan of the 8 histograms in place; with a gate, only when
// *gate != 0 and only the digits below the top kTopPasses.
cudaError_t launch_hist_scan(nl_ctx *ctx, cudaStream_t s, const uint32_t *gate = nullptr);
// What the gated full sort needs to recompute the keys.
struct SortRecompute {
    const float4 *pos;
    int64_t n;
    float Lx, Ly, Lz, Sx, Sy, Sz;
    int curve;
};
// The sort of ctx->keys[0]/vals[0] (keys, histograms scanned): onesweep
// passes over the top kTopPasses digits and the prefix-run finish; behind
// them a gated full sort (keys recomputed, 8 passes) that runs only when a
// prefix run was longer than kRunMax.  Writes keys to keys_final (NULL: not
// kept) and indices to vals_final; with pos_sorted, also the positions in
// that order, (rk.pos[index].xyz, index) (the gather fused into the run
// finish, and a gated gather behind the full sort).
cudaError_t launch_radix_passes(nl_ctx *ctx, int64_t n, uint64_t *keys_final,
                                uint32_t *vals_final, cudaStream_t s, const SortRecompute &rk,
                                float4 *pos_sorted = nullptr);
// out[k] = (pos[perm[k]].xyz, perm[k]).  Returns at once when `flags` holds
// kFlagTimeout (perm may then be stale), or when gate is given and *gate == 0.
cudaError_t launch_gather(nl_ctx *ctx, int64_t n, const float4 *pos, const int32_t *perm,
                          float4 *out, const uint32_t *flags, cudaStream_t s,
                          const uint32_t *gate = nullptr);

// Cell binning of `pos` into ctx->cell_pos (cell order, x-sorted in cells).
cudaError_t launch_binning(nl_ctx *ctx, int64_t n, const float4 *pos, const CellGrid &g,
                           cudaStream_t s);
// One-time kernel attributes of the pair search (large dynamic shared memory).
cudaError_t pairs_set_attributes();
// Close-pair outputs of a build (device pointers): smallest pair r2 and the
// number of directed pairs with r2 < close_d2.
struct CloseOut {
    float close_d2;
    float *min_d2;
    int64_t *n_close;
};
// Pair search over the binned atoms; close may be NULL.
cudaError_t launch_pairs(nl_ctx *ctx, int64_t n, const CellGrid &g, int32_t capacity,
                         int32_t *nbr, int32_t *counts, cudaStream_t s, int *used_fast,
                         const CloseOut *close);

// Re-sort in place along the Hilbert curve of `pos` (S = fl(2^21 / L) per
// axis): pos, and ids / aux when not NULL, are permuted by the stable
// (key, slot) order.  Uses the sort scratch and the build's per-atom scratch.
cudaError_t launch_resort(nl_ctx *ctx, int64_t n, float4 *pos, int32_t *ids, float4 *aux,
                          float Lx, float Ly, float Lz, float Sx, float Sy, float Sz,
                          cudaStream_t s);

// CSR form of padded rows: offsets (int64 row_ptr[n + 1]; block_sums is
// scratch of csr_block_count(n) int64), then entries and, with edges, their
// features.
cudaError_t launch_csr_offsets(nl_ctx *ctx, int64_t n, const int32_t *counts, int32_t K,
                               int64_t *row_ptr, int64_t *block_sums, cudaStream_t s);
int64_t csr_block_count(int64_t n);
cudaError_t launch_csr_fill(nl_ctx *ctx, int64_t n, const int32_t *nbr, const int32_t *counts,
                            int32_t K, const int64_t *row_ptr, int32_t *col, const float4 *pos,
                            float Lx, float Ly, float Lz, float4 *edges, cudaStream_t s);

// Edge features (dx, dy, dz, r) of padded rows into out[n][K].
cudaError_t launch_edge_features(nl_ctx *ctx, int64_t n, const float4 *pos, float Lx, float Ly,
                                 float Lz, const int32_t *nbr, const int32_t *counts, int32_t K,
                                 float4 *out, cudaStream_t s);

// Skin check.  decisions/step may be NULL; cond_handle 0 = none.
cudaError_t launch_skin(nl_ctx *ctx, int64_t n, const float4 *pos, float Lx, float Ly,
                        float Lz, float h2, int32_t *rebuild_out, float *max_d2_out,
                        int32_t *decisions, const int32_t *step,
                        unsigned long long cond_handle, cudaStream_t s);

}  // namespace nl

namespace nl {

// Grid of a grid-stride kernel: `want` CTAs of `threads` threads, at most
// one resident wave (the SMs times the CTAs per SM the kernel's registers
// and shared memory allow), so no CTA waits for a second wave.
template <class Kernel>
inline unsigned resident_grid(const nl_ctx *ctx, Kernel kernel, int threads, size_t smem,
                              int64_t want)
{
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t cap = (int64_t)ctx->sm_count * per_sm;
    if (want > cap) want = cap;
    return (unsigned)(want < 1 ? 1 : want);
}

}  // namespace nl

#define NL_CUDA_TRY(expr)                                   \
    do {                                                    \
        cudaError_t _e = (expr);                            \
        if (_e != cudaSuccess) return _e;                   \
    } while (0)
