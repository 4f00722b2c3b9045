// nl_api.cu -- the C ABI of libnl.so (declared in include/nl.h).
//
// Host side: argument checks, the cell grid, scratch ownership, the replay
// graph and the timing hooks.  All arithmetic of the path runs in the
// kernels of the other sources.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>

#include "nl_internal.cuh"

using namespace nl;

namespace {

inline cudaStream_t S(void *s) { return reinterpret_cast<cudaStream_t>(s); }

template <typename T>
cudaError_t alloc(T **p, size_t count)
{
    *p = nullptr;
    if (count == 0) count = 1;
    return cudaMalloc(reinterpret_cast<void **>(p), count * sizeof(T));
}

void free_ctx(nl_ctx *c)
{
    if (!c) return;
    if (c->replay_exec) cudaGraphExecDestroy(c->replay_exec);
    if (c->replay_graph) cudaGraphDestroy(c->replay_graph);
    void *bufs[] = {c->keys[0], c->keys[1], c->vals[0], c->vals[1], c->hist, c->sort_status,
                    c->sort_ctr, c->cell_count, c->cell_start, c->scan_status, c->scan_ctr,
                    c->atom_cell, c->atom_rank, c->cell_pos, c->ref, c->zero_block,
                    c->fb_list, c->fb_list2, c->cell_tab};
    for (void *b : bufs)
        if (b) cudaFree(b);
    if (c->prof_ev) {
        for (int i = 0; i < 2 * nl_ctx::kProfSlots; ++i) cudaEventDestroy(c->prof_ev[i]);
        delete[] c->prof_ev;
        delete[] c->prof_phase;
    }
    delete c;
}

bool finite_pos(float v) { return std::isfinite(v) && v > 0.0f; }

nl_status check_box(const float *box)
{
    if (!box) return NL_ERR_ARG;
    for (int a = 0; a < 3; ++a)
        if (!finite_pos(box[a])) return NL_ERR_ARG;
    return NL_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Cell grid.  Preferred ("column") grid: cells at least rl wide along x and
// rl/2 wide along y and z, so a neighbor lies within +-1 cell in x and +-2
// cells in y and z; it needs >= 5 cells in x and >= 7 in y and z so that the
// periodic shift of every stencil cell is known (see nl_pairs.cu).  Smaller
// boxes get cells at least rl wide on every axis (>= 3 per axis, else
// NL_ERR_BOX) and the literal minimum image.  A cell's width carries a margin
// of rl*2^-20 + L*2^-20 over its nominal minimum, so the fp32 rounding of the
// cell assignment floor(w * fl(n/L)) never moves a neighbor outside the
// stencil.  Grids above the context's cell budget are coarsened.
nl_status make_grid(nl_ctx *ctx, const float *box, float cutoff, float skin, CellGrid *g)
{
    g->n_rows = INT64_MAX;
    g->n_dev = nullptr;
    if (!std::isfinite(cutoff) || !std::isfinite(skin) || cutoff < 0.0f || skin < 0.0f)
        return NL_ERR_ARG;
    volatile float rl = cutoff + skin;
    if (!(rl > 0.0f)) return NL_ERR_ARG;
    volatile float rl2 = rl * rl;
    const double eps = std::ldexp(1.0, -20);
    auto cells = [&](int a, double width) {
        const double L = box[a];
        const double m = std::floor(L / (width * (1.0 + eps) + L * eps));
        return m > 8192.0 ? (int64_t)8192 : (int64_t)m;
    };
    int64_t n[3];
    int wy = 2, wz = 2, literal = 0;
    n[0] = cells(0, (double)rl);
    n[1] = cells(1, 0.5 * (double)rl);
    n[2] = cells(2, 0.5 * (double)rl);
    bool columns = n[0] >= 5 && n[1] >= 7 && n[2] >= 7;
    if (columns) {
        while (n[0] * n[1] * n[2] > ctx->max_cells) {
            int a = n[0] > n[1] ? (n[0] > n[2] ? 0 : 2) : (n[1] > n[2] ? 1 : 2);
            n[a] = n[a] * 7 / 8;
        }
        columns = n[0] >= 5 && n[1] >= 7 && n[2] >= 7;
    }
    if (!columns) {
        wy = wz = 1;
        for (int a = 0; a < 3; ++a) {
            n[a] = cells(a, (double)rl);
            if (n[a] < 3) return NL_ERR_BOX;
        }
        while (n[0] * n[1] * n[2] > ctx->max_cells) {
            int a = n[0] > n[1] ? (n[0] > n[2] ? 0 : 2) : (n[1] > n[2] ? 1 : 2);
            n[a] = n[a] * 7 / 8;
            if (n[a] < 3) return NL_ERR_BOX;
        }
        literal = (n[0] < 5 || n[1] < 5 || n[2] < 5) ? 1 : 0;
    }
    g->nx = (int)n[0];
    g->ny = (int)n[1];
    g->nz = (int)n[2];
    g->Lx = box[0];
    g->Ly = box[1];
    g->Lz = box[2];
    volatile float tx = (float)g->nx / box[0];
    volatile float ty = (float)g->ny / box[1];
    volatile float tz = (float)g->nz / box[2];
    g->Tx = tx;
    g->Ty = ty;
    g->Tz = tz;
    g->rl2 = rl2;
    g->ncell = n[0] * n[1] * n[2];
    g->wy = wy;
    g->wz = wz;
    g->literal = literal;
    return NL_OK;
}

nl_status sort_impl(nl_ctx *ctx, int64_t n, const float *pos, const float *box, int32_t *perm,
                    float *pos_sorted, uint64_t *keys_out, void *stream, int curve)
{
    if (!ctx || n < 0) return NL_ERR_ARG;
    if (n > ctx->max_atoms) return NL_ERR_CAPACITY;
    if (check_box(box) != NL_OK) return NL_ERR_ARG;
    if (n == 0) return NL_OK;
    if (!pos || !perm || !pos_sorted || !aligned16(pos) || !aligned16(pos_sorted))
        return NL_ERR_ARG;
    cudaStream_t s = S(stream);
    volatile float sx = 2097152.0f / box[0];
    volatile float sy = 2097152.0f / box[1];
    volatile float sz = 2097152.0f / box[2];
    const float4 *p4 = reinterpret_cast<const float4 *>(pos);
    if (cudaMemsetAsync(ctx->hist, 0, sizeof(uint32_t) * kKeyPasses * kRadixBins, s) != cudaSuccess)
        return NL_ERR_CUDA;
    {
        ProfScope ps(ctx, PH_KEYS, s);
        if (launch_keys(ctx, n, p4, box[0], box[1], box[2], sx, sy, sz, curve, s) != cudaSuccess)
            return NL_ERR_CUDA;
    }
    {
        ProfScope ps(ctx, PH_KEY_SCAN, s);
        if (launch_hist_scan(ctx, s) != cudaSuccess) return NL_ERR_CUDA;
    }
    {
        ProfScope ps(ctx, PH_SORT, s);
        const SortRecompute rk{p4, n, box[0], box[1], box[2], sx, sy, sz, curve};
        if (launch_radix_passes(ctx, n, keys_out, reinterpret_cast<uint32_t *>(perm), s, rk,
                                reinterpret_cast<float4 *>(pos_sorted)) != cudaSuccess)
            return NL_ERR_CUDA;
    }
    return NL_OK;
}

nl_status build_checked(nl_ctx *ctx, int64_t n, const float *pos, const float *box, float cutoff,
                        float skin, int32_t capacity, int32_t *nbr, int32_t *counts, CellGrid *g,
                        bool need_rows = true)
{
    if (!ctx || n < 0) return NL_ERR_ARG;
    if (n > ctx->max_atoms || capacity > ctx->max_capacity) return NL_ERR_CAPACITY;
    if (capacity < 1) return NL_ERR_ARG;
    if (check_box(box) != NL_OK) return NL_ERR_ARG;
    if (n > 0 && (!pos || !aligned16(pos))) return NL_ERR_ARG;
    if (n > 0 && need_rows && (!nbr || !counts)) return NL_ERR_ARG;
    return make_grid(ctx, box, cutoff, skin, g);
}

nl_status build_enqueue(nl_ctx *ctx, int64_t n, const float *pos, const CellGrid &g,
                        int32_t capacity, int32_t *nbr, int32_t *counts, cudaStream_t s, int *fast,
                        const CloseOut *close = nullptr)
{
    // g.n_rows (INT64_MAX unless the caller set it) limits the rows written
    const float4 *p4 = reinterpret_cast<const float4 *>(pos);
    if (launch_binning(ctx, n, p4, g, s) != cudaSuccess) return NL_ERR_CUDA;
    if (launch_pairs(ctx, n, g, capacity, nbr, counts, s, fast, close) != cudaSuccess)
        return NL_ERR_CUDA;
    return NL_OK;
}

__global__ void k_close_init(float *min_d2, int64_t *n_close)
{
    *min_d2 = __int_as_float(0x7f800000);
    *n_close = 0;
}

// ------------------------------------------------------------- replay
__global__ void k_replay_init(int32_t *step) { *step = 0; }

__global__ void k_replay_advance(int32_t *step, int32_t n_steps, unsigned long long loop)
{
    const int32_t next = *step + 1;
    *step = next;
    cudaGraphSetConditional((cudaGraphConditionalHandle)loop, next < n_steps ? 1u : 0u);
}

// Adds `params` as a node after the current capture dependencies of `cs` and
// makes it the new dependency.
cudaError_t add_node_in_capture(cudaStream_t cs, cudaGraphNodeParams *params, cudaGraphNode_t *node)
{
    cudaStreamCaptureStatus st;
    cudaGraph_t g;
    const cudaGraphNode_t *deps = nullptr;
    size_t ndeps = 0;
    NL_CUDA_TRY(cudaStreamGetCaptureInfo(cs, &st, nullptr, &g, &deps, &ndeps));
    if (st != cudaStreamCaptureStatusActive) return cudaErrorStreamCaptureInvalidated;
    NL_CUDA_TRY(cudaGraphAddNode(node, g, deps, ndeps, params));
    return cudaStreamUpdateCaptureDependencies(cs, node, 1, cudaStreamSetCaptureDependencies);
}

cudaError_t add_child_in_capture(cudaStream_t cs, cudaGraph_t child)
{
    cudaStreamCaptureStatus st;
    cudaGraph_t g;
    const cudaGraphNode_t *deps = nullptr;
    size_t ndeps = 0;
    cudaGraphNode_t node;
    NL_CUDA_TRY(cudaStreamGetCaptureInfo(cs, &st, nullptr, &g, &deps, &ndeps));
    if (st != cudaStreamCaptureStatusActive) return cudaErrorStreamCaptureInvalidated;
    NL_CUDA_TRY(cudaGraphAddChildGraphNode(&node, g, deps, ndeps, child));
    return cudaStreamUpdateCaptureDependencies(cs, &node, 1, cudaStreamSetCaptureDependencies);
}

// What a rebuild re-sorts, when it does (nl_replay_resort).
struct ResortArgs {
    int32_t *ids;
    float *aux;
    float Sx, Sy, Sz;
};

// Builds the interval graph:
//   init(step = 0) -> WHILE(loop) { [step graph] -> skin check (sets cond) ->
//                                   IF(cond) { [re-sort] -> nl_build } -> advance(step++) }
cudaError_t make_replay_graph(nl_ctx *ctx, cudaGraph_t step_graph, int32_t n_steps, int64_t n,
                              float *pos, const CellGrid &g, float h2, int32_t capacity,
                              int32_t *nbr, int32_t *counts, int32_t *decisions,
                              const ResortArgs *rs, cudaGraph_t *out)
{
    cudaStream_t cs;
    NL_CUDA_TRY(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
    cudaGraph_t top = nullptr;
    cudaError_t e = cudaSuccess;
    const float4 *p4 = reinterpret_cast<const float4 *>(pos);
    int fast = 0;
    do {
        // top level
        e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed);
        if (e != cudaSuccess) break;
        k_replay_init<<<1, 1, 0, cs>>>(ctx->step);
        cudaStreamCaptureStatus st;
        cudaGraph_t capg;
        e = cudaStreamGetCaptureInfo(cs, &st, nullptr, &capg, nullptr, nullptr);
        if (e != cudaSuccess) break;
        cudaGraphConditionalHandle loop;
        e = cudaGraphConditionalHandleCreate(&loop, capg, n_steps > 0 ? 1u : 0u,
                                             cudaGraphCondAssignDefault);
        if (e != cudaSuccess) break;
        cudaGraphNodeParams wp = {};
        wp.type = cudaGraphNodeTypeConditional;
        wp.conditional.handle = loop;
        wp.conditional.type = cudaGraphCondTypeWhile;
        wp.conditional.size = 1;
        cudaGraphNode_t wnode;
        e = add_node_in_capture(cs, &wp, &wnode);
        if (e != cudaSuccess) break;
        cudaGraph_t body = wp.conditional.phGraph_out[0];
        e = cudaStreamEndCapture(cs, &top);
        if (e != cudaSuccess) break;

        // loop body
        cudaGraphConditionalHandle cond;
        e = cudaGraphConditionalHandleCreate(&cond, body, 0u, 0u);
        if (e != cudaSuccess) break;
        e = cudaStreamBeginCaptureToGraph(cs, body, nullptr, nullptr, 0, cudaStreamCaptureModeRelaxed);
        if (e != cudaSuccess) break;
        if (step_graph) {
            e = add_child_in_capture(cs, step_graph);
            if (e != cudaSuccess) break;
        }
        e = launch_skin(ctx, n, p4, g.Lx, g.Ly, g.Lz, h2, ctx->rebuild_tmp, nullptr, decisions,
                        ctx->step, (unsigned long long)cond, cs);
        if (e != cudaSuccess) break;
        cudaGraphNodeParams ip = {};
        ip.type = cudaGraphNodeTypeConditional;
        ip.conditional.handle = cond;
        ip.conditional.type = cudaGraphCondTypeIf;
        ip.conditional.size = 1;
        cudaGraphNode_t inode;
        e = add_node_in_capture(cs, &ip, &inode);
        if (e != cudaSuccess) break;
        cudaGraph_t ifbody = ip.conditional.phGraph_out[0];
        k_replay_advance<<<1, 1, 0, cs>>>(ctx->step, n_steps, (unsigned long long)loop);
        e = cudaGetLastError();
        if (e != cudaSuccess) break;
        cudaGraph_t tmp;
        e = cudaStreamEndCapture(cs, &tmp);
        if (e != cudaSuccess) break;

        // rebuild body
        e = cudaStreamBeginCaptureToGraph(cs, ifbody, nullptr, nullptr, 0,
                                          cudaStreamCaptureModeRelaxed);
        if (e != cudaSuccess) break;
        if (rs)
            e = launch_resort(ctx, n, reinterpret_cast<float4 *>(pos), rs->ids,
                              reinterpret_cast<float4 *>(rs->aux), g.Lx, g.Ly, g.Lz, rs->Sx, rs->Sy,
                              rs->Sz, cs);
        if (e == cudaSuccess &&
            build_enqueue(ctx, n, pos, g, capacity, nbr, counts, cs, &fast) != NL_OK)
            e = cudaErrorUnknown;
        cudaGraph_t tmp2;
        cudaError_t e2 = cudaStreamEndCapture(cs, &tmp2);
        if (e == cudaSuccess) e = e2;
    } while (0);
    if (e != cudaSuccess) {
        cudaStreamCaptureStatus st;
        if (cudaStreamIsCapturing(cs, &st) == cudaSuccess && st != cudaStreamCaptureStatusNone) {
            cudaGraph_t junk = nullptr;
            cudaStreamEndCapture(cs, &junk);
            if (junk) cudaGraphDestroy(junk);
        }
        if (top) cudaGraphDestroy(top);
        top = nullptr;
        cudaGetLastError();
    }
    cudaStreamDestroy(cs);
    *out = top;
    return e;
}

}  // namespace

// ------------------------------------------------------------ profiling
namespace nl {

int prof_begin(nl_ctx *ctx, int phase, cudaStream_t s)
{
    if (!ctx || !ctx->prof_on) return -1;
    cudaStreamCaptureStatus st;
    if (cudaStreamIsCapturing(s, &st) != cudaSuccess || st != cudaStreamCaptureStatusNone)
        return -1;
    if (ctx->prof_used >= nl_ctx::kProfSlots) {
        ++ctx->prof_dropped;
        return -1;
    }
    const int slot = ctx->prof_used++;
    ctx->prof_phase[slot] = phase;
    cudaEventRecord(ctx->prof_ev[2 * slot], s);
    return slot;
}

void prof_end(nl_ctx *ctx, int slot, cudaStream_t s)
{
    if (slot < 0) return;
    cudaEventRecord(ctx->prof_ev[2 * slot + 1], s);
}

}  // namespace nl

// ---------------------------------------------------------------- C ABI
extern "C" {

const char *nl_status_string(nl_status s)
{
    switch (s) {
    case NL_OK: return "NL_OK";
    case NL_OVERFLOW: return "NL_OVERFLOW: a row has more neighbors than the capacity";
    case NL_ERR_ARG: return "NL_ERR_ARG: invalid argument";
    case NL_ERR_BOX: return "NL_ERR_BOX: box narrower than three cells of width cutoff+skin";
    case NL_ERR_CUDA: return "NL_ERR_CUDA: CUDA runtime error";
    case NL_ERR_TIMEOUT: return "NL_ERR_TIMEOUT: a bounded device wait gave up";
    case NL_ERR_CAPACITY: return "NL_ERR_CAPACITY: n or capacity above the context maximum";
    case NL_ERR_HALO: return "NL_ERR_HALO: a halo block or buffer was too small; rows incomplete";
    }
    return "unknown nl_status";
}

nl_status nl_create(nl_ctx **out, int64_t max_atoms, int32_t max_capacity)
{
    if (!out) return NL_ERR_ARG;
    *out = nullptr;
    if (max_atoms < 0 || max_atoms > (int64_t(1) << 30) || max_capacity < 1) return NL_ERR_ARG;
    nl_ctx *c = new (std::nothrow) nl_ctx();
    if (!c) return NL_ERR_CUDA;
    if (cudaGetDevice(&c->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device) !=
            cudaSuccess) {
        delete c;
        cudaGetLastError();
        return NL_ERR_CUDA;
    }
    const int64_t N = max_atoms > 0 ? max_atoms : 1;
    c->max_atoms = max_atoms;
    c->max_capacity = max_capacity;
    c->max_cells = N > 32768 ? N : 32768;
    c->max_sort_tiles = (N + kSortTile - 1) / kSortTile;
    c->max_scan_tiles = (c->max_cells + kScanTile - 1) / kScanTile;
    bool ok = true;
    ok &= alloc(&c->keys[0], N) == cudaSuccess;
    ok &= alloc(&c->keys[1], N) == cudaSuccess;
    ok &= alloc(&c->vals[0], N) == cudaSuccess;
    ok &= alloc(&c->vals[1], N) == cudaSuccess;
    ok &= alloc(&c->hist, kKeyPasses * kRadixBins) == cudaSuccess;
    ok &= alloc(&c->sort_status, (size_t)kStatusPasses * c->max_sort_tiles * kRadixBins) == cudaSuccess;
    ok &= alloc(&c->sort_ctr, kStatusPasses) == cudaSuccess;
    ok &= alloc(&c->cell_count, c->max_cells) == cudaSuccess;
    ok &= alloc(&c->cell_start, c->max_cells + 1) == cudaSuccess;
    ok &= alloc(&c->scan_status, c->max_scan_tiles) == cudaSuccess;
    ok &= alloc(&c->scan_ctr, 1) == cudaSuccess;
    ok &= alloc(&c->atom_cell, N) == cudaSuccess;
    ok &= alloc(&c->atom_rank, N) == cudaSuccess;
    ok &= alloc(&c->cell_pos, N) == cudaSuccess;
    ok &= alloc(&c->ref, N) == cudaSuccess;
    ok &= alloc(&c->zero_block, 64) == cudaSuccess;
    ok &= alloc(&c->fb_list, c->max_cells) == cudaSuccess;
    ok &= alloc(&c->fb_list2, c->max_cells) == cudaSuccess;
    ok &= alloc(&c->cell_tab, (size_t)c->max_cells * 16) == cudaSuccess;
    if (ok) {
        c->flags = c->zero_block;
        c->skin_acc = c->zero_block + 4;
        c->step = reinterpret_cast<int32_t *>(c->zero_block + 8);
        c->rebuild_tmp = reinterpret_cast<int32_t *>(c->zero_block + 9);
        c->unsorted = c->zero_block + 12;
        c->fb_count = c->zero_block + 13;
        c->tile_ctr = c->zero_block + 14;
        c->fb_count2 = c->zero_block + 15;
        c->tile_ctr2 = c->zero_block + 16;
        c->sort_gate = c->zero_block + 17;
        c->probe_word = c->zero_block + 18;
        ok &= pairs_set_attributes() == cudaSuccess;
        ok &= cudaMemset(c->zero_block, 0, 64 * sizeof(uint32_t)) == cudaSuccess;
        ok &= cudaDeviceSynchronize() == cudaSuccess;
    }
    if (!ok) {
        cudaGetLastError();
        free_ctx(c);
        return NL_ERR_CUDA;
    }
    *out = c;
    return NL_OK;
}

void nl_destroy(nl_ctx *ctx)
{
    if (!ctx) return;
    cudaDeviceSynchronize();
    free_ctx(ctx);
}

nl_status nl_sort_hilbert(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                          int32_t *perm_out, float *pos_sorted_out, uint64_t *keys_out,
                          void *stream)
{
    return sort_impl(ctx, n, pos, box, perm_out, pos_sorted_out, keys_out, stream, 0);
}

nl_status nl_sort_morton(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                         int32_t *perm_out, float *pos_sorted_out, uint64_t *keys_out,
                         void *stream)
{
    return sort_impl(ctx, n, pos, box, perm_out, pos_sorted_out, keys_out, stream, 1);
}

nl_status nl_build(nl_ctx *ctx, int64_t n, const float *pos, const float *box, float cutoff,
                   float skin, int32_t capacity, int32_t *nbr_out, int32_t *counts_out,
                   void *stream)
{
    CellGrid g;
    nl_status st = build_checked(ctx, n, pos, box, cutoff, skin, capacity, nbr_out, counts_out, &g);
    if (st != NL_OK) return st;
    int fast = 0;
    st = build_enqueue(ctx, n, pos, g, capacity, nbr_out, counts_out, S(stream), &fast);
    if (st != NL_OK) return st;
    ctx->last_n = n;
    ctx->last_grid = g;
    ctx->last_fast = fast;
    return NL_OK;
}

nl_status nl_build_rows_dev(nl_ctx *ctx, int64_t n_max, const int64_t *n_dev, int64_t n_rows,
                            const float *pos, const float *box, float cutoff, float skin,
                            int32_t capacity, int32_t *nbr_out, int32_t *counts_out, void *stream)
{
    if (!n_dev || n_rows < 0 || n_rows > n_max) return NL_ERR_ARG;
    CellGrid g;
    nl_status st = build_checked(ctx, n_max, pos, box, cutoff, skin, capacity, nbr_out,
                                 counts_out, &g, n_rows > 0);
    if (st != NL_OK) return st;
    g.n_rows = n_rows;
    g.n_dev = n_dev;
    int fast = 0;
    st = build_enqueue(ctx, n_max, pos, g, capacity, nbr_out, counts_out, S(stream), &fast);
    if (st != NL_OK) return st;
    ctx->last_n = n_max;
    ctx->last_grid = g;
    ctx->last_grid.n_dev = nullptr;   // the pointer is the caller's
    ctx->last_fast = fast;
    return NL_OK;
}

nl_status nl_build_rows(nl_ctx *ctx, int64_t n, int64_t n_rows, const float *pos,
                        const float *box, float cutoff, float skin, int32_t capacity,
                        int32_t *nbr_out, int32_t *counts_out, void *stream)
{
    if (n_rows < 0 || n_rows > n) return NL_ERR_ARG;
    CellGrid g;
    nl_status st = build_checked(ctx, n, pos, box, cutoff, skin, capacity, nbr_out, counts_out, &g,
                                 n_rows > 0);
    if (st != NL_OK) return st;
    g.n_rows = n_rows;
    int fast = 0;
    st = build_enqueue(ctx, n, pos, g, capacity, nbr_out, counts_out, S(stream), &fast);
    if (st != NL_OK) return st;
    ctx->last_n = n;
    ctx->last_grid = g;
    ctx->last_fast = fast;
    return NL_OK;
}

nl_status nl_build_close(nl_ctx *ctx, int64_t n, const float *pos, const float *box, float cutoff,
                         float skin, int32_t capacity, int32_t *nbr_out, int32_t *counts_out,
                         float close_d2, float *min_d2_out, int64_t *n_close_out, void *stream)
{
    if (!min_d2_out || !n_close_out || !std::isfinite(close_d2) || close_d2 < 0.0f)
        return NL_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(min_d2_out) & 3u) || (reinterpret_cast<uintptr_t>(n_close_out) & 7u))
        return NL_ERR_ARG;
    CellGrid g;
    nl_status st = build_checked(ctx, n, pos, box, cutoff, skin, capacity, nbr_out, counts_out, &g);
    if (st != NL_OK) return st;
    k_close_init<<<1, 1, 0, S(stream)>>>(min_d2_out, n_close_out);
    if (cudaGetLastError() != cudaSuccess) return NL_ERR_CUDA;
    CloseOut close{close_d2, min_d2_out, n_close_out};
    int fast = 0;
    st = build_enqueue(ctx, n, pos, g, capacity, nbr_out, counts_out, S(stream), &fast, &close);
    if (st != NL_OK) return st;
    ctx->last_n = n;
    ctx->last_grid = g;
    ctx->last_fast = fast;
    return NL_OK;
}

nl_status nl_skin_check(nl_ctx *ctx, int64_t n, const float *pos, const float *box, float skin,
                        int32_t *rebuild_out, float *max_d2_out, void *stream)
{
    if (!ctx || n < 0 || !rebuild_out || check_box(box) != NL_OK) return NL_ERR_ARG;
    if (!std::isfinite(skin) || skin < 0.0f) return NL_ERR_ARG;
    if (n != ctx->last_n) return NL_ERR_ARG;
    if (n > 0 && (!pos || !aligned16(pos))) return NL_ERR_ARG;
    volatile float h = skin * 0.5f;
    volatile float h2 = h * h;
    if (launch_skin(ctx, n, reinterpret_cast<const float4 *>(pos), box[0], box[1], box[2], h2,
                    rebuild_out, max_d2_out, nullptr, nullptr, 0ull, S(stream)) != cudaSuccess)
        return NL_ERR_CUDA;
    return NL_OK;
}

nl_status nl_edge_features(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                           const int32_t *nbr, const int32_t *counts, int32_t capacity,
                           float *edges_out, void *stream)
{
    if (!ctx || n < 0 || n > ((int64_t)1 << 30) || capacity < 1 || check_box(box) != NL_OK)
        return NL_ERR_ARG;
    if (n > 0 && (!pos || !nbr || !counts || !edges_out || !aligned16(pos) ||
                  !aligned16(edges_out)))
        return NL_ERR_ARG;
    if (launch_edge_features(ctx, n, reinterpret_cast<const float4 *>(pos), box[0], box[1], box[2],
                             nbr, counts, capacity, reinterpret_cast<float4 *>(edges_out),
                             S(stream)) != cudaSuccess)
        return NL_ERR_CUDA;
    return NL_OK;
}

}  // extern "C"

namespace {

nl_status replay_impl(nl_ctx *ctx, void *step_graph, int32_t n_steps, int64_t n, float *pos,
                      const float *box, float cutoff, float skin, int32_t capacity, int32_t *nbr,
                      int32_t *counts, int32_t *decisions_out, void *stream, bool resort,
                      int32_t *ids, float *aux)
{
    if (n_steps < 0 || (n_steps > 0 && !decisions_out)) return NL_ERR_ARG;
    CellGrid g;
    nl_status st = build_checked(ctx, n, pos, box, cutoff, skin, capacity, nbr, counts, &g);
    if (st != NL_OK) return st;
    if (n != ctx->last_n) return NL_ERR_ARG;
    if (n_steps == 0) return NL_OK;
    volatile float h = skin * 0.5f;
    volatile float h2 = h * h;

    unsigned char key[128];
    int kl = 0;
    auto put = [&](const void *p, size_t sz) {
        memcpy(key + kl, p, sz);
        kl += (int)sz;
    };
    put(&step_graph, sizeof(void *));
    put(&n_steps, sizeof(n_steps));
    put(&n, sizeof(n));
    put(&pos, sizeof(pos));
    put(box, 3 * sizeof(float));
    put(&cutoff, sizeof(float));
    put(&skin, sizeof(float));
    put(&capacity, sizeof(capacity));
    put(&nbr, sizeof(nbr));
    put(&counts, sizeof(counts));
    put(&decisions_out, sizeof(decisions_out));
    const unsigned char rflag = resort ? 1 : 0;
    put(&rflag, 1);
    put(&ids, sizeof(ids));
    put(&aux, sizeof(aux));
    if (!ctx->replay_exec || ctx->replay_key_len != kl || memcmp(ctx->replay_key, key, kl) != 0) {
        if (ctx->replay_exec) cudaGraphExecDestroy(ctx->replay_exec);
        if (ctx->replay_graph) cudaGraphDestroy(ctx->replay_graph);
        ctx->replay_exec = nullptr;
        ctx->replay_graph = nullptr;
        cudaGraph_t gr = nullptr;
        ResortArgs ra{ids, aux, 0.0f, 0.0f, 0.0f};
        if (resort) {
            volatile float sx = 2097152.0f / box[0];
            volatile float sy = 2097152.0f / box[1];
            volatile float sz = 2097152.0f / box[2];
            ra.Sx = sx;
            ra.Sy = sy;
            ra.Sz = sz;
        }
        cudaError_t e = make_replay_graph(ctx, reinterpret_cast<cudaGraph_t>(step_graph), n_steps,
                                          n, pos, g, h2, capacity, nbr, counts, decisions_out,
                                          resort ? &ra : nullptr, &gr);
        if (e != cudaSuccess || !gr) {
            fprintf(stderr, "nl_replay: graph construction failed: %s\n", cudaGetErrorString(e));
            return NL_ERR_CUDA;
        }
        cudaGraphExec_t ex = nullptr;
        e = cudaGraphInstantiate(&ex, gr, 0);
        if (e != cudaSuccess) {
            fprintf(stderr, "nl_replay: instantiate failed: %s\n", cudaGetErrorString(e));
            cudaGraphDestroy(gr);
            cudaGetLastError();
            return NL_ERR_CUDA;
        }
        ctx->replay_graph = gr;
        ctx->replay_exec = ex;
        memcpy(ctx->replay_key, key, kl);
        ctx->replay_key_len = kl;
    }
    if (cudaGraphLaunch(ctx->replay_exec, S(stream)) != cudaSuccess) return NL_ERR_CUDA;
    ctx->last_grid = g;
    return NL_OK;
}

// One thread polls a word that nothing writes, under the rule of the
// look-back waits (a 64 ns sleep between polls after the first 64), and
// records the timeout in the status word as a look-back that gives up does.
__global__ void k_wait_selftest(const uint32_t *word, uint32_t max_polls, uint32_t *flags)
{
    if (threadIdx.x != 0) return;
    for (uint32_t spins = 0u; ld_volatile_u32(word) == 0u;) {
        if (++spins >= max_polls) {
            atomicOr(flags, kFlagTimeout);
            return;
        }
        if (spins > 64u) __nanosleep(64);
    }
}

}  // namespace

extern "C" {

nl_status nl_csr_offsets(nl_ctx *ctx, int64_t n, const int32_t *counts, int32_t capacity,
                         int64_t *row_ptr_out, void *stream)
{
    if (!ctx || n < 0 || capacity < 1 || !row_ptr_out || (n > 0 && !counts)) return NL_ERR_ARG;
    if (n > ctx->max_atoms) return NL_ERR_CAPACITY;
    // the sort's look-back words serve as the scan's block sums (int64)
    static_assert(sizeof(int64_t) == 2 * sizeof(uint32_t), "int64 block sums");
    if (launch_csr_offsets(ctx, n, counts, capacity, row_ptr_out,
                           reinterpret_cast<int64_t *>(ctx->sort_status), S(stream)) != cudaSuccess)
        return NL_ERR_CUDA;
    return NL_OK;
}

nl_status nl_csr_fill(nl_ctx *ctx, int64_t n, const int32_t *nbr, const int32_t *counts,
                      int32_t capacity, const int64_t *row_ptr, int32_t *col_out,
                      const float *pos, const float *box, float *edges_out, void *stream)
{
    if (!ctx || n < 0 || capacity < 1) return NL_ERR_ARG;
    if (n > 0 && (!nbr || !counts || !row_ptr || !col_out)) return NL_ERR_ARG;
    if (edges_out && (check_box(box) != NL_OK || (n > 0 && (!pos || !aligned16(pos))) ||
                      !aligned16(edges_out)))
        return NL_ERR_ARG;
    const float Lx = edges_out ? box[0] : 1.0f, Ly = edges_out ? box[1] : 1.0f,
                Lz = edges_out ? box[2] : 1.0f;
    if (launch_csr_fill(ctx, n, nbr, counts, capacity, row_ptr, col_out,
                        reinterpret_cast<const float4 *>(pos), Lx, Ly, Lz,
                        reinterpret_cast<float4 *>(edges_out), S(stream)) != cudaSuccess)
        return NL_ERR_CUDA;
    return NL_OK;
}

nl_status nl_replay(nl_ctx *ctx, void *step_graph, int32_t n_steps, int64_t n, float *pos,
                    const float *box, float cutoff, float skin, int32_t capacity, int32_t *nbr,
                    int32_t *counts, int32_t *decisions_out, void *stream)
{
    return replay_impl(ctx, step_graph, n_steps, n, pos, box, cutoff, skin, capacity, nbr, counts,
                       decisions_out, stream, false, nullptr, nullptr);
}

nl_status nl_replay_resort(nl_ctx *ctx, void *step_graph, int32_t n_steps, int64_t n, float *pos,
                           int32_t *ids, float *aux, const float *box, float cutoff, float skin,
                           int32_t capacity, int32_t *nbr, int32_t *counts,
                           int32_t *decisions_out, void *stream)
{
    if (aux && !aligned16(aux)) return NL_ERR_ARG;
    return replay_impl(ctx, step_graph, n_steps, n, pos, box, cutoff, skin, capacity, nbr, counts,
                       decisions_out, stream, true, ids, aux);
}

const int32_t *nl_step_counter(nl_ctx *ctx) { return ctx ? ctx->step : nullptr; }

nl_status nl_wait_selftest(nl_ctx *ctx, int32_t max_polls, void *stream)
{
    if (!ctx || max_polls < 1 || (uint32_t)max_polls > kSpinLimit) return NL_ERR_ARG;
    k_wait_selftest<<<1, 32, 0, S(stream)>>>(ctx->probe_word, (uint32_t)max_polls, ctx->flags);
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

nl_status nl_sync_status(nl_ctx *ctx, void *stream)
{
    if (!ctx) return NL_ERR_ARG;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return NL_ERR_CUDA;
    uint32_t f = 0;
    if (cudaMemcpy(&f, ctx->flags, sizeof(f), cudaMemcpyDeviceToHost) != cudaSuccess)
        return NL_ERR_CUDA;
    if (f && cudaMemset(ctx->flags, 0, sizeof(uint32_t)) != cudaSuccess) return NL_ERR_CUDA;
    if (f & kFlagTimeout) return NL_ERR_TIMEOUT;
    if (f & kFlagHalo) return NL_ERR_HALO;
    if (f & kFlagOverflow) return NL_OVERFLOW;
    return NL_OK;
}

nl_status nl_last_build_info(nl_ctx *ctx, int64_t out[8])
{
    if (!ctx || !out) return NL_ERR_ARG;
    out[0] = ctx->last_grid.nx;
    out[1] = ctx->last_grid.ny;
    out[2] = ctx->last_grid.nz;
    out[3] = ctx->last_fast;
    out[4] = ctx->last_grid.ncell;
    out[5] = ctx->last_grid.literal;
    out[6] = 0;
    out[7] = 0;
    return NL_OK;
}

nl_status nl_profile_enable(nl_ctx *ctx, int on)
{
    if (!ctx) return NL_ERR_ARG;
    if (on && !ctx->prof_ev) {
        ctx->prof_ev = new (std::nothrow) cudaEvent_t[2 * nl_ctx::kProfSlots];
        ctx->prof_phase = new (std::nothrow) int[nl_ctx::kProfSlots];
        if (!ctx->prof_ev || !ctx->prof_phase) return NL_ERR_CUDA;
        for (int i = 0; i < 2 * nl_ctx::kProfSlots; ++i)
            if (cudaEventCreate(&ctx->prof_ev[i]) != cudaSuccess) return NL_ERR_CUDA;
    }
    ctx->prof_on = on ? 1 : 0;
    return NL_OK;
}

int32_t nl_profile_read(nl_ctx *ctx, double *ms_out, int64_t *launches_out, int32_t max_phases)
{
    if (!ctx) return -1;
    if (ctx->prof_used > 0) {
        if (cudaDeviceSynchronize() != cudaSuccess) return -1;
        for (int s = 0; s < ctx->prof_used; ++s) {
            float ms = 0.0f;
            if (cudaEventElapsedTime(&ms, ctx->prof_ev[2 * s], ctx->prof_ev[2 * s + 1]) == cudaSuccess) {
                ctx->prof_ms[ctx->prof_phase[s]] += ms;
                ctx->prof_launches[ctx->prof_phase[s]] += 1;
            }
        }
        ctx->prof_used = 0;
    }
    const int np = PH_COUNT < max_phases ? PH_COUNT : max_phases;
    for (int p = 0; p < np; ++p) {
        if (ms_out) ms_out[p] = ctx->prof_ms[p];
        if (launches_out) launches_out[p] = ctx->prof_launches[p];
    }
    for (int p = 0; p < PH_COUNT; ++p) {
        ctx->prof_ms[p] = 0.0;
        ctx->prof_launches[p] = 0;
    }
    return PH_COUNT;
}

const char *nl_profile_phase_name(int32_t phase)
{
    static const char *names[PH_COUNT] = {"keys",        "key_scan",   "radix_sort", "gather",
                                          "bin_count",   "cell_scan",  "bin_scatter",
                                          "cell_sort",   "pair_search", "pair_search_listed",
                                          "skin_check",  "edge_features"};
    if (phase < 0 || phase >= PH_COUNT) return "";
    return names[phase];
}

}  // extern "C"
