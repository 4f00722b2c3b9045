/*
 * nl.h -- C ABI of libnl.so, the B200 (sm_100a) periodic neighbor-list build.
 *
 * Method source: "Ab Initio Accuracy Beyond the Cutoff: Distributed
 * Message-Passing Equivariant Attention at Tens-of-Millions-of-Atom Scale"
 * (Tessera), abstract.  The runtime described there sorts atoms along a
 * space-filling curve, searches neighbors through a multi-level structure,
 * keeps tensor shapes fixed between rebuilds with a conservative neighbor
 * skin, and replays each rebuild interval as one CUDA Graph.  The pages give
 * no formulas or API; the definitions below are this library's readings.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Positions      `pos` is a DEVICE pointer to n x 4 floats (float4 per atom,
 *                16-byte aligned): x, y, z in angstrom; the 4th float is
 *                ignored on input.  Coordinates must be finite; they may lie
 *                outside the box (they are wrapped, see below).
 * Box            `box` is a HOST pointer to 3 floats (Lx, Ly, Lz), an
 *                orthorhombic periodic box with its corner at the origin.
 * Wrap           w = x - L*floor(x/L) in fp32, then one fold into [0, L)
 *                (add L if negative, subtract L if >= L, 0 if still outside).
 * Distance       d = w_j - w_i; d = d - L*rintf(d/L) per axis;
 *                r2 = (dx*dx + dy*dy) + dz*dz, every operation an fp32
 *                round-to-nearest-even without fused multiply-add.
 * Neighbors      N(i) = { j != i : r2 < rl*rl }, rl = fl(cutoff + skin),
 *                strict inequality; a full (directed) list.
 * Streams        `stream` is a cudaStream_t (NULL = the legacy default
 *                stream).  Every call only enqueues work on it and returns;
 *                no call synchronizes except nl_sync_status.
 * Ownership      all array arguments are caller-owned device buffers; the
 *                context owns all scratch.  After nl_create no call
 *                allocates device memory.
 * Errors         the return value reports argument and launch errors only.
 *                Conditions found on the device (row overflow, a bounded
 *                spin that gave up) are accumulated in the context and
 *                returned, then cleared, by nl_sync_status.
 */
#ifndef NL_H
#define NL_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct nl_ctx nl_ctx;

typedef enum {
    NL_OK = 0,
    NL_OVERFLOW = 1,       /* some atom has more than `capacity` neighbors:
                              counts are true counts, such rows hold `capacity`
                              of them, every other row is complete */
    NL_ERR_ARG = -1,       /* NULL pointer, n < 0, bad float, misaligned pos */
    NL_ERR_BOX = -2,       /* box narrower than three cells of width rl on
                              some axis (a cell must be at least rl wide) */
    NL_ERR_CUDA = -3,      /* a CUDA runtime call failed */
    NL_ERR_TIMEOUT = -4,   /* a bounded device-side wait gave up; results of
                              that call are not valid */
    NL_ERR_CAPACITY = -5,  /* n > max_atoms or capacity > max_capacity */
    NL_ERR_HALO = -6       /* a halo block or the halo buffer of a sharded build
                              was too small (nl_halo_fill_blocks,
                              nl_halo_pack): atoms were dropped and the rows
                              of that build are incomplete; retry with larger
                              blocks */
} nl_status;

/* Creates a context on the current CUDA device and allocates all scratch for
 * up to `max_atoms` atoms (<= 2^30) and rows of up to `max_capacity`
 * neighbors.  Returns NL_ERR_CUDA if the allocation fails. */
nl_status nl_create(nl_ctx **ctx, int64_t max_atoms, int32_t max_capacity);

/* Frees the context and its scratch.  Waits for the context's work. */
void nl_destroy(nl_ctx *ctx);

/* Space-filling-curve order (Tessera abstract: atoms are sorted along a
 * space-filling curve).  Per atom: wrap, quantize each axis to 21 bits as
 * q = min(floor(w * fl(2^21/L)), 2^21-1), form the 63-bit 3-D Hilbert index
 * of (qx, qy, qz) (J. Skilling, "Programming the Hilbert curve", 2004:
 * axes-to-transpose, index bits from the top level down, x first in each
 * triple), then sort (key, original index) pairs ascending with a stable
 * LSD radix sort, so equal keys keep index order.
 * Outputs (device): perm_out[k] = original index of the k-th atom (int32,
 * n entries); pos_sorted_out[k] = (x, y, z of atom perm_out[k] as given,
 * 4th float = perm_out[k] as int32 bits) (n float4); keys_out[k] = its key
 * (uint64, may be NULL). */
nl_status nl_sort_hilbert(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                          int32_t *perm_out, float *pos_sorted_out, uint64_t *keys_out,
                          void *stream);

/* As nl_sort_hilbert with the Morton (Z-order) key instead: key bit 3l+2 =
 * bit l of qx, 3l+1 = qy, 3l = qz.  The baseline order the Tessera abstract
 * compares against. */
nl_status nl_sort_morton(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                         int32_t *perm_out, float *pos_sorted_out, uint64_t *keys_out,
                         void *stream);

/* Fixed-capacity neighbor list (Tessera abstract: workload shapes fixed
 * between rebuilds; neighbor search through curve order, cells and pairs).
 * Outputs (device): nbr_out is n x capacity int32, row-major; row i holds
 * the indices (into `pos`) of N(i) in an unspecified order, then -1 up to
 * `capacity`; if |N(i)| > capacity the row holds `capacity` members of N(i).
 * counts_out[i] = |N(i)| (true count, int32).  Also snapshots `pos` as the
 * reference positions of nl_skin_check.  Requires every box side to hold at
 * least three cells of width rl (else NL_ERR_BOX); rl <= 0 or capacity < 1
 * is NL_ERR_ARG. */
nl_status nl_build(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                   float cutoff, float skin, int32_t capacity,
                   int32_t *nbr_out, int32_t *counts_out, void *stream);

/* nl_build that writes rows for the first n_rows atoms of `pos` only
 * (0 <= n_rows <= n): their neighbors are searched among all n atoms, but
 * the atoms at n_rows.. (a halo received from other GPUs, say) get no row.
 * nbr_out is n_rows x capacity, counts_out int32[n_rows] (either may be NULL
 * when n_rows == 0); everything else as nl_build, which is n_rows == n.
 * n_rows outside [0, n] is NL_ERR_ARG. */
nl_status nl_build_rows(nl_ctx *ctx, int64_t n, int64_t n_rows, const float *pos,
                        const float *box, float cutoff, float skin, int32_t capacity,
                        int32_t *nbr_out, int32_t *counts_out, void *stream);

/* nl_build_rows whose atom count lives in device memory: *n_dev (int64,
 * device, read by the kernels; values outside [0, n_max] are clamped) atoms
 * of `pos` take part, pos holding room for n_max.  n_max bounds every launch
 * and the context check (n_max <= max_atoms), so the host never reads the
 * count: a sharded build can size its halo on the device and build without a
 * synchronization.  The pair search's shared-memory stages are sized for
 * n_max atoms in the box.  n_rows <= n_max rows are written; a NULL n_dev or
 * n_rows outside [0, n_max] is NL_ERR_ARG.  Everything else as
 * nl_build_rows. */
nl_status nl_build_rows_dev(nl_ctx *ctx, int64_t n_max, const int64_t *n_dev, int64_t n_rows,
                            const float *pos, const float *box, float cutoff, float skin,
                            int32_t capacity, int32_t *nbr_out, int32_t *counts_out,
                            void *stream);

/* nl_build with a close-pair detector as a by-product (Tessera abstract:
 * the simulations show no anomalously close pairs; this reports them while
 * the list is built).  Same arguments, results and status as nl_build, plus:
 *   *min_d2_out  (device float[1], 4-byte aligned): the smallest r2 over all
 *                directed neighbor pairs (i, j in N(i)), counted before the
 *                capacity cut; +inf when there is no pair within rl;
 *   *n_close_out (device int64[1], 8-byte aligned): the number of directed
 *                neighbor pairs with r2 < close_d2 (strict), again over the
 *                full neighbor sets.
 * r2 is the same fp32 value that decides membership.  close_d2 must be
 * finite and >= 0, and both pointers non-NULL, else NL_ERR_ARG.  Both
 * outputs are written on `stream` (initialised there before the search). */
nl_status nl_build_close(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                         float cutoff, float skin, int32_t capacity,
                         int32_t *nbr_out, int32_t *counts_out, float close_d2,
                         float *min_d2_out, int64_t *n_close_out, void *stream);

/* Edge features of padded rows (Tessera abstract: the model consumes the
 * neighbor topology as fixed-shape tensors; the page on batching and kernel
 * fusion: padded, dense per-atom neighborhoods).  For row i and slot
 * s < min(counts[i], capacity), with j = nbr[i][s]:
 *     edges_out[i][s] = (dx, dy, dz, r),
 * (dx, dy, dz) the minimum-image displacement from atom i to atom j (the
 * same fp32 values as in nl_build's predicate: wrapped coordinates, per axis
 * d - L*rintf(d/L) of d = w_j - w_i) and r = sqrt((dx*dx + dy*dy) + dz*dz),
 * correctly rounded.  All other slots, and slots whose index lies outside
 * [0, n), are (0, 0, 0, 0).
 * Inputs (device): pos as for nl_build (n x 4 float, 16-byte aligned, the
 * positions the rows were built from or any others), nbr n x capacity int32
 * and counts int32[n] as nl_build writes them.
 * Output (device): edges_out, n x capacity x 4 float32 row-major, 16-byte
 * aligned, caller-owned.  Needs no scratch and does not touch the context's
 * build state.  NULL pointers (n > 0), misalignment, n < 0 or n > 2^30,
 * capacity < 1 or a bad box are NL_ERR_ARG. */
nl_status nl_edge_features(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                           const int32_t *nbr, const int32_t *counts, int32_t capacity,
                           float *edges_out, void *stream);

/* Compressed-sparse-row form of padded rows, in two calls (the number of
 * entries is known on the device only after the first):
 *   nl_csr_offsets: row_ptr_out (device int64[n + 1]) = 0 followed by the
 *     running sum of v_i = min(max(counts[i], 0), capacity), the valid
 *     entries of row i; row_ptr_out[n] = E, all valid entries.
 *   nl_csr_fill: col_out (device int32[E]) gets the first v_i entries of
 *     row i at row_ptr[i] ..; when edges_out is not NULL (device float32
 *     [E][4], 16-byte aligned) each entry also gets its edge feature, the
 *     value nl_edge_features writes for its slot (pos and box as there).
 * nbr, counts, capacity as nl_build writes them (any rows of that shape are
 * accepted).  n > max_atoms of the context is NL_ERR_CAPACITY; NULL
 * pointers (where needed), misalignment or a bad box are NL_ERR_ARG.  The
 * offsets use the context's sort scratch, so they must not run concurrently
 * with a sort of the same context. */
nl_status nl_csr_offsets(nl_ctx *ctx, int64_t n, const int32_t *counts, int32_t capacity,
                         int64_t *row_ptr_out, void *stream);
nl_status nl_csr_fill(nl_ctx *ctx, int64_t n, const int32_t *nbr, const int32_t *counts,
                      int32_t capacity, const int64_t *row_ptr, int32_t *col_out,
                      const float *pos, const float *box, float *edges_out, void *stream);

/* Skin check (Tessera abstract: a conservative neighbor skin preserves the
 * topology across updates).  m = max over atoms of the squared minimum-image
 * displacement between `pos` and the positions of the last nl_build (raw,
 * unwrapped coordinates, same fp32 formula as above);
 * *rebuild_out = (m > fl(h*h)) with h = fl(skin * 0.5), strict.
 * rebuild_out: device int32[1]; max_d2_out: device float[1] or NULL.
 * `n` must equal the n of the last nl_build. */
nl_status nl_skin_check(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                        float skin, int32_t *rebuild_out, float *max_d2_out, void *stream);

/* One rebuild interval replayed as one CUDA Graph (Tessera abstract: each
 * rebuild interval replays as one CUDA Graph).  Runs n_steps iterations of
 *     [step_graph] -> skin check -> if rebuild: nl_build (same arguments)
 * inside a single graph launch (a conditional WHILE node around an IF node),
 * and records decisions_out[t] = 1 if iteration t rebuilt, else 0 (device
 * int32[n_steps]).  step_graph is a cudaGraph_t with the caller's per-step
 * work (it may read the iteration index from nl_step_counter); NULL means no
 * per-step work.  nl_build must have run on `pos` before (it sets the
 * reference positions).  The executable graph is cached in the context and
 * rebuilt when any argument changes. */
nl_status nl_replay(nl_ctx *ctx, void *step_graph, int32_t n_steps,
                    int64_t n, float *pos, const float *box, float cutoff, float skin,
                    int32_t capacity, int32_t *nbr, int32_t *counts,
                    int32_t *decisions_out, void *stream);

/* nl_replay with a re-sort in every rebuild (Tessera abstract: atoms are
 * kept in space-filling-curve order).  Each rebuild first permutes the atoms
 * in place into the order nl_sort_hilbert gives for their current positions
 * (stable: equal keys keep their slot order), then runs nl_build on the
 * permuted `pos`.  The same permutation is applied to ids (device int32[n],
 * e.g. initialised to 0..n-1 so that ids[k] names the atom now in slot k)
 * and to aux (device n x 4 float, 16-byte aligned, per-atom state such as
 * velocities) when they are not NULL.  nbr, counts and the skin-check
 * reference then refer to the new slots.  Other arguments, results and
 * errors as nl_replay; the step graph sees the permuted arrays at the same
 * addresses. */
nl_status nl_replay_resort(nl_ctx *ctx, void *step_graph, int32_t n_steps, int64_t n,
                           float *pos, int32_t *ids, float *aux, const float *box,
                           float cutoff, float skin, int32_t capacity, int32_t *nbr,
                           int32_t *counts, int32_t *decisions_out, void *stream);

/* Device pointer to the 0-based iteration index that nl_replay maintains
 * while its graph runs (int32[1], owned by the context). */
const int32_t *nl_step_counter(nl_ctx *ctx);

/* Synchronizes `stream`, returns the device-detected status accumulated
 * since the last call (NL_ERR_TIMEOUT, else NL_OVERFLOW, else NL_OK) and
 * clears it. */
nl_status nl_sync_status(nl_ctx *ctx, void *stream);

/* Failure-path self-test of the bounded device waits.  Every spin-wait of
 * the path (the look-back scans of the sort and the cell binning, the
 * stage barrier of the pair search) gives up after a bounded number of
 * polls and records NL_ERR_TIMEOUT in the context's status word instead of
 * hanging.  This call enqueues on `stream` one device thread that polls a
 * context word which nothing writes, under the look-back rule (a 64 ns
 * sleep between polls after the first 64), and gives up after max_polls
 * polls, recording the timeout the same way.  nl_sync_status then returns
 * NL_ERR_TIMEOUT and clears it.  Nothing else is written, so the context
 * stays usable.  max_polls outside [1, 2^22] is NL_ERR_ARG. */
nl_status nl_wait_selftest(nl_ctx *ctx, int32_t max_polls, void *stream);

/* Static, human-readable name of a status code. */
const char *nl_status_string(nl_status s);

/* Build statistics of the last nl_build (host values, no synchronization):
 * out[0..2] = cells per axis, out[3] = 1 if the staged pair-search kernel
 * was used (0 = the per-atom kernel), out[4] = cells in total. */
nl_status nl_last_build_info(nl_ctx *ctx, int64_t out[8]);

/* Curve sort that allocates nothing.  The paper has no counterpart: this
 * entry point exists for callers that cannot call cudaMalloc (code running
 * inside a framework that owns all device memory, or a plugin whose host
 * forbids allocation).  It computes exactly what nl_sort_hilbert computes,
 * with the same arguments and outputs and no context; its scratch lives in a
 * static device array inside libnl.so (about 28 MiB, held by every GPU that
 * loads the library until the process exits), which bounds n to at most
 * 2^20 = 1,048,576 atoms: larger n returns NL_ERR_CAPACITY without touching
 * the GPU.  The first call on each device looks up the array's device
 * address (with that device current; a failed lookup is retried by the next
 * call); make that first call before any stream capture.  All calls share the array, so calls whose work overlaps
 * on the GPU race; order them on one stream.  status_out (device int32[1],
 * may be NULL) receives NL_OK, or NL_ERR_TIMEOUT if a bounded device wait
 * gave up during this call. */
nl_status nl_sort_hilbert_noalloc(int64_t n, const float *pos, const float *box,
                                  int32_t *perm_out, float *pos_sorted_out, uint64_t *keys_out,
                                  int32_t *status_out, void *stream);

/* Per-kernel timing with CUDA events recorded on the call's stream.
 * nl_profile_enable(ctx, 1) starts recording; nl_profile_read synchronizes
 * the device, writes for each phase p < max_phases the summed milliseconds
 * ms_out[p] and launches launches_out[p] since the last read, and returns the
 * number of phases.  Phase names: nl_profile_phase_name. */
nl_status nl_profile_enable(nl_ctx *ctx, int on);
int32_t nl_profile_read(nl_ctx *ctx, double *ms_out, int64_t *launches_out, int32_t max_phases);
const char *nl_profile_phase_name(int32_t phase);

#ifdef __cplusplus
}
#endif

#endif /* NL_H */
