/*
 * nl_shard.h -- halo selection for equal-count shards along the curve.
 *
 * Tessera abstract: the atoms are sorted along a space-filling curve and
 * cut into equal-count shards, one per GPU, each of which needs the atoms
 * within the search radius of its own (its halo) to build its rows.  These
 * calls find, per rank, which of its atoms every other rank needs; moving
 * them between GPUs (all-reduce, all-to-all) is left to the caller's
 * communicator (NCCL through torch.distributed in the Python layer).
 *
 * Conventions
 *   pos        device, n x 4 float32, 16-byte aligned; the fourth float of
 *              each atom holds its global id (int32 bits), which travels
 *              with the atom and names it in the final rows.
 *   dims       host int32[3]: the coarse periodic grid from nl_halo_grid
 *              (cells wider than rl = cutoff + skin, at most 1024 a side).
 *   occ, need  device int32[dims[0] * dims[1] * dims[2]], caller-owned.
 *   ranks      1 <= nranks <= 32, 0 <= rank < nranks.
 *   errors     NL_ERR_ARG for NULL pointers, misalignment or bad sizes;
 *              NL_ERR_CUDA if a launch fails.  No call synchronizes.
 * The steps, per rank: nl_halo_mark -> sum of all ranks' occ (all-reduce;
 * the rank bits are distinct, so the sum is their or) -> nl_halo_needed ->
 * nl_halo_count -> exchange counts -> nl_halo_fill_blocks -> all-to-all of
 * the fixed blocks -> nl_halo_pack -> nl_build_rows_dev on [own atoms;
 * received halo] with n_rows = own atoms -> nl_map_ids.  No step needs a
 * count on the host.  (nl_halo_fill with exact offsets remains for callers
 * that size the exchange on the host.)
 */
#ifndef NL_SHARD_H
#define NL_SHARD_H

#include <stdint.h>
#include "nl.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The coarse grid (host): per axis floor(L / (rl (1 + 2^-10) + L 2^-16)),
 * clamped to [1, 1024], so two atoms within rl lie in the same or adjacent
 * cells (periodically) whatever the fp32 rounding of the cell assignment. */
nl_status nl_halo_grid(const float *box, float cutoff, float skin, int32_t dims_out[3]);

/* occ_out[c] = 1 << rank for every coarse cell c holding one of the n atoms
 * of pos, 0 elsewhere (the array is cleared first). */
nl_status nl_halo_mark(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                       const int32_t dims[3], int32_t rank, int32_t *occ_out, void *stream);

/* need_out[c] = bitwise or of occ_all over the 27 cells around c (periodic),
 * occ_all being the sum over ranks of their nl_halo_mark outputs. */
nl_status nl_halo_needed(nl_ctx *ctx, const float *box, const int32_t dims[3],
                         const int32_t *occ_all, int32_t *need_out, void *stream);

/* counts_out[q] (device int32[nranks], cleared first) = number of this
 * rank's atoms whose coarse cell c has bit q set in need[c], q != rank. */
nl_status nl_halo_count(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                        const int32_t dims[3], const int32_t *need, int32_t rank, int32_t nranks,
                        int32_t *counts_out, void *stream);

/* Writes those atoms (their float4 as in pos) to send_out (device, 16-byte
 * aligned, sum(counts) x 4 float32): the atoms for rank q at
 * offsets[q] .. offsets[q] + counts[q] - 1, in no particular order.  offsets
 * and counts are device int32[nranks] (counts from nl_halo_count on the same
 * inputs), cursor is device int32[nranks] scratch.  send_out may be NULL
 * when every count is 0. */
nl_status nl_halo_fill(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                       const int32_t dims[3], const int32_t *need, int32_t rank, int32_t nranks,
                       const int32_t *offsets, const int32_t *counts, int32_t *cursor,
                       float *send_out, void *stream);

/* nl_halo_fill into fixed blocks, so that nothing on the host depends on
 * the counts: the atoms for rank q go to send_out[q * block ..], at most
 * `block` of them (send_out: device, 16-byte aligned, nranks * block x 4
 * float32; the blocks are exchanged by an all-to-all of equal splits).  A
 * count above `block` drops the excess and makes nl_sync_status report
 * NL_ERR_HALO.  block < 1 or a NULL buffer is NL_ERR_ARG. */
nl_status nl_halo_fill_blocks(nl_ctx *ctx, int64_t n, const float *pos, const float *box,
                              const int32_t dims[3], const int32_t *need, int32_t rank,
                              int32_t nranks, int32_t block, const int32_t *counts,
                              int32_t *cursor, float *send_out, void *stream);

/* Appends the halo received as fixed blocks to the own atoms, on the device:
 * recv (device, nranks * block x 4 float32) holds in block q the
 * min(recv_counts[q], block) atoms rank q sent (recv_counts: device
 * int32[nranks], the all-to-all of the senders' counts); they are written
 * to pos_all after its first n_own (own) atoms, block after block, and the
 * total atom count to *n_all_out (device int64), clamped to n_max (pos_all
 * holds room for n_max atoms).  A count above `block` or a total above
 * n_max makes nl_sync_status report NL_ERR_HALO.  The count is meant for
 * nl_build_rows_dev. */
nl_status nl_halo_pack(nl_ctx *ctx, int32_t nranks, int32_t block, const int32_t *recv_counts,
                       const float *recv, int64_t n_own, int64_t n_max, float *pos_all,
                       int64_t *n_all_out, void *stream);

/* In place: every entry j >= 0 of the n_rows x capacity rows nbr (indices
 * into pos_all, n_all atoms) becomes the global id in pos_all[j]'s fourth
 * float; -1 stays.  counts (device int32[n_rows], the build's) may be NULL;
 * given, only the first min(counts[i], capacity) entries of row i are read,
 * which is all a build writes before its -1 padding. */
nl_status nl_map_ids(nl_ctx *ctx, int64_t n_rows, int32_t capacity, int32_t *nbr,
                     const int32_t *counts, int64_t n_all, const float *pos_all, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NL_SHARD_H */
