/*
 * nl_standin.h -- synthetic MD-step stand-in exported by libnl.so.
 *
 * Not part of the neighbor-list method: the pages' MD driver integrates
 * forces from a trained model, which this library does not have.  To drive
 * the skin check and the replayed rebuild interval, tests and benchmarks
 * move atoms by a seeded, counter-based displacement:
 *   u = SplitMix64(SplitMix64(seed) + ((step << 42) | (atom << 2) | axis))
 *   g = sum of the four 16-bit fields of u, minus 131070 (exact integer)
 *   delta = fl(g * A),  A = fl(sigma * sqrt(3) / 65536)   (std. dev. sigma)
 *   x <- fl(x + delta)
 * (SplitMix64: Steele, Lea & Flood, OOPSLA 2014.)  `atom` is the index in
 * the array that is moved, or ids[index] when an id array is given (it
 * follows the atoms through re-sorts); step numbers start at 1.
 */
#ifndef NL_STANDIN_H
#define NL_STANDIN_H

#include <stdint.h>
#include "nl.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Moves n atoms of `pos` (device, n x 4 floats, 4th float untouched) by the
 * displacement of step `step`, or of step (*step_dev + 1) when step_dev (a
 * device int32[1], e.g. nl_step_counter) is not NULL.  Enqueued on `stream`. */
nl_status nls_displace(int64_t n, float *pos, uint64_t seed, int64_t step,
                       const int32_t *step_dev, float sigma, void *stream);

/* Creates a cudaGraph_t holding one nls_displace launch that reads its step
 * from step_dev (device int32[1]); for use as nl_replay's step graph.  The
 * caller releases it with nls_graph_destroy. */
nl_status nls_step_graph(void **graph_out, int64_t n, float *pos, uint64_t seed,
                         const int32_t *step_dev, float sigma);
/* The same with atom = ids[slot] (device int32[n], read at each replay, so
 * it may be the id array that nl_replay_resort permutes); ids NULL is
 * nls_step_graph. */
nl_status nls_step_graph_ids(void **graph_out, int64_t n, float *pos, const int32_t *ids,
                             uint64_t seed, const int32_t *step_dev, float sigma);
void nls_graph_destroy(void *graph);

#ifdef __cplusplus
}
#endif

#endif /* NL_STANDIN_H */
