// nl_device.cuh -- constants, the cell grid and the device helpers of the
// libnl kernels (the arithmetic every kernel shares).
//
// Internal to libnl.so; the public C ABI is include/nl.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nl {

// ----------------------------------------------------------------- constants
constexpr int kQBits = 21;                    // bits per axis of the curve grid
constexpr uint32_t kQMax = (1u << kQBits) - 1u;
constexpr int kRadixBits = 8;                 // LSD digit width
constexpr int kRadixBins = 1 << kRadixBits;
constexpr int kKeyPasses = 8;                 // 63-bit keys: 8 digits of 8 bits
constexpr int kTopPasses = 3;                 // fast path: the top digits (bits 40..63)
constexpr int kStatusPasses = kKeyPasses + kTopPasses;   // look-back status slots
constexpr int kPrefixShift = 8 * (kKeyPasses - kTopPasses);  // key >> this = sorted prefix
constexpr int kRunMax = 64;                   // longest prefix run the run finish takes

// Onesweep tile: 256 threads x 8 keys.
constexpr int kSortThreads = 256;
constexpr int kSortItems = 12;
constexpr int kSortTile = kSortThreads * kSortItems;

// Cell-count scan tile: 256 threads x 16 cells.
constexpr int kScanThreads = 256;
constexpr int kScanItems = 16;
constexpr int kScanTile = kScanThreads * kScanItems;

// Look-back status words: 2 flag bits over a 30-bit count.
constexpr uint32_t kStAggregate = 1u << 30;
constexpr uint32_t kStPrefix = 2u << 30;
constexpr uint32_t kStValue = (1u << 30) - 1u;
// Polls of one status word before a bounded wait gives up.
constexpr uint32_t kSpinLimit = 1u << 22;

// Device-detected conditions, accumulated in ctx->flags.
constexpr uint32_t kFlagOverflow = 1u;
constexpr uint32_t kFlagTimeout = 2u;
constexpr uint32_t kFlagHalo = 4u;       // a halo block or buffer was too small

enum Phase {
    PH_KEYS = 0,
    PH_KEY_SCAN,
    PH_SORT,
    PH_GATHER,
    PH_BIN_COUNT,
    PH_CELL_SCAN,
    PH_BIN_SCATTER,
    PH_CELL_SORT,
    PH_PAIRS,
    PH_PAIRS_LISTED,
    PH_SKIN,
    PH_EDGES,
    PH_COUNT
};

// Cell grid of one build, all values computed on the host.
struct CellGrid {
    int nx, ny, nz;          // cells per axis
    float Lx, Ly, Lz;        // box
    float Tx, Ty, Tz;        // fl(n_a / L_a): cell coordinate = floor(w * T)
    float rl2;               // fl(rl * rl)
    int64_t ncell;
    int wy, wz;              // stencil half-width in y and z (x is always 1)
    int literal;             // 1: literal minimum image (small boxes)
    int64_t n_rows;          // rows are written for atoms of index < n_rows only
    const int64_t *n_dev;    // when set: the atom count, read on the device (at most n)
};

// Atoms of a build: n, or the device-side count when the grid carries one.
__device__ __forceinline__ int64_t atoms_of(const CellGrid &g, int64_t n)
{
    if (!g.n_dev) return n;
    const int64_t d = *g.n_dev;
    return d < 0 ? 0 : (d < n ? d : n);
}


// ------------------------------------------------------- device helpers
__device__ __forceinline__ float wrap_coord(float x, float L)
{
    // w = x - L*floor(x/L), one fold into [0, L), else 0.
    // For 0 < x <= fl_down(L*(1 - 2^-23)) the quotient x/L rounds to a float
    // below 1, so t = 0 and w = fl(x - 0) = x: the same bits without the
    // division (zeros take the full path, which maps -0 to +0).
    if (x > 0.0f && x <= __fmul_rd(L, 0.99999988f)) return x;
    float t = floorf(__fdiv_rn(x, L));
    float w = __fsub_rn(x, __fmul_rn(L, t));
    if (w < 0.0f) w = __fadd_rn(w, L);
    if (w >= L) w = __fsub_rn(w, L);
    if (!(w >= 0.0f && w < L)) w = 0.0f;
    return w;
}

// Literal minimum image d - L*rintf(d/L).
__device__ __forceinline__ float min_image_literal(float d, float L)
{
    float r = rintf(__fdiv_rn(d, L));
    return __fsub_rn(d, __fmul_rn(L, r));
}

__device__ __forceinline__ float r2_of(float dx, float dy, float dz)
{
    return __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)), __fmul_rn(dz, dz));
}

__device__ __forceinline__ int cell_coord(float w, float T, int n)
{
    float f = floorf(__fmul_rn(w, T));
    int c = f >= 0.0f ? (int)f : 0;
    return c < n ? c : n - 1;
}

__device__ __forceinline__ uint32_t ld_volatile_u32(const uint32_t *p)
{
    return *(const volatile uint32_t *)p;
}

__device__ __forceinline__ void st_volatile_u32(uint32_t *p, uint32_t v)
{
    *(volatile uint32_t *)p = v;
}

// True once a bounded wait has given up (kFlagTimeout in the status word).
// A look-back pass that gives up goes on with a partial prefix, so its output
// is not a permutation (sort) or its cell starts are not monotonic (binning).
// Every kernel that consumes such output checks this at entry and returns,
// so a partial prefix never becomes an index, an address or a copy size.
// The bit stays set until nl_sync_status reads and clears it.
__device__ __forceinline__ bool timed_out(const uint32_t *flags)
{
    return (ld_volatile_u32(flags) & kFlagTimeout) != 0u;
}

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace nl
