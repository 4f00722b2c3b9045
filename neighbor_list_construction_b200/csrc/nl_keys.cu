// nl_keys.cu -- curve keys, digit histograms and the final gather.
//
// Tessera abstract: atoms are sorted along a space-filling curve (a Morton
// order is the baseline it is compared against).  The curve here is the
// 3-D Hilbert curve of J. Skilling, "Programming the Hilbert curve" (AIP
// Conf. Proc. 707, 2004), on a 2^21 grid per axis, giving 63-bit keys,
// evaluated as a table-driven state machine built from that transform.
#include "nl_internal.cuh"

namespace nl {
namespace {

// Places bit k of a (k < 21) at bit 3k of the result.
__device__ __forceinline__ uint64_t spread3(uint32_t a)
{
    uint64_t x = a & 0x1fffffu;
    x = (x | (x << 32)) & 0x001f00000000ffffull;
    x = (x | (x << 16)) & 0x001f0000ff0000ffull;
    x = (x | (x << 8)) & 0x100f00f00f00f00full;
    x = (x | (x << 4)) & 0x10c30c30c30c30c3ull;
    x = (x | (x << 2)) & 0x1249249249249249ull;
    return x;
}

// Skilling's transform as a state machine.  Going down the levels, the
// axes-to-transpose step at a level only changes the bits below it (it
// inverts the low bits of axis 0, or exchanges them with those of axis 1 or
// 2, depending on the level's bits); so every lower level sees the same
// signed permutation of the three axes, fixed by the levels above.  The Gray
// code and its correction turn a level's three transposed bits into the
// key's three bits, with one carried bit: the parity of the third Gray bit
// over the levels above.  State = (signed permutation, parity): 48 are
// reachable from the identity.  A step reads one level's octant (x bit, y
// bit, z bit) and gives the key digit and the next state; the tables here
// hold one step and two steps (12 bits: next state, two digits).
struct HState {
    int pi[3];   // transposed axis i reads input axis pi[i]
    int f;       // bit i: transposed axis i is inverted
    int p;       // parity carried by the Gray correction
};

constexpr bool hstate_eq(const HState &a, const HState &b)
{
    return a.pi[0] == b.pi[0] && a.pi[1] == b.pi[1] && a.pi[2] == b.pi[2] && a.f == b.f &&
           a.p == b.p;
}

constexpr HState hstep(const HState &s, int oct, int &digit)
{
    const int a[3] = {(oct >> 2) & 1, (oct >> 1) & 1, oct & 1};
    const int v0 = a[s.pi[0]] ^ (s.f & 1);
    const int v1 = a[s.pi[1]] ^ ((s.f >> 1) & 1);
    const int v2 = a[s.pi[2]] ^ ((s.f >> 2) & 1);
    const int g0 = v0, g1 = v0 ^ v1, g2 = v0 ^ v1 ^ v2;   // Gray code of the level
    digit = ((g0 ^ s.p) << 2) | ((g1 ^ s.p) << 1) | (g2 ^ s.p);
    int pi[3] = {s.pi[0], s.pi[1], s.pi[2]};
    int f[3] = {s.f & 1, (s.f >> 1) & 1, (s.f >> 2) & 1};
    // the level's operations on the lower bits, axis 0, 1, 2 in turn
    if (v0) f[0] ^= 1;
    if (v1) {
        f[0] ^= 1;
    } else {
        const int tp = pi[0], tf = f[0];
        pi[0] = pi[1]; f[0] = f[1];
        pi[1] = tp; f[1] = tf;
    }
    if (v2) {
        f[0] ^= 1;
    } else {
        const int tp = pi[0], tf = f[0];
        pi[0] = pi[2]; f[0] = f[2];
        pi[2] = tp; f[2] = tf;
    }
    return HState{{pi[0], pi[1], pi[2]}, f[0] | (f[1] << 1) | (f[2] << 2), s.p ^ g2};
}

constexpr int kHStates = 48;

struct HilbertTables {
    uint16_t one[kHStates * 8];    // (next << 3) | digit
    uint16_t two[kHStates * 64];   // (next << 6) | (digit of the upper level << 3) | digit
};

constexpr HilbertTables make_hilbert_tables()
{
    HilbertTables t{};
    HState st[kHStates] = {};
    int ns = 1;
    st[0] = HState{{0, 1, 2}, 0, 0};
    for (int i = 0; i < ns; ++i)
        for (int o = 0; o < 8; ++o) {
            int d = 0;
            const HState n = hstep(st[i], o, d);
            int j = 0;
            while (j < ns && !hstate_eq(st[j], n)) ++j;
            if (j == ns) st[ns++] = n;   // more than kHStates would not compile
            t.one[i * 8 + o] = (uint16_t)((j << 3) | d);
        }
    for (int i = 0; i < kHStates; ++i)
        for (int o = 0; o < 64; ++o) {
            const int e1 = t.one[i * 8 + (o >> 3)];
            const int e2 = t.one[(e1 >> 3) * 8 + (o & 7)];
            t.two[i * 64 + o] = (uint16_t)(((e2 >> 3) << 6) | ((e1 & 7) << 3) | (e2 & 7));
        }
    return t;
}

__device__ const HilbertTables g_hilbert = make_hilbert_tables();

// 63-bit Hilbert key of (x, y, z) from the octants of the Morton code m:
// the top level by one step, the other 20 by two-level steps.
__device__ __forceinline__ uint64_t hilbert_index(uint64_t m, const uint16_t *one,
                                                  const uint16_t *two)
{
    uint32_t e = one[(uint32_t)(m >> 60) & 7u];   // from state 0
    uint64_t k = e & 7u;
    uint32_t s = e >> 3;
#pragma unroll
    for (int l = 19; l >= 1; l -= 2) {
        e = two[s * 64u + ((uint32_t)(m >> (3 * (l - 1))) & 63u)];
        k = (k << 6) | (e & 63u);
        s = e >> 6;
    }
    return k;
}

__device__ __forceinline__ uint64_t morton_index(uint32_t x, uint32_t y, uint32_t z)
{
    return (spread3(x) << 2) | (spread3(y) << 1) | spread3(z);
}

__device__ __forceinline__ uint32_t quantize(float w, float S)
{
    float f = floorf(__fmul_rn(w, S));
    if (!(f >= 0.0f)) return 0u;
    if (f >= 2097152.0f) return kQMax;
    uint32_t q = (uint32_t)f;
    return q > kQMax ? kQMax : q;
}

constexpr int kKeysUnroll = 2;

template <int CURVE>
__global__ void __launch_bounds__(256) k_keys(const float4 *__restrict__ pos, int64_t n,
                                              float Lx, float Ly, float Lz, float Sx,
                                              float Sy, float Sz, uint64_t *__restrict__ keys,
                                              uint32_t *__restrict__ vals,
                                              uint32_t *__restrict__ hist,
                                              const uint32_t *gate, uint32_t *zero,
                                              int64_t zero_words)
{
    // First pass: the histograms of the top kTopPasses digits, which the
    // fast sort uses.  Gated recompute (the full sort's keys): only when the
    // gate is set, with the histograms of the remaining low digits; it also
    // clears zero[0, zero_words) (the full sort's look-back status).
    const bool recompute = gate != nullptr;
    if (recompute && ld_volatile_u32(gate) == 0u) return;
    constexpr int kLow = kKeyPasses - kTopPasses;
    const int d0 = recompute ? 0 : kLow;
    const int d1 = recompute ? kLow : kKeyPasses;
    __shared__ uint32_t sh[kKeyPasses * kRadixBins];
    __shared__ uint16_t s_one[kHStates * 8];
    __shared__ uint16_t s_two[kHStates * 64];
    if (CURVE == 0) {
        for (int i = threadIdx.x; i < kHStates * 8; i += blockDim.x) s_one[i] = g_hilbert.one[i];
        for (int i = threadIdx.x; i < kHStates * 64; i += blockDim.x) s_two[i] = g_hilbert.two[i];
    }
    for (int i = threadIdx.x; i < kKeyPasses * kRadixBins; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < zero_words; i += stride)
        zero[i] = 0u;
    // kKeysUnroll atoms per thread and round: their loads first, then their
    // table walks side by side
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n;
         i0 += stride * kKeysUnroll) {
        float4 p[kKeysUnroll];
#pragma unroll
        for (int u = 0; u < kKeysUnroll; ++u)
            if (i0 + stride * u < n) p[u] = pos[i0 + stride * u];
#pragma unroll
        for (int u = 0; u < kKeysUnroll; ++u) {
            const int64_t i = i0 + stride * u;
            if (i < n) {
                const uint32_t qx = quantize(wrap_coord(p[u].x, Lx), Sx);
                const uint32_t qy = quantize(wrap_coord(p[u].y, Ly), Sy);
                const uint32_t qz = quantize(wrap_coord(p[u].z, Lz), Sz);
                const uint64_t m = morton_index(qx, qy, qz);
                const uint64_t k = CURVE == 0 ? hilbert_index(m, s_one, s_two) : m;
                keys[i] = k;
                vals[i] = (uint32_t)i;
                for (int d = d0; d < d1; ++d)
                    atomicAdd(&sh[d * kRadixBins + (uint32_t)((k >> (kRadixBits * d)) & 0xffu)],
                              1u);
            }
        }
    }
    __syncthreads();
    for (int i = d0 * kRadixBins + threadIdx.x; i < d1 * kRadixBins; i += blockDim.x) {
        const uint32_t v = sh[i];
        if (v) atomicAdd(&hist[i], v);
    }
}

// One block per digit position: exclusive scan of its 256 counts.  With a
// gate: only when the gate is set.
__global__ void __launch_bounds__(256) k_hist_scan(uint32_t *hist, const uint32_t *gate)
{
    if (gate && ld_volatile_u32(gate) == 0u) return;
    __shared__ uint32_t warp_tot[8];
    uint32_t *h = hist + blockIdx.x * kRadixBins;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const uint32_t v = h[t];
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    uint32_t before = 0;
    for (int i = 0; i < w; ++i) before += warp_tot[i];
    h[t] = before + x - v;
}

// Each thread gathers kGatherItems elements of its CTA's block, issuing all
// index loads and then all (random) position loads before any store, so a
// warp keeps several gathers in flight.
constexpr int kGatherItems = 4;

__global__ void __launch_bounds__(256)
k_gather(int64_t n, const float4 *__restrict__ pos, const int32_t *__restrict__ perm,
         float4 *__restrict__ out, const uint32_t *flags, const uint32_t *gate)
{
    if (gate && ld_volatile_u32(gate) == 0u) return;   // gated gather not needed
    if (timed_out(flags)) return;   // perm may not be a permutation
    for (int64_t base = (int64_t)blockIdx.x * (256 * kGatherItems) + threadIdx.x; base < n;
         base += (int64_t)gridDim.x * (256 * kGatherItems)) {
        int32_t i[kGatherItems];
#pragma unroll
        for (int u = 0; u < kGatherItems; ++u) {
            const int64_t k = base + 256 * u;
            i[u] = k < n ? perm[k] : -1;
        }
        float4 p[kGatherItems];
#pragma unroll
        for (int u = 0; u < kGatherItems; ++u)
            if (i[u] >= 0) p[u] = pos[i[u]];
#pragma unroll
        for (int u = 0; u < kGatherItems; ++u) {
            const int64_t k = base + 256 * u;
            if (k < n) out[k] = make_float4(p[u].x, p[u].y, p[u].z, __int_as_float(i[u]));
        }
    }
}

}  // namespace

cudaError_t launch_keys(nl_ctx *ctx, int64_t n, const float4 *pos, float Lx, float Ly, float Lz,
                        float Sx, float Sy, float Sz, int curve, cudaStream_t s,
                        const uint32_t *gate, uint32_t *zero, int64_t zero_words)
{
    if (n <= 0) return cudaSuccess;
    const int64_t want = (n + 256 * kKeysUnroll - 1) / (256 * kKeysUnroll);
    const unsigned blocks = curve == 0 ? resident_grid(ctx, k_keys<0>, 256, 0, want)
                                       : resident_grid(ctx, k_keys<1>, 256, 0, want);
    if (curve == 0)
        k_keys<0><<<(unsigned)blocks, 256, 0, s>>>(pos, n, Lx, Ly, Lz, Sx, Sy, Sz, ctx->keys[0],
                                                    ctx->vals[0], ctx->hist, gate, zero,
                                                    zero_words);
    else
        k_keys<1><<<(unsigned)blocks, 256, 0, s>>>(pos, n, Lx, Ly, Lz, Sx, Sy, Sz, ctx->keys[0],
                                                    ctx->vals[0], ctx->hist, gate, zero,
                                                    zero_words);
    return cudaGetLastError();
}

cudaError_t launch_hist_scan(nl_ctx *ctx, cudaStream_t s, const uint32_t *gate)
{
    // ungated: all digits (the low ones are still zero); gated: the low ones
    const int digits = gate ? kKeyPasses - kTopPasses : kKeyPasses;
    k_hist_scan<<<digits, kRadixBins, 0, s>>>(ctx->hist, gate);
    return cudaGetLastError();
}

cudaError_t launch_gather(nl_ctx *ctx, int64_t n, const float4 *pos, const int32_t *perm,
                          float4 *out, const uint32_t *flags, cudaStream_t s, const uint32_t *gate)
{
    if (n <= 0) return cudaSuccess;
    const int64_t want = (n + 256 * kGatherItems - 1) / (256 * kGatherItems);
    // gated: one resident wave, so a clear gate costs few CTAs
    const unsigned blocks = gate ? resident_grid(ctx, k_gather, 256, 0, want) : (unsigned)want;
    k_gather<<<blocks, 256, 0, s>>>(n, pos, perm, out, flags, gate);
    return cudaGetLastError();
}

}  // namespace nl
