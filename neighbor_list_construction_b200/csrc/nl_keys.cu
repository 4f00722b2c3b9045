// nl_keys.cu -- curve keys, digit histograms and the final gather.
//
// Tessera abstract: atoms are sorted along a space-filling curve (a Morton
// order is the baseline it is compared against).  The curve here is the
// 3-D Hilbert curve of J. Skilling, "Programming the Hilbert curve" (AIP
// Conf. Proc. 707, 2004), on a 2^21 grid per axis, giving 63-bit keys.
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

// Skilling's axes-to-transpose transform for three 21-bit axes, then the
// transposed index read level by level (x first in each triple).
__device__ __forceinline__ uint64_t hilbert_index(uint32_t x, uint32_t y, uint32_t z)
{
#pragma unroll
    for (int l = kQBits - 1; l >= 1; --l) {
        const uint32_t Q = 1u << l;
        const uint32_t P = Q - 1u;
        // axis 0 against itself: the exchange is empty, only the inversion
        x ^= (x & Q) ? P : 0u;
        // axis 1: invert the low bits of x, or exchange them with y's
        uint32_t t = (x ^ y) & P;
        if (y & Q) {
            x ^= P;
        } else {
            x ^= t;
            y ^= t;
        }
        // axis 2
        t = (x ^ z) & P;
        if (z & Q) {
            x ^= P;
        } else {
            x ^= t;
            z ^= t;
        }
    }
    // Gray encode
    y ^= x;
    z ^= y;
    // bit k of the correction = parity of z's bits at levels k+1 .. 20
    uint32_t t = (z & ~1u) >> 1;
    t ^= t >> 1;
    t ^= t >> 2;
    t ^= t >> 4;
    t ^= t >> 8;
    t ^= t >> 16;
    x ^= t;
    y ^= t;
    z ^= t;
    return (spread3(x) << 2) | (spread3(y) << 1) | spread3(z);
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

template <int CURVE>
__global__ void __launch_bounds__(256) k_keys(const float4 *__restrict__ pos, int64_t n,
                                              float Lx, float Ly, float Lz, float Sx,
                                              float Sy, float Sz, uint64_t *__restrict__ keys,
                                              uint32_t *__restrict__ vals,
                                              uint32_t *__restrict__ hist,
                                              const uint32_t *gate)
{
    // First pass: the histograms of the top kTopPasses digits, which the
    // fast sort uses.  Gated recompute (the full sort's keys): only when the
    // gate is set, with the histograms of the remaining low digits.
    const bool recompute = gate != nullptr;
    if (recompute && ld_volatile_u32(gate) == 0u) return;
    constexpr int kLow = kKeyPasses - kTopPasses;
    const int d0 = recompute ? 0 : kLow;
    const int d1 = recompute ? kLow : kKeyPasses;
    __shared__ uint32_t sh[kKeyPasses * kRadixBins];
    for (int i = threadIdx.x; i < kKeyPasses * kRadixBins; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float4 p = pos[i];
        const uint32_t qx = quantize(wrap_coord(p.x, Lx), Sx);
        const uint32_t qy = quantize(wrap_coord(p.y, Ly), Sy);
        const uint32_t qz = quantize(wrap_coord(p.z, Lz), Sz);
        const uint64_t k = CURVE == 0 ? hilbert_index(qx, qy, qz) : morton_index(qx, qy, qz);
        keys[i] = k;
        vals[i] = (uint32_t)i;
        for (int d = d0; d < d1; ++d)
            atomicAdd(&sh[d * kRadixBins + (uint32_t)((k >> (kRadixBits * d)) & 0xffu)], 1u);
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

__global__ void k_gather(int64_t n, const float4 *__restrict__ pos, const int32_t *__restrict__ perm,
                         float4 *__restrict__ out)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride) {
        const int32_t i = perm[k];
        const float4 p = pos[i];
        out[k] = make_float4(p.x, p.y, p.z, __int_as_float(i));
    }
}

}  // namespace

cudaError_t launch_keys(nl_ctx *ctx, int64_t n, const float4 *pos, float Lx, float Ly, float Lz,
                        float Sx, float Sy, float Sz, int curve, cudaStream_t s,
                        const uint32_t *gate)
{
    if (n <= 0) return cudaSuccess;
    const int64_t want = (n + 255) / 256;
    const unsigned blocks = curve == 0 ? resident_grid(ctx, k_keys<0>, 256, 0, want)
                                       : resident_grid(ctx, k_keys<1>, 256, 0, want);
    if (curve == 0)
        k_keys<0><<<(unsigned)blocks, 256, 0, s>>>(pos, n, Lx, Ly, Lz, Sx, Sy, Sz, ctx->keys[0],
                                                    ctx->vals[0], ctx->hist, gate);
    else
        k_keys<1><<<(unsigned)blocks, 256, 0, s>>>(pos, n, Lx, Ly, Lz, Sx, Sy, Sz, ctx->keys[0],
                                                    ctx->vals[0], ctx->hist, gate);
    return cudaGetLastError();
}

cudaError_t launch_hist_scan(nl_ctx *ctx, cudaStream_t s, const uint32_t *gate)
{
    // ungated: all digits (the low ones are still zero); gated: the low ones
    const int digits = gate ? kKeyPasses - kTopPasses : kKeyPasses;
    k_hist_scan<<<digits, kRadixBins, 0, s>>>(ctx->hist, gate);
    return cudaGetLastError();
}

cudaError_t launch_gather(int64_t n, const float4 *pos, const int32_t *perm, float4 *out,
                          cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 65535 * 8) blocks = 65535 * 8;
    k_gather<<<(unsigned)blocks, 256, 0, s>>>(n, pos, perm, out);
    return cudaGetLastError();
}

}  // namespace nl
