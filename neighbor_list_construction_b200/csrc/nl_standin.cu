// nl_standin.cu -- synthetic displacement that stands in for an MD step.
//
// Not part of the neighbor-list method (see include/nl_standin.h): it only
// moves atoms so that the skin check and the replayed interval have work.
#include <cmath>

#include "nl_internal.cuh"
#include "nl_standin.h"

namespace {

// SplitMix64 output function for one 64-bit counter (Steele, Lea & Flood 2014).
__device__ __forceinline__ uint64_t splitmix64(uint64_t x)
{
    uint64_t z = x + 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

// The atom of slot k is ids[k] when ids is given (so that a re-sort does not
// change which random stream moves which atom), else k.
__global__ void k_displace(int64_t n, float *__restrict__ pos, const int32_t *__restrict__ ids,
                           uint64_t seed_mix, int64_t step, const int32_t *__restrict__ step_dev,
                           float A)
{
    const int64_t t = step_dev ? (int64_t)(*step_dev) + 1 : step;
    const int64_t total = 3 * n;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
        const int64_t slot = e / 3;
        const int axis = (int)(e - slot * 3);
        const int64_t atom = ids ? (int64_t)ids[slot] : slot;
        const uint64_t ctr = ((uint64_t)t << 42) | ((uint64_t)atom << 2) | (uint64_t)axis;
        const uint64_t u = splitmix64(seed_mix + ctr);
        const int32_t g = (int32_t)(u & 0xffffu) + (int32_t)((u >> 16) & 0xffffu) +
                          (int32_t)((u >> 32) & 0xffffu) + (int32_t)(u >> 48) - 131070;
        float *x = pos + slot * 4 + axis;
        *x = __fadd_rn(*x, __fmul_rn((float)g, A));
    }
}

uint64_t host_splitmix64(uint64_t x)
{
    uint64_t z = x + 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

unsigned blocks_for(int64_t n)
{
    int64_t b = (3 * n + 255) / 256;
    if (b < 1) b = 1;
    if (b > 148 * 16) b = 148 * 16;
    return (unsigned)b;
}

}  // namespace

extern "C" {

nl_status nls_displace(int64_t n, float *pos, uint64_t seed, int64_t step,
                       const int32_t *step_dev, float sigma, void *stream)
{
    if (n < 0 || (n > 0 && !pos) || !std::isfinite(sigma)) return NL_ERR_ARG;
    if (n == 0) return NL_OK;
    const float A = (float)((double)sigma * std::sqrt(3.0) / 65536.0);
    k_displace<<<blocks_for(n), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        n, pos, nullptr, host_splitmix64(seed), step, step_dev, A);
    return cudaGetLastError() == cudaSuccess ? NL_OK : NL_ERR_CUDA;
}

nl_status nls_step_graph(void **graph_out, int64_t n, float *pos, uint64_t seed,
                         const int32_t *step_dev, float sigma)
{
    return nls_step_graph_ids(graph_out, n, pos, nullptr, seed, step_dev, sigma);
}

nl_status nls_step_graph_ids(void **graph_out, int64_t n, float *pos, const int32_t *ids,
                             uint64_t seed, const int32_t *step_dev, float sigma)
{
    if (!graph_out || !step_dev || n <= 0 || !pos) return NL_ERR_ARG;
    *graph_out = nullptr;
    const float A = (float)((double)sigma * std::sqrt(3.0) / 65536.0);
    uint64_t mix = host_splitmix64(seed);
    int64_t step0 = 0;
    void *args[] = {(void *)&n, (void *)&pos, (void *)&ids, (void *)&mix, (void *)&step0,
                    (void *)&step_dev, (void *)&A};
    cudaGraph_t g = nullptr;
    if (cudaGraphCreate(&g, 0) != cudaSuccess) return NL_ERR_CUDA;
    cudaKernelNodeParams p = {};
    p.func = (void *)k_displace;
    p.gridDim = dim3(blocks_for(n));
    p.blockDim = dim3(256);
    p.kernelParams = args;
    cudaGraphNode_t node;
    if (cudaGraphAddKernelNode(&node, g, nullptr, 0, &p) != cudaSuccess) {
        cudaGraphDestroy(g);
        return NL_ERR_CUDA;
    }
    *graph_out = g;
    return NL_OK;
}

void nls_graph_destroy(void *graph)
{
    if (graph) cudaGraphDestroy(reinterpret_cast<cudaGraph_t>(graph));
}

}  // extern "C"
