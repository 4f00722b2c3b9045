// nl_skin.cu -- max-displacement reduction (the skin check).
//
// Tessera abstract: a conservative neighbor skin preserves topology across
// updates, so the list is rebuilt only when some atom may have crossed the
// skin.  Reading: rebuild when max_i |x_i - ref_i|^2 (minimum image, fp32 as
// in the pair predicate) exceeds fl(h*h), h = fl(skin/2).  The max of
// non-negative floats is exact, so the reduction order does not matter; it is
// taken on the float bit patterns with atomicMax, and the last CTA to finish
// (by ticket) publishes the decision and resets the accumulator.
#include "nl_internal.cuh"

namespace nl {
namespace {

__global__ void __launch_bounds__(256)
k_skin(const float4 *__restrict__ pos, const float4 *__restrict__ ref, int64_t n, float Lx,
       float Ly, float Lz, float h2, uint32_t *acc, int32_t *rebuild_out, float *max_out,
       int32_t *decisions, const int32_t *step, unsigned long long cond)
{
    __shared__ float s_wmax[8];
    __shared__ bool s_last;
    float m = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float4 a = ref[i];
        const float4 b = pos[i];
        const float dx = min_image_literal(__fsub_rn(b.x, a.x), Lx);
        const float dy = min_image_literal(__fsub_rn(b.y, a.y), Ly);
        const float dz = min_image_literal(__fsub_rn(b.z, a.z), Lz);
        const float r2 = r2_of(dx, dy, dz);
        if (r2 > m) m = r2;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float y = __shfl_xor_sync(0xffffffffu, m, o);
        if (y > m) m = y;
    }
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (lane == 0) s_wmax[w] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float bm = 0.0f;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i)
            if (s_wmax[i] > bm) bm = s_wmax[i];
        if (bm > 0.0f) atomicMax(&acc[0], __float_as_uint(bm));
        __threadfence();
        s_last = atomicAdd(&acc[1], 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (s_last && threadIdx.x == 0) {
        __threadfence();
        const float mx = __uint_as_float(atomicAdd(&acc[0], 0u));
        const int32_t rb = mx > h2 ? 1 : 0;
        rebuild_out[0] = rb;
        if (max_out) max_out[0] = mx;
        if (decisions) decisions[*step] = rb;
        if (cond) cudaGraphSetConditional((cudaGraphConditionalHandle)cond, (unsigned)rb);
        acc[0] = 0u;
        acc[1] = 0u;
        __threadfence();
    }
}

}  // namespace

cudaError_t launch_skin(nl_ctx *ctx, int64_t n, const float4 *pos, float Lx, float Ly, float Lz,
                        float h2, int32_t *rebuild_out, float *max_d2_out, int32_t *decisions,
                        const int32_t *step, unsigned long long cond, cudaStream_t s)
{
    ProfScope ps(ctx, PH_SKIN, s);
    const unsigned blocks = resident_grid(ctx, k_skin, 256, 0, (n + 255) / 256);
    k_skin<<<(unsigned)blocks, 256, 0, s>>>(pos, ctx->ref, n, Lx, Ly, Lz, h2, ctx->skin_acc,
                                            rebuild_out, max_d2_out, decisions, step, cond);
    return cudaGetLastError();
}

}  // namespace nl
