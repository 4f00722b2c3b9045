// nl_edges.cu -- per-slot edge features of the padded neighbor rows.
//
// Tessera abstract (and the page on batching and kernel fusion): the
// message-passing layers consume the neighbor topology as dense, padded
// tensors.  For row i and slot s < min(counts[i], K) with j = nbr[i][s] the
// feature is (dx, dy, dz, r): the minimum-image displacement w_j - w_i of
// the wrapped coordinates, per axis d - L*rintf(d/L), and r = sqrt_rn of
// (dx*dx + dy*dy) + dz*dz -- the same fp32 values that decided membership.
// Every other slot, and a slot whose index lies outside [0, n), is zero.
//
// The kernel streams: each row is read once (index entries of the valid
// prefix only) and its K float4 features are written once with
// evict-first stores, so the positions gathered for the neighbors keep L2.
// One warp per row, lanes over slots: 128-byte index reads and 512-byte
// feature writes per warp instruction, both fully coalesced.  Each lane
// issues the index loads and position gathers of 8 slots before using any,
// so a warp keeps 8 dependent load chains in flight instead of one.
#include "nl_internal.cuh"

namespace nl {
namespace {

__device__ __forceinline__ float3 wrap3(const float4 p, float Lx, float Ly, float Lz)
{
    return make_float3(wrap_coord(p.x, Lx), wrap_coord(p.y, Ly), wrap_coord(p.z, Lz));
}

constexpr int kEdgeUnroll = 8;   // slots per lane in flight: 256 per warp

__global__ void __launch_bounds__(128)
k_edge_features(const float4 *__restrict__ pos, int64_t n, float Lx, float Ly, float Lz,
                const int32_t *__restrict__ nbr, const int32_t *__restrict__ counts, int32_t K,
                float4 *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += nw) {
        int32_t c = __ldg(counts + i);
        c = c < K ? c : K;
        const float3 wi = wrap3(__ldg(pos + i), Lx, Ly, Lz);
        const int32_t *row = nbr + i * (int64_t)K;
        float4 *o = out + i * (int64_t)K;
        for (int32_t base = 0; base < K; base += 32 * kEdgeUnroll) {
            // all index loads of the chunk, then all position gathers, then
            // the arithmetic and stores: kEdgeUnroll independent chains per lane
            int32_t j[kEdgeUnroll];
#pragma unroll
            for (int u = 0; u < kEdgeUnroll; ++u) {
                const int32_t s = base + lane + 32 * u;
                j[u] = s < c ? __ldcs(row + s) : -1;
            }
            float4 q[kEdgeUnroll];
#pragma unroll
            for (int u = 0; u < kEdgeUnroll; ++u) {
                q[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if ((uint64_t)(int64_t)j[u] < (uint64_t)n) q[u] = __ldg(pos + j[u]);
            }
#pragma unroll
            for (int u = 0; u < kEdgeUnroll; ++u) {
                const int32_t s = base + lane + 32 * u;
                if (s >= K) break;
                float4 e = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if ((uint64_t)(int64_t)j[u] < (uint64_t)n) {
                    const float3 wj = wrap3(q[u], Lx, Ly, Lz);
                    const float dx = min_image_literal(__fsub_rn(wj.x, wi.x), Lx);
                    const float dy = min_image_literal(__fsub_rn(wj.y, wi.y), Ly);
                    const float dz = min_image_literal(__fsub_rn(wj.z, wi.z), Lz);
                    e = make_float4(dx, dy, dz, __fsqrt_rn(r2_of(dx, dy, dz)));
                }
                __stcs(o + s, e);
            }
        }
    }
}

}  // namespace

cudaError_t launch_edge_features(nl_ctx *ctx, int64_t n, const float4 *pos, float Lx, float Ly,
                                 float Lz, const int32_t *nbr, const int32_t *counts, int32_t K,
                                 float4 *out, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    ProfScope ps(ctx, PH_EDGES, s);
    // one resident wave of CTAs; the warps stride over rows
    if (ctx->edge_blocks_per_sm == 0) {   // per context, so per device
        int per_sm = 0;
        NL_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_edge_features, 128, 0));
        ctx->edge_blocks_per_sm = per_sm < 1 ? 1 : per_sm;
    }
    const int per_sm = ctx->edge_blocks_per_sm;
    int64_t blocks = (n + 3) / 4;
    const int64_t cap = (int64_t)ctx->sm_count * per_sm;
    if (blocks > cap) blocks = cap;
    k_edge_features<<<(unsigned)blocks, 128, 0, s>>>(pos, n, Lx, Ly, Lz, nbr, counts, K, out);
    return cudaGetLastError();
}

}  // namespace nl
