// nl_csr.cu -- compressed-sparse-row form of the padded neighbor rows.
//
// The padded [n][K] rows are the fixed-shape form (Tessera abstract: shapes
// stay fixed between rebuilds); a message-passing layer that walks edges
// wants them without the padding: row_ptr[i] = the number of valid entries
// of the rows before i, and the valid entries (the first min(counts[i], K)
// of row i) back to back.  Optionally each entry carries its edge feature
// (dx, dy, dz, r), the same values nl_edge_features writes for its slot.
//
// Offsets: a three-kernel int64 scan (block sums, one scan of the block
// sums, block-local scans), since the number of edges of a large system
// passes 2^30.  Fill: one warp per row, as the edge-feature kernel.
#include "nl_internal.cuh"

namespace nl {
namespace {

constexpr int kCsrThreads = 256;
constexpr int kCsrItems = 8;
constexpr int kCsrBlock = kCsrThreads * kCsrItems;   // rows per scan block

__device__ __forceinline__ int64_t valid_of(const int32_t *counts, int64_t i, int64_t n, int32_t K)
{
    if (i >= n) return 0;
    const int32_t c = counts[i];
    return c < 0 ? 0 : (c < K ? c : K);
}

// Inclusive scan of one value per thread over the CTA (kCsrThreads).
__device__ __forceinline__ int64_t block_scan(int64_t x, int64_t *s_warp, int64_t &total)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[w] = x;
    __syncthreads();
    int64_t before = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < kCsrThreads / 32; ++i) {
        if (i < w) before += s_warp[i];
        tot += s_warp[i];
    }
    __syncthreads();
    total = tot;
    return before + x;
}

// sums[b] = valid entries of the rows of block b.
__global__ void __launch_bounds__(kCsrThreads)
k_csr_block_sums(const int32_t *__restrict__ counts, int64_t n, int32_t K, int64_t *__restrict__ sums)
{
    __shared__ int64_t s_warp[kCsrThreads / 32];
    const int64_t base = (int64_t)blockIdx.x * kCsrBlock + (int64_t)threadIdx.x * kCsrItems;
    int64_t x = 0;
#pragma unroll
    for (int k = 0; k < kCsrItems; ++k) x += valid_of(counts, base + k, n, K);
    int64_t total = 0;
    block_scan(x, s_warp, total);
    if (threadIdx.x == 0) sums[blockIdx.x] = total;
}

// Exclusive scan of the block sums in place (one CTA, any number of blocks).
__global__ void __launch_bounds__(kCsrThreads)
k_csr_scan_sums(int64_t *__restrict__ sums, int64_t nb)
{
    __shared__ int64_t s_warp[kCsrThreads / 32];
    int64_t carry = 0;
    for (int64_t b0 = 0; b0 < nb; b0 += kCsrThreads) {
        const int64_t b = b0 + threadIdx.x;
        const int64_t v = b < nb ? sums[b] : 0;
        int64_t total = 0;
        const int64_t incl = block_scan(v, s_warp, total);
        if (b < nb) sums[b] = carry + incl - v;
        carry += total;
    }
}

// row_ptr[i] for the rows of each block, and row_ptr[n] = all entries.
__global__ void __launch_bounds__(kCsrThreads)
k_csr_offsets(const int32_t *__restrict__ counts, int64_t n, int32_t K,
              const int64_t *__restrict__ sums, int64_t *__restrict__ row_ptr)
{
    __shared__ int64_t s_warp[kCsrThreads / 32];
    const int64_t base = (int64_t)blockIdx.x * kCsrBlock + (int64_t)threadIdx.x * kCsrItems;
    int64_t v[kCsrItems];
    int64_t x = 0;
#pragma unroll
    for (int k = 0; k < kCsrItems; ++k) {
        v[k] = valid_of(counts, base + k, n, K);
        x += v[k];
    }
    int64_t total = 0;
    int64_t run = sums[blockIdx.x] + block_scan(x, s_warp, total) - x;
#pragma unroll
    for (int k = 0; k < kCsrItems; ++k) {
        if (base + k < n) row_ptr[base + k] = run;
        if (base + k == n - 1) row_ptr[n] = run + v[k];
        run += v[k];
    }
}

__device__ __forceinline__ float3 wrap3(const float4 p, float Lx, float Ly, float Lz)
{
    return make_float3(wrap_coord(p.x, Lx), wrap_coord(p.y, Ly), wrap_coord(p.z, Lz));
}

// One warp per row: the row's valid entries to col[row_ptr[i] ...] and,
// when edges is set, their features (as the edge-feature kernel).  Each lane
// issues the index loads and position gathers of kFillUnroll entries before
// it uses any.
constexpr int kFillUnroll = 8;

__global__ void __launch_bounds__(128)
k_csr_fill(int64_t n, const int32_t *__restrict__ nbr, const int32_t *__restrict__ counts,
           int32_t K, const int64_t *__restrict__ row_ptr, int32_t *__restrict__ col,
           const float4 *__restrict__ pos, float Lx, float Ly, float Lz, float4 *__restrict__ edges)
{
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += nw) {
        const int32_t c = (int32_t)valid_of(counts, i, n, K);
        const int64_t base = row_ptr[i];
        const int32_t *row = nbr + i * (int64_t)K;
        float3 wi = make_float3(0.0f, 0.0f, 0.0f);
        if (edges) wi = wrap3(__ldg(pos + i), Lx, Ly, Lz);
        for (int32_t s0 = 0; s0 < c; s0 += 32 * kFillUnroll) {
            int32_t j[kFillUnroll];
#pragma unroll
            for (int u = 0; u < kFillUnroll; ++u) {
                const int32_t s = s0 + lane + 32 * u;
                j[u] = s < c ? __ldcs(row + s) : -1;
            }
            float4 q[kFillUnroll];
#pragma unroll
            for (int u = 0; u < kFillUnroll; ++u) {
                q[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (edges && (uint64_t)(int64_t)j[u] < (uint64_t)n) q[u] = __ldg(pos + j[u]);
            }
#pragma unroll
            for (int u = 0; u < kFillUnroll; ++u) {
                const int32_t s = s0 + lane + 32 * u;
                if (s >= c) break;
                col[base + s] = j[u];
                if (edges) {
                    float4 e = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if ((uint64_t)(int64_t)j[u] < (uint64_t)n) {
                        const float3 wj = wrap3(q[u], Lx, Ly, Lz);
                        const float dx = min_image_literal(__fsub_rn(wj.x, wi.x), Lx);
                        const float dy = min_image_literal(__fsub_rn(wj.y, wi.y), Ly);
                        const float dz = min_image_literal(__fsub_rn(wj.z, wi.z), Lz);
                        e = make_float4(dx, dy, dz, __fsqrt_rn(r2_of(dx, dy, dz)));
                    }
                    __stcs(edges + base + s, e);
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_csr_offsets(nl_ctx *ctx, int64_t n, const int32_t *counts, int32_t K,
                               int64_t *row_ptr, int64_t *block_sums, cudaStream_t s)
{
    if (n <= 0) return cudaMemsetAsync(row_ptr, 0, sizeof(int64_t), s);
    const int64_t nb = (n + kCsrBlock - 1) / kCsrBlock;
    k_csr_block_sums<<<(unsigned)nb, kCsrThreads, 0, s>>>(counts, n, K, block_sums);
    NL_CUDA_TRY(cudaGetLastError());
    k_csr_scan_sums<<<1, kCsrThreads, 0, s>>>(block_sums, nb);
    NL_CUDA_TRY(cudaGetLastError());
    k_csr_offsets<<<(unsigned)nb, kCsrThreads, 0, s>>>(counts, n, K, block_sums, row_ptr);
    return cudaGetLastError();
}

int64_t csr_block_count(int64_t n) { return (n + kCsrBlock - 1) / kCsrBlock; }

cudaError_t launch_csr_fill(nl_ctx *ctx, int64_t n, const int32_t *nbr, const int32_t *counts,
                            int32_t K, const int64_t *row_ptr, int32_t *col, const float4 *pos,
                            float Lx, float Ly, float Lz, float4 *edges, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    k_csr_fill<<<resident_grid(ctx, k_csr_fill, 128, 0, (n + 3) / 4), 128, 0, s>>>(
        n, nbr, counts, K, row_ptr, col, pos, Lx, Ly, Lz, edges);
    return cudaGetLastError();
}

}  // namespace nl
