// nl_sort.cu -- sort of (63-bit key, 32-bit index) pairs: onesweep LSD radix
// passes, and a prefix-run finish.
//
// Fast path: the three most significant 8-bit digits (bits 40..63) by
// onesweep passes; the array is then ordered by its 24-bit key prefix, with
// equal prefixes in index order.  A prefix is one cell of a 256^3 grid over
// the box, so a run of equal prefixes holds about n / 2^24 keys (a handful
// at most for atoms at liquid density); each element of a run is placed by
// its rank in (key, index) within the run.  A run longer than kRunMax keys
// (strongly clustered input) sets a gate word, and a gated copy of the full
// eight-pass sort, already enqueued behind, then recomputes the keys and
// redoes the whole order; when the gate is clear those launches return at
// once.
//
// One kernel launch per 8-bit digit, one resident wave of CTAs.  A CTA takes
// tiles of kSortTile keys from an atomic ticket until none is left (so a tile
// only ever waits on tiles whose CTAs are already running), ranks each
// tile's keys stably with warp match/popc, publishes its per-digit counts,
// and finds the counts of all earlier tiles by decoupled look-back over
// per-(tile, digit) status words.  The global digit starts come from
// histograms made by the key kernel (those of the low digits only by its
// gated recompute).  Waits on a status word are bounded: past kSpinLimit
// polls the kernel records kFlagTimeout and carries on, so a stuck
// predecessor cannot hang the device; every later pass, the run finish and
// the gather then return at entry (timed_out).
#include "nl_internal.cuh"

namespace nl {
namespace {

constexpr int kWarps = kSortThreads / 32;
constexpr int kLookBack = 8;   // predecessor status words read per look-back round
constexpr size_t kSortDynSmem = (size_t)kSortTile * (sizeof(uint64_t) + sizeof(uint32_t));

template <bool WRITE_KEYS>
__global__ void __launch_bounds__(kSortThreads, 3)
k_onesweep(const uint64_t *__restrict__ keys_in, const uint32_t *__restrict__ vals_in,
           uint64_t *__restrict__ keys_out, uint32_t *__restrict__ vals_out, int64_t n,
           int shift, const uint32_t *__restrict__ digit_start, uint32_t *status,
           uint32_t *ticket, uint32_t *flags, const uint32_t *gate)
{
    if (gate && ld_volatile_u32(gate) == 0u) return;   // gated pass not needed
    // an earlier wait gave up (a CTA of this pass may set the bit while
    // others start: one decision per CTA)
    if (__syncthreads_or(timed_out(flags))) return;
    extern __shared__ __align__(16) unsigned char sort_smem[];
    uint64_t *s_keys = reinterpret_cast<uint64_t *>(sort_smem);
    uint32_t *s_vals = reinterpret_cast<uint32_t *>(sort_smem + sizeof(uint64_t) * kSortTile);
    __shared__ uint32_t s_whist[kWarps][kRadixBins];  // per-warp counts -> prefixes
    __shared__ uint32_t s_tdig[kRadixBins];           // digit start inside the tile
    __shared__ uint32_t s_gbase[kRadixBins];          // global start of digit in tile
    __shared__ uint32_t s_wtot[kWarps];
    __shared__ uint32_t s_tile;

    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int64_t ntiles = (n + kSortTile - 1) / kSortTile;
    for (;;) {   // tiles by ticket until none is left
        if (t == 0) s_tile = atomicAdd(ticket, 1u);
        for (int i = t; i < kWarps * kRadixBins; i += kSortThreads) (&s_whist[0][0])[i] = 0u;
        __syncthreads();
        const uint32_t tile = s_tile;
        if ((int64_t)tile >= ntiles) return;
        const int64_t base = (int64_t)tile * kSortTile;

        // warp w owns elements [base + Ew, base + Ew + E), E = 32 kSortItems; item
        // k of lane l is element base + Ew + 32k + l, so (k, lane) order is index
        // order.
        uint64_t key[kSortItems];
        uint32_t val[kSortItems];
        uint32_t rank[kSortItems];
#pragma unroll
        for (int k = 0; k < kSortItems; ++k) {
            const int64_t idx = base + (int64_t)w * (32 * kSortItems) + k * 32 + lane;
            if (idx < n) {
                key[k] = keys_in[idx];
                val[k] = vals_in[idx];
            } else {
                key[k] = ~0ull;  // digit 255 in every pass, never written
                val[k] = 0u;
            }
        }
        const uint32_t lt = lanemask_lt();
#pragma unroll
        for (int k = 0; k < kSortItems; ++k) {
            const int64_t idx = base + (int64_t)w * (32 * kSortItems) + k * 32 + lane;
            const uint32_t d = idx < n ? (uint32_t)(key[k] >> shift) & 0xffu : 0x100u;
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            const int leader = __ffs(peers) - 1;
            uint32_t before = 0u;
            if (lane == leader && d < 0x100u) {
                before = s_whist[w][d];
                s_whist[w][d] = before + __popc(peers);
            }
            before = __shfl_sync(0xffffffffu, before, leader);
            rank[k] = before + __popc(peers & lt);
            __syncwarp();
        }
        __syncthreads();

        // thread t now owns digit t
        uint32_t cnt = 0u;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) {
            const uint32_t c = s_whist[ww][t];
            s_whist[ww][t] = cnt;
            cnt += c;
        }
        uint32_t *st = status + (size_t)tile * kRadixBins + t;
        uint32_t excl = 0u;
        if (tile == 0) {
            st_volatile_u32(st, kStPrefix | cnt);
        } else {
            st_volatile_u32(st, kStAggregate | cnt);
            // look back kLookBack predecessors per round: their status words are
            // read with independent loads, then taken in order until a prefix
            // (done) or a word not yet published (poll again from there)
            int64_t j = (int64_t)tile - 1;
            uint32_t spins = 0u;
            bool done = false;
            while (!done) {
                uint32_t sw[kLookBack];
#pragma unroll
                for (int q = 0; q < kLookBack; ++q)
                    sw[q] = j - q >= 0 ? ld_volatile_u32(status + (size_t)(j - q) * kRadixBins + t)
                                       : kStPrefix;
                int q = 0;
#pragma unroll
                for (int qq = 0; qq < kLookBack; ++qq) {
                    if (q == qq && !done) {
                        const uint32_t f = sw[qq] & ~kStValue;
                        if (f != 0u) {
                            excl += sw[qq] & kStValue;
                            done = f == kStPrefix;
                            ++q;
                        }
                    }
                }
                j -= q;
                if (!done && q < kLookBack) {   // word j not yet published
                    if (++spins >= kSpinLimit) {
                        atomicOr(flags, kFlagTimeout);
                        break;
                    }
                    if (spins > 64u) __nanosleep(64);
                }
            }
            st_volatile_u32(st, kStPrefix | ((excl + cnt) & kStValue));
        }
        s_gbase[t] = digit_start[t] + excl;

        // exclusive scan of the tile's digit counts
        uint32_t x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_wtot[w] = x;
        __syncthreads();
        uint32_t before = 0u;
        for (int i = 0; i < w; ++i) before += s_wtot[i];
        s_tdig[t] = before + x - cnt;
        __syncthreads();

        // stage the tile in digit order
#pragma unroll
        for (int k = 0; k < kSortItems; ++k) {
            const int64_t idx = base + (int64_t)w * (32 * kSortItems) + k * 32 + lane;
            if (idx < n) {
                const uint32_t d = (uint32_t)(key[k] >> shift) & 0xffu;
                const uint32_t p = s_tdig[d] + s_whist[w][d] + rank[k];
                s_keys[p] = key[k];
                s_vals[p] = val[k];
            }
        }
        __syncthreads();

        // runs of equal digits go to consecutive global addresses
        const int64_t rem = n - base;
        const int tile_n = rem < kSortTile ? (int)rem : kSortTile;
        for (int p = t; p < tile_n; p += kSortThreads) {
            const uint64_t k = s_keys[p];
            const uint32_t d = (uint32_t)(k >> shift) & 0xffu;
            const uint32_t out = s_gbase[d] + ((uint32_t)p - s_tdig[d]);
            if (WRITE_KEYS) keys_out[out] = k;
            vals_out[out] = s_vals[p];
        }
        __syncthreads();   // the next tile reuses the shared arrays
    }
}

// Finishes the runs of equal 24-bit key prefix (the output of the passes
// over bits 40..63).  Each thread takes one element p: it finds p's run
// [h, e) and places p at h + (number of run members smaller in (key,
// index)) -- a rank, so every element moves in parallel and no thread
// sorts a whole run.  A CTA stages its tile of kRunTile keys plus kRunMax + 1
// on either side in shared memory; a run that reaches the end of that window
// is longer than kRunMax and sets *gate instead (the full sort then redoes
// everything).  With gdst, each placed element also gathers its position:
// gdst[out] = (gsrc[index].xyz, index).
constexpr int kRunThreads = 256;
constexpr int kRunItems = 8;
constexpr int kRunTile = kRunThreads * kRunItems;
constexpr int kRunHalo = kRunMax + 1;

__global__ void __launch_bounds__(kRunThreads)
k_run_sort(const uint64_t *__restrict__ keys, const uint32_t *__restrict__ vals, int64_t n,
           uint64_t *__restrict__ keys_out, uint32_t *__restrict__ vals_out, uint32_t *gate,
           const uint32_t *flags, const float4 *__restrict__ gsrc, float4 *__restrict__ gdst)
{
    if (timed_out(flags)) return;
    __shared__ uint64_t s_k[kRunTile + 2 * kRunHalo];
    __shared__ uint32_t s_v[kRunTile + 2 * kRunHalo];
    const int64_t t0 = (int64_t)blockIdx.x * kRunTile;
    const int64_t lo = t0 - kRunHalo > 0 ? t0 - kRunHalo : 0;
    const int64_t hi = t0 + kRunTile + kRunHalo < n ? t0 + kRunTile + kRunHalo : n;
    const int w = (int)(hi - lo);
    for (int q = threadIdx.x; q < w; q += kRunThreads) {
        s_k[q] = keys[lo + q];
        s_v[q] = vals[lo + q];
    }
    __syncthreads();
    bool too_long = false;
    int64_t outs[kRunItems];
    uint32_t vps[kRunItems];
#pragma unroll
    for (int u = 0; u < kRunItems; ++u) {
        outs[u] = -1;
        vps[u] = 0u;
        const int64_t p = t0 + threadIdx.x + (int64_t)kRunThreads * u;
        if (p >= n) continue;
        const int a = (int)(p - lo);
        const uint64_t kp = s_k[a];
        const uint32_t vp = s_v[a];
        const uint64_t pre = kp >> kPrefixShift;
        int h = a;
        while (h > 0 && (s_k[h - 1] >> kPrefixShift) == pre) --h;
        int e = a + 1;
        while (e < w && (s_k[e] >> kPrefixShift) == pre) ++e;
        // a run cut by the window edge (h == 0 with lo > 0, or e == w with
        // hi < n) is at least kRunMax + 2 long, so the length test covers it
        if (e - h > kRunMax) {
            too_long = true;
            continue;
        }
        int rank = 0;
        for (int q = h; q < e; ++q) {
            const uint64_t kq = s_k[q];
            rank += (kq < kp || (kq == kp && s_v[q] < vp)) ? 1 : 0;
        }
        const int64_t out = lo + h + rank;
        if (keys_out) keys_out[out] = kp;
        vals_out[out] = vp;
        outs[u] = out;
        vps[u] = vp;
    }
    if (gdst) {   // the gather, fused: every random load issued before any store
        float4 g[kRunItems];
#pragma unroll
        for (int u = 0; u < kRunItems; ++u)
            if (outs[u] >= 0) g[u] = gsrc[vps[u]];
#pragma unroll
        for (int u = 0; u < kRunItems; ++u)
            if (outs[u] >= 0)
                gdst[outs[u]] = make_float4(g[u].x, g[u].y, g[u].z, __int_as_float((int)vps[u]));
    }
    if (__any_sync(0xffffffffu, too_long) && (threadIdx.x & 31) == 0) atomicOr(gate, 1u);
}

}  // namespace

cudaError_t launch_radix_passes(nl_ctx *ctx, int64_t n, uint64_t *keys_final,
                                uint32_t *vals_final, cudaStream_t s, const SortRecompute &rk,
                                float4 *pos_sorted)
{
    if (n <= 0) return cudaSuccess;
    const int64_t tiles = (n + kSortTile - 1) / kSortTile;
    // the tile (36 KB) and the static arrays (10 KB) fit the 48 KB a CTA gets
    // without opt-in, so the passes need no per-device attribute
    static_assert(kSortDynSmem + 4 * (kWarps * kRadixBins + 2 * kRadixBins + kWarps + 1) + 64 <=
                      48 * 1024,
                  "onesweep tile needs the opt-in shared memory");
    // look-back status: the fast path's slots now; the full sort's slots are
    // cleared by its gated key recompute, so a clear gate costs no clearing
    const size_t slot_words = (size_t)tiles * kRadixBins;
    NL_CUDA_TRY(cudaMemsetAsync(ctx->sort_status + kKeyPasses * slot_words, 0,
                                sizeof(uint32_t) * kTopPasses * slot_words, s));
    NL_CUDA_TRY(cudaMemsetAsync(ctx->sort_ctr, 0, sizeof(uint32_t) * kStatusPasses, s));
    NL_CUDA_TRY(cudaMemsetAsync(ctx->sort_gate, 0, sizeof(uint32_t), s));
    // every pass is one resident wave whose CTAs loop over tile tickets, so
    // a gated pass whose gate is clear costs one wave of CTAs that return
    const unsigned grid = resident_grid(ctx, k_onesweep<true>, kSortThreads, kSortDynSmem, tiles);
    // fast path: the top kTopPasses digits, then the prefix runs
    int src = 0;
    for (int q = 0; q < kTopPasses; ++q) {
        const int p = kKeyPasses - kTopPasses + q;   // digit
        const int slot = kKeyPasses + q;             // status slot of the fast path
        uint32_t *status = ctx->sort_status + (size_t)slot * slot_words;
        k_onesweep<true><<<grid, kSortThreads, kSortDynSmem, s>>>(
            ctx->keys[src], ctx->vals[src], ctx->keys[1 - src], ctx->vals[1 - src], n,
            kRadixBits * p, ctx->hist + p * kRadixBins, status, ctx->sort_ctr + slot, ctx->flags,
            nullptr);
        NL_CUDA_TRY(cudaGetLastError());
        src = 1 - src;
    }
    {
        const int64_t blocks = (n + kRunTile - 1) / kRunTile;
        k_run_sort<<<(unsigned)blocks, kRunThreads, 0, s>>>(ctx->keys[src], ctx->vals[src], n,
                                                           keys_final, vals_final, ctx->sort_gate,
                                                           ctx->flags, rk.pos, pos_sorted);
        NL_CUDA_TRY(cudaGetLastError());
    }
    // full sort, gated: runs only when a prefix run was too long
    NL_CUDA_TRY(launch_keys(ctx, rk.n, rk.pos, rk.Lx, rk.Ly, rk.Lz, rk.Sx, rk.Sy, rk.Sz,
                            rk.curve, s, ctx->sort_gate, ctx->sort_status,
                            (int64_t)(kKeyPasses * slot_words)));
    NL_CUDA_TRY(launch_hist_scan(ctx, s, ctx->sort_gate));
    src = 0;
    for (int p = 0; p < kKeyPasses; ++p) {
        const bool last = p == kKeyPasses - 1;
        uint64_t *ko = last ? (keys_final ? keys_final : ctx->keys[1 - src]) : ctx->keys[1 - src];
        uint32_t *vo = last ? vals_final : ctx->vals[1 - src];
        uint32_t *status = ctx->sort_status + (size_t)p * slot_words;
        if (last && !keys_final)
            k_onesweep<false><<<grid, kSortThreads, kSortDynSmem, s>>>(
                ctx->keys[src], ctx->vals[src], ko, vo, n, kRadixBits * p,
                ctx->hist + p * kRadixBins, status, ctx->sort_ctr + p, ctx->flags, ctx->sort_gate);
        else
            k_onesweep<true><<<grid, kSortThreads, kSortDynSmem, s>>>(
                ctx->keys[src], ctx->vals[src], ko, vo, n, kRadixBits * p,
                ctx->hist + p * kRadixBins, status, ctx->sort_ctr + p, ctx->flags, ctx->sort_gate);
        NL_CUDA_TRY(cudaGetLastError());
        src = 1 - src;
    }
    // the gather of the full sort's order, gated like its passes
    if (pos_sorted)
        NL_CUDA_TRY(launch_gather(ctx, n, rk.pos, reinterpret_cast<const int32_t *>(vals_final),
                                  pos_sorted, ctx->flags, s, ctx->sort_gate));
    return cudaSuccess;
}

}  // namespace nl
