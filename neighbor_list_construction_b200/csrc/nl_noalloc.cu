// nl_noalloc.cu -- curve sort that allocates nothing, for callers that
// cannot call cudaMalloc.
//
// Some callers cannot allocate device memory at all: code running under a
// framework that owns every allocation (a custom caching allocator, a memory
// pool fixed at start-up), plugins loaded into such a host, or code that must
// not allocate between stream captures.  For them nl_sort_hilbert_noalloc
// runs the same kernels as nl_sort_hilbert, with the sort's scratch (key and
// index ping-pong buffers, digit histograms, look-back words, tile tickets,
// status word) in one file-scope __device__ array below instead of in a
// context.  The array is part of the library image: every GPU that loads
// libnl.so holds it (kNoallocScratchBytes, about 28 MiB) until the process
// exits.
//
// Host code cannot use the array's name as a device address (in host code it
// names a host-side shadow), so the first call on each device asks the
// runtime for the device address with cudaGetSymbolAddress, with that device
// current, and keeps it; a lookup that fails is not kept, and the next call
// tries again.  That first call should come before any stream capture.  Every call shares the one array: calls whose work overlaps on the
// GPU (different streams, or several host threads) race and must be ordered
// by the caller.
#include <cmath>
#include <mutex>

#include "nl_internal.cuh"

namespace {

constexpr int64_t kNoallocMaxAtoms = int64_t(1) << 20;
constexpr int64_t kNoallocTiles = (kNoallocMaxAtoms + nl::kSortTile - 1) / nl::kSortTile;

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
constexpr size_t kOffKeys0 = 0;
constexpr size_t kOffKeys1 = align256(kOffKeys0 + sizeof(uint64_t) * kNoallocMaxAtoms);
constexpr size_t kOffVals0 = align256(kOffKeys1 + sizeof(uint64_t) * kNoallocMaxAtoms);
constexpr size_t kOffVals1 = align256(kOffVals0 + sizeof(uint32_t) * kNoallocMaxAtoms);
constexpr size_t kOffHist = align256(kOffVals1 + sizeof(uint32_t) * kNoallocMaxAtoms);
constexpr size_t kOffStatus = align256(kOffHist + sizeof(uint32_t) * nl::kKeyPasses * nl::kRadixBins);
constexpr size_t kOffCtr = align256(kOffStatus + sizeof(uint32_t) * nl::kStatusPasses *
                                                     kNoallocTiles * nl::kRadixBins);
constexpr size_t kOffFlags = align256(kOffCtr + sizeof(uint32_t) * nl::kStatusPasses);
constexpr size_t kNoallocScratchBytes = align256(kOffFlags + 2 * sizeof(uint32_t));   // flags, gate

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the array and SM count, per device, filled in by the
// first call on that device that succeeds in looking them up.  A failed
// lookup stores nothing, so the next call tries again.
struct DeviceScratch {
    unsigned char *base = nullptr;
    int sm_count = 0;
};
constexpr int kMaxDevices = 64;
DeviceScratch g_devices[kMaxDevices];
std::mutex g_devices_mu;

// The array's address on the current device `dev` (looked up on first use).
cudaError_t device_scratch(int dev, DeviceScratch *out)
{
    std::lock_guard<std::mutex> lock(g_devices_mu);
    DeviceScratch &d = g_devices[dev];
    if (!d.base) {
        void *p = nullptr;
        int sms = 0;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess || !p) {
            (void)cudaGetLastError();   // leave no stale error for the caller's next check
            return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
        }
        d.sm_count = sms;
        d.base = static_cast<unsigned char *>(p);
    }
    *out = d;
    return cudaSuccess;
}

__global__ void k_noalloc_status(const uint32_t *flags, int32_t *status_out)
{
    *status_out = (*flags & nl::kFlagTimeout) ? (int32_t)NL_ERR_TIMEOUT : (int32_t)NL_OK;
}

}  // namespace

extern "C" nl_status nl_sort_hilbert_noalloc(int64_t n, const float *pos, const float *box,
                                             int32_t *perm_out, float *pos_sorted_out,
                                             uint64_t *keys_out, int32_t *status_out,
                                             void *stream)
{
    if (n < 0 || !box) return NL_ERR_ARG;
    if (n > kNoallocMaxAtoms) return NL_ERR_CAPACITY;
    for (int a = 0; a < 3; ++a)
        if (!std::isfinite(box[a]) || !(box[a] > 0.0f)) return NL_ERR_ARG;
    if (n > 0 && (!pos || !perm_out || !pos_sorted_out ||
                  (reinterpret_cast<uintptr_t>(pos) & 15u) ||
                  (reinterpret_cast<uintptr_t>(pos_sorted_out) & 15u)))
        return NL_ERR_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NL_ERR_CUDA;
    DeviceScratch d;
    if (device_scratch(dev, &d) != cudaSuccess) return NL_ERR_CUDA;

    // A context view over the static array; nothing here allocates.
    nl_ctx view;
    view.device = dev;
    view.sm_count = d.sm_count;
    view.max_atoms = kNoallocMaxAtoms;
    view.max_sort_tiles = kNoallocTiles;
    view.keys[0] = reinterpret_cast<uint64_t *>(d.base + kOffKeys0);
    view.keys[1] = reinterpret_cast<uint64_t *>(d.base + kOffKeys1);
    view.vals[0] = reinterpret_cast<uint32_t *>(d.base + kOffVals0);
    view.vals[1] = reinterpret_cast<uint32_t *>(d.base + kOffVals1);
    view.hist = reinterpret_cast<uint32_t *>(d.base + kOffHist);
    view.sort_status = reinterpret_cast<uint32_t *>(d.base + kOffStatus);
    view.sort_ctr = reinterpret_cast<uint32_t *>(d.base + kOffCtr);
    view.flags = reinterpret_cast<uint32_t *>(d.base + kOffFlags);
    view.sort_gate = view.flags + 1;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: clear what must start at 0
    if (cudaMemsetAsync(view.flags, 0, 2 * sizeof(uint32_t), s) != cudaSuccess) return NL_ERR_CUDA;
    if (n > 0) {
        volatile float sx = 2097152.0f / box[0];
        volatile float sy = 2097152.0f / box[1];
        volatile float sz = 2097152.0f / box[2];
        const float4 *p4 = reinterpret_cast<const float4 *>(pos);
        if (cudaMemsetAsync(view.hist, 0, sizeof(uint32_t) * nl::kKeyPasses * nl::kRadixBins, s) !=
            cudaSuccess)
            return NL_ERR_CUDA;
        if (nl::launch_keys(&view, n, p4, box[0], box[1], box[2], sx, sy, sz, 0, s) != cudaSuccess)
            return NL_ERR_CUDA;
        if (nl::launch_hist_scan(&view, s) != cudaSuccess) return NL_ERR_CUDA;
        const nl::SortRecompute rk{p4, n, box[0], box[1], box[2], sx, sy, sz, 0};
        if (nl::launch_radix_passes(&view, n, keys_out, reinterpret_cast<uint32_t *>(perm_out), s,
                                    rk, reinterpret_cast<float4 *>(pos_sorted_out)) != cudaSuccess)
            return NL_ERR_CUDA;
    }
    if (status_out) {
        k_noalloc_status<<<1, 1, 0, s>>>(view.flags, status_out);
        if (cudaGetLastError() != cudaSuccess) return NL_ERR_CUDA;
    }
    return NL_OK;
}
