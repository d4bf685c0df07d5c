// sz_noalloc.cu -- sz_encode_noalloc: encode without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they encode:
// a serving engine that reserves all of a GPU's memory for its KV pool at
// start-up and hands the codec only the tensor and the destination buffer, or
// a transfer-engine hook that receives source, destination and a stream but no
// way to reach an allocator.  For them this entry point runs the ordinary
// encode kernel on a scratch area that the library itself holds: a file-scope
// device array, present on every GPU that loads the library until the process
// exits.  Nothing is allocated per call.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "splitzip.h"
#include "sz_common.cuh"
#include "sz_internal.h"

namespace {

// Largest tensor this entry point accepts, and the scratch it needs: the
// workspace of one tensor of that size (control block, histogram, ticket, one
// look-back status word per 4096-element tile and one per 32 of them) --
// 271,888 bytes.
constexpr uint64_t kNoAllocMaxTiles = SZ_NOALLOC_MAX_ELEMS / sz::kBlock;
constexpr size_t kNoAllocScratchBytes = sz::ws_layout(1, kNoAllocMaxTiles).bytes;
static_assert(kNoAllocScratchBytes == 271888, "the header states the scratch size");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
std::atomic<void *> g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  The host-side
// name g_noalloc_scratch is only a stand-in; the address is looked up once per
// device, with that device current, and cached.
sz_status scratch_address(int dev, void **out) {
    void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (p == nullptr) {
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
                return SZ_ERR_CUDA;
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return SZ_OK;
}

}  // namespace

extern "C" sz_status sz_encode_noalloc(sz_dtype dtype, const sz_plan_t *d_plan, const void *d_in,
                                       uint64_t n, void *d_out, size_t out_cap,
                                       uint32_t *d_status, cudaStream_t stream) {
    if (dtype != SZ_BF16 && dtype != SZ_FP8_E5M2) return SZ_ERR_UNSUPPORTED_DTYPE;
    if (n > SZ_NOALLOC_MAX_ELEMS) return SZ_ERR_BUFFER_TOO_SMALL;  // beyond the static scratch
    if (d_status != nullptr && (reinterpret_cast<uintptr_t>(d_status) & 3u) != 0) return SZ_ERR_INVALID_ARG;
    // The scratch used is the current device's: a stream of another device
    // would run the kernel there against this device's array, so it is refused.
    int dev = 0, stream_dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SZ_ERR_CUDA;
    // (the default streams always belong to the current device)
    if (stream != nullptr && stream != cudaStreamLegacy && stream != cudaStreamPerThread) {
        if (cudaStreamGetDevice(stream, &stream_dev) != cudaSuccess) return SZ_ERR_INVALID_ARG;
        if (stream_dev != dev) return SZ_ERR_INVALID_ARG;
    }
    void *scratch = nullptr;
    sz_status s = scratch_address(dev, &scratch);
    if (s != SZ_OK) return s;
    const size_t ws_bytes = sz_workspace_bytes(dtype, n);
    if (ws_bytes == 0 || ws_bytes > kNoAllocScratchBytes) return SZ_ERR_BUFFER_TOO_SMALL;
    // Every argument check of sz_encode first, so that a call refused on the
    // host enqueues nothing (not even the memset below).
    const void *in[1] = {d_in};
    void *out[1] = {d_out};
    s = sz::check_encode_args(dtype, 1, d_plan, in, &n, out, &out_cap, nullptr, scratch, ws_bytes);
    if (s != SZ_OK) return s;
    // The scratch keeps the previous call's contents.  Zero the control block
    // (error word, job and done counters) and this call's look-back status
    // words, which the kernel expects to start at zero.
    if (cudaMemsetAsync(scratch, 0, ws_bytes, stream) != cudaSuccess) return SZ_ERR_CUDA;
    s = sz_encode(dtype, d_plan, d_in, n, d_out, out_cap, scratch, ws_bytes, stream);
    if (s != SZ_OK) return s;
    // Device-side errors of this call (plan mismatch, output capacity,
    // look-back timeout) land in the scratch's error word; copy it out.
    if (d_status != nullptr &&
        cudaMemcpyAsync(d_status, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, stream) !=
            cudaSuccess)
        return SZ_ERR_CUDA;
    return SZ_OK;
}
