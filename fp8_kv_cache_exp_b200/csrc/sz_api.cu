// sz_api.cu -- the extern "C" entry points of libsplitzip (see include/splitzip.h).
// Host-side argument checks, workspace partitioning and kernel dispatch.  No
// device memory is allocated here; every device buffer belongs to the caller.
#include <cuda_runtime.h>

#include "splitzip.h"
#include "sz_common.cuh"
#include "sz_internal.h"

namespace {

using namespace sz;

bool dtype_ok(sz_dtype d) { return d == SZ_BF16 || d == SZ_FP8_E5M2; }

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

uint64_t total_tiles(int T, const uint64_t *n) {
    uint64_t s = 0;
    for (int t = 0; t < T; ++t) s += cdiv(n[t], kBlock);
    return s;
}

int num_sms() {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    sms = cache[dev].load(std::memory_order_acquire);
    if (sms > 0) return sms;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(sms, std::memory_order_release);
    return sms;
}

// Shared checks of a batch: dtype, T, element counts, workspace.
sz_status check_batch(sz_dtype dtype, int T, const uint64_t *n, const void *d_ws, size_t ws_bytes) {
    if (!dtype_ok(dtype)) return SZ_ERR_UNSUPPORTED_DTYPE;
    if (T < 1 || T > SZ_MAX_BATCH || !n || !d_ws || !aligned(d_ws, 8)) return SZ_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t)
        if (n[t] >= (1ull << 32)) return SZ_ERR_INVALID_ARG;
    if (ws_bytes < sz_workspace_bytes_batched(dtype, T, n)) return SZ_ERR_BUFFER_TOO_SMALL;
    return SZ_OK;
}

}  // namespace

extern "C" {

const char *sz_status_string(sz_status s) {
    switch (s) {
        case SZ_OK: return "ok";
        case SZ_ERR_INVALID_ARG: return "invalid argument";
        case SZ_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype";
        case SZ_ERR_BUFFER_TOO_SMALL: return "buffer too small";
        case SZ_ERR_CORRUPT_STREAM: return "corrupt stream";
        case SZ_ERR_CUDA: return "CUDA runtime error";
        case SZ_ERR_TIMEOUT: return "look-back wait timed out";
        case SZ_ERR_PLAN_MISMATCH: return "data or sizes do not match the plan";
        case SZ_ERR_INTERNAL: return "internal consistency check failed";
    }
    return "unknown status";
}

size_t sz_workspace_bytes_batched(sz_dtype dtype, int T, const uint64_t *n) {
    if (!dtype_ok(dtype) || T < 1 || T > SZ_MAX_BATCH || !n) return 0;
    return ws_layout(T, total_tiles(T, n)).bytes;
}

size_t sz_workspace_bytes(sz_dtype dtype, uint64_t n) { return sz_workspace_bytes_batched(dtype, 1, &n); }

size_t sz_stream_bytes(sz_dtype dtype, uint64_t n, uint64_t E) {
    if (!dtype_ok(dtype)) return 0;
    return stream_layout(dtype, n, E).total;
}

size_t sz_max_compressed_size(sz_dtype dtype, uint64_t n) { return sz_stream_bytes(dtype, n, n); }

sz_status sz_workspace_init(void *d_ws, size_t ws_bytes, cudaStream_t stream) {
    if (!d_ws || !aligned(d_ws, 8) || ws_bytes < size_t(kCtlWords) * 4) return SZ_ERR_INVALID_ARG;
    return cudaMemsetAsync(d_ws, 0, ws_bytes, stream) == cudaSuccess ? SZ_OK : SZ_ERR_CUDA;
}

sz_status sz_plan_batched(sz_dtype dtype, int T, const void *const *d_in, const uint64_t *n,
                          void *d_ws, size_t ws_bytes, sz_plan_t *d_plans, cudaStream_t stream) {
    sz_status s = check_batch(dtype, T, n, d_ws, ws_bytes);
    if (s != SZ_OK) return s;
    if (!d_in || !d_plans || !aligned(d_plans, 8)) return SZ_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t)
        if (n[t] && (!d_in[t] || !aligned(d_in[t], 16))) return SZ_ERR_INVALID_ARG;
    const WsLayout w = ws_layout(T, total_tiles(T, n));
    uint8_t *ws = static_cast<uint8_t *>(d_ws);
    PlanArgs a;
    a.dtype = dtype;
    a.T = T;
    a.num_sms = num_sms();
    if (a.num_sms <= 0) return SZ_ERR_CUDA;
    a.in = d_in;
    a.n = n;
    a.ctl = reinterpret_cast<uint32_t *>(ws);
    a.hist = reinterpret_cast<uint32_t *>(ws + w.hist);
    a.ticket = reinterpret_cast<uint32_t *>(ws + w.ticket);
    a.plans = reinterpret_cast<uint8_t *>(d_plans);
    a.paged = nullptr;
    return launch_plan(a, stream);
}

sz_status sz_plan(sz_dtype dtype, const void *d_in, uint64_t n, void *d_ws, size_t ws_bytes,
                  sz_plan_t *d_plan, cudaStream_t stream) {
    const void *in[1] = {d_in};
    return sz_plan_batched(dtype, 1, in, &n, d_ws, ws_bytes, d_plan, stream);
}

sz_status sz_compressed_sizes(int T, const sz_plan_t *d_plans, uint64_t *h_bytes,
                              cudaStream_t stream) {
    if (T < 1 || T > SZ_MAX_BATCH || !d_plans || !h_bytes) return SZ_ERR_INVALID_ARG;
    sz_plan_t host[SZ_MAX_BATCH];
    if (cudaMemcpyAsync(host, d_plans, sizeof(sz_plan_t) * T, cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return SZ_ERR_CUDA;
    for (int t = 0; t < T; ++t) {
        uint64_t v = 0;
        for (int b = 0; b < 8; ++b) v |= uint64_t(host[t].bytes[40 + b]) << (8 * b);
        h_bytes[t] = v;
    }
    return SZ_OK;
}

sz_status sz_compressed_size(const sz_plan_t *d_plan, uint64_t *h_bytes, cudaStream_t stream) {
    return sz_compressed_sizes(1, d_plan, h_bytes, stream);
}

sz_status sz_plan_set_flags(int T, sz_plan_t *d_plans, unsigned flags, cudaStream_t stream) {
    if (T < 1 || T > SZ_MAX_BATCH || !d_plans || !aligned(d_plans, 8)) return SZ_ERR_INVALID_ARG;
    if (flags & ~unsigned(SZ_FLAG_RAW_BLOCKS)) return SZ_ERR_INVALID_ARG;
    // byte 39 of each of the T consecutive 64-byte plans: one strided memset
    if (cudaMemset2DAsync(reinterpret_cast<uint8_t *>(d_plans) + 39, sizeof(sz_plan_t), int(flags), 1, size_t(T),
                          stream) != cudaSuccess)
        return SZ_ERR_CUDA;
    return SZ_OK;
}

}  // extern "C"

namespace sz {

sz_status check_encode_args(sz_dtype dtype, int T, const sz_plan_t *d_plans, const void *const *d_in,
                            const uint64_t *n, void *const *d_out, const size_t *out_cap, const uint64_t *d_totals,
                            const void *d_ws, size_t ws_bytes) {
    sz_status s = check_batch(dtype, T, n, d_ws, ws_bytes);
    if (s != SZ_OK) return s;
    if (!d_plans || !aligned(d_plans, 8) || !d_in || !d_out || !out_cap) return SZ_ERR_INVALID_ARG;
    if (d_totals && !aligned(d_totals, 8)) return SZ_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t) {
        if (n[t] && (!d_in[t] || !aligned(d_in[t], 16))) return SZ_ERR_INVALID_ARG;
        if (!d_out[t] || !aligned(d_out[t], 16)) return SZ_ERR_INVALID_ARG;
        // the smallest stream for n (no escapes) must fit in any case
        if (out_cap[t] < stream_layout(dtype, n[t], 0).total) return SZ_ERR_BUFFER_TOO_SMALL;
    }
    return SZ_OK;
}

}  // namespace sz

extern "C" {

namespace {

// Ordinary encode (plans are the tensors' own) or codebook reuse (plans give
// codebooks only).
sz_status encode_common(sz_dtype dtype, int T, const sz_plan_t *d_plans, const void *const *d_in,
                        const uint64_t *n, void *const *d_out, const size_t *out_cap, uint64_t *d_totals,
                        bool reuse, const sz_paged_t *paged, void *d_ws, size_t ws_bytes, cudaStream_t stream) {
    const sz_status s = check_encode_args(dtype, T, d_plans, d_in, n, d_out, out_cap, d_totals, d_ws, ws_bytes);
    if (s != SZ_OK) return s;
    const uint64_t tiles = total_tiles(T, n);
    const WsLayout w = ws_layout(T, tiles);
    uint8_t *ws = static_cast<uint8_t *>(d_ws);
    EncodeArgs a;
    a.dtype = dtype;
    a.T = T;
    a.num_sms = num_sms();
    a.plans = reinterpret_cast<const uint8_t *>(d_plans);
    a.in = d_in;
    a.n = n;
    a.out = d_out;
    a.cap = out_cap;
    a.ctl = reinterpret_cast<uint32_t *>(ws);
    a.status = reinterpret_cast<unsigned long long *>(ws + w.status);
    a.group = reinterpret_cast<unsigned long long *>(ws + w.group);
    a.totals = reinterpret_cast<unsigned long long *>(d_totals);
    a.reuse = reuse ? 1 : 0;
    a.paged = paged;
    return launch_encode(a, stream);
}

}  // namespace

sz_status sz_encode_batched(sz_dtype dtype, int T, const sz_plan_t *d_plans,
                            const void *const *d_in, const uint64_t *n, void *const *d_out,
                            const size_t *out_cap, void *d_ws, size_t ws_bytes,
                            cudaStream_t stream) {
    return encode_common(dtype, T, d_plans, d_in, n, d_out, out_cap, nullptr, false, nullptr, d_ws, ws_bytes,
                         stream);
}

sz_status sz_encode(sz_dtype dtype, const sz_plan_t *d_plan, const void *d_in, uint64_t n,
                    void *d_out, size_t out_cap, void *d_ws, size_t ws_bytes, cudaStream_t stream) {
    const void *in[1] = {d_in};
    void *out[1] = {d_out};
    return sz_encode_batched(dtype, 1, d_plan, in, &n, out, &out_cap, d_ws, ws_bytes, stream);
}

sz_status sz_encode_reuse_batched(sz_dtype dtype, int T, const sz_plan_t *d_codebooks,
                                  const void *const *d_in, const uint64_t *n, void *const *d_out,
                                  const size_t *out_cap, uint64_t *d_totals, void *d_ws, size_t ws_bytes,
                                  cudaStream_t stream) {
    return encode_common(dtype, T, d_codebooks, d_in, n, d_out, out_cap, d_totals, true, nullptr, d_ws,
                         ws_bytes, stream);
}

sz_status sz_encode_reuse(sz_dtype dtype, const sz_plan_t *d_codebook, const void *d_in, uint64_t n,
                          void *d_out, size_t out_cap, uint64_t *d_total, void *d_ws, size_t ws_bytes,
                          cudaStream_t stream) {
    const void *in[1] = {d_in};
    void *out[1] = {d_out};
    return sz_encode_reuse_batched(dtype, 1, d_codebook, in, &n, out, &out_cap, d_total, d_ws, ws_bytes,
                                   stream);
}

namespace {

sz_status decode_common(sz_dtype dtype, int T, const void *const *d_comp, const size_t *comp_bytes,
                        void *const *d_out, const uint64_t *n, const sz_paged_t *paged, void *d_ws,
                        size_t ws_bytes, cudaStream_t stream) {
    sz_status s = check_batch(dtype, T, n, d_ws, ws_bytes);
    if (s != SZ_OK) return s;
    if (!d_comp || !comp_bytes || !d_out) return SZ_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t) {
        if (!d_comp[t] || !aligned(d_comp[t], 16)) return SZ_ERR_INVALID_ARG;
        if (n[t] && (!d_out[t] || !aligned(d_out[t], 16))) return SZ_ERR_INVALID_ARG;
        // every plane of an n-element stream must lie inside the buffer
        if (comp_bytes[t] < stream_layout(dtype, n[t], 0).total) return SZ_ERR_CORRUPT_STREAM;
    }
    DecodeArgs a;
    a.dtype = dtype;
    a.T = T;
    a.num_sms = num_sms();
    a.comp = d_comp;
    a.comp_bytes = comp_bytes;
    a.out = d_out;
    a.n = n;
    a.ctl = static_cast<uint32_t *>(d_ws);
    a.paged = paged;
    return launch_decode(a, stream);
}

}  // namespace

sz_status sz_decode_batched(sz_dtype dtype, int T, const void *const *d_comp,
                            const size_t *comp_bytes, void *const *d_out, const uint64_t *n,
                            void *d_ws, size_t ws_bytes, cudaStream_t stream) {
    return decode_common(dtype, T, d_comp, comp_bytes, d_out, n, nullptr, d_ws, ws_bytes, stream);
}

sz_status sz_decode(sz_dtype dtype, const void *d_comp, size_t comp_bytes, void *d_out, uint64_t n,
                    void *d_ws, size_t ws_bytes, cudaStream_t stream) {
    const void *comp[1] = {d_comp};
    void *out[1] = {d_out};
    return sz_decode_batched(dtype, 1, comp, &comp_bytes, out, &n, d_ws, ws_bytes, stream);
}

sz_status sz_enable_peer_access(int device, int peer) {
    if (device < 0 || peer < 0) return SZ_ERR_INVALID_ARG;
    if (device == peer) return SZ_OK;
    int prev = 0, can = 0;
    if (cudaGetDevice(&prev) != cudaSuccess) return SZ_ERR_CUDA;
    if (cudaDeviceCanAccessPeer(&can, device, peer) != cudaSuccess || !can) return SZ_ERR_CUDA;
    if (cudaSetDevice(device) != cudaSuccess) return SZ_ERR_CUDA;
    cudaError_t e = cudaDeviceEnablePeerAccess(peer, 0);
    if (e == cudaErrorPeerAccessAlreadyEnabled) {
        cudaGetLastError();  // clear the sticky-free "already enabled" status
        e = cudaSuccess;
    }
    const bool ok = e == cudaSuccess;
    if (cudaSetDevice(prev) != cudaSuccess) return SZ_ERR_CUDA;
    return ok ? SZ_OK : SZ_ERR_CUDA;
}

sz_status sz_last_device_status(void *d_ws, cudaStream_t stream) {
    if (!d_ws || !aligned(d_ws, 8)) return SZ_ERR_INVALID_ARG;
    uint32_t err[2] = {0, 0};
    if (cudaMemcpyAsync(err, d_ws, sizeof(err), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return SZ_ERR_CUDA;
    if (err[0] != 0) {
        if (cudaMemsetAsync(d_ws, 0, sizeof(err), stream) != cudaSuccess) return SZ_ERR_CUDA;
    }
    return static_cast<sz_status>(err[0]);
}

}  // extern "C"

// ------------------------------------------------------------- paged tensors

namespace sz {

PageRef page_ref(const sz_paged_t *d) {
    PageRef r;
    r.pages = d ? d->pages : nullptr;
    r.pool_pages = d ? d->pool_pages : 0;
    r.page_bytes = d ? d->page_bytes : 0;
    r.page_elems = d ? d->page_elems : 0;
    return r;
}

}  // namespace sz

namespace {

// Host checks of T page descriptors; fills pools[t] with each pool's base.
sz_status check_paged(sz_dtype dtype, int T, const sz_paged_t *pg, const uint64_t *n, const void **pools) {
    if (!pg || !n || T < 1 || T > SZ_MAX_BATCH) return SZ_ERR_INVALID_ARG;
    const uint64_t eb = dtype == SZ_BF16 ? 2 : 1;
    for (int t = 0; t < T; ++t) {
        const sz_paged_t &d = pg[t];
        pools[t] = d.pool;
        if (n[t] == 0) continue;
        if (!d.pool || !aligned(d.pool, 16) || !d.pages || !aligned(d.pages, 4) || d.pool_pages == 0)
            return SZ_ERR_INVALID_ARG;
        if (d.page_elems == 0 || d.page_elems % 1024u != 0 || d.page_elems > (1u << 18) || d.page_bytes % 16 != 0 ||
            d.page_bytes < uint64_t(d.page_elems) * eb)
            return SZ_ERR_INVALID_ARG;
    }
    return SZ_OK;
}

}  // namespace

sz_status sz_plan_paged_batched(sz_dtype dtype, int T, const sz_paged_t *src, const uint64_t *n,
                                void *d_ws, size_t ws_bytes, sz_plan_t *d_plans, cudaStream_t stream) {
    if (!dtype_ok(dtype)) return SZ_ERR_UNSUPPORTED_DTYPE;
    const void *pools[SZ_MAX_BATCH];
    sz_status s = check_paged(dtype, T, src, n, pools);
    if (s != SZ_OK) return s;
    s = check_batch(dtype, T, n, d_ws, ws_bytes);
    if (s != SZ_OK) return s;
    if (!d_plans || !aligned(d_plans, 8)) return SZ_ERR_INVALID_ARG;
    const WsLayout w = ws_layout(T, total_tiles(T, n));
    uint8_t *ws = static_cast<uint8_t *>(d_ws);
    PlanArgs a;
    a.dtype = dtype;
    a.T = T;
    a.num_sms = num_sms();
    if (a.num_sms <= 0) return SZ_ERR_CUDA;
    a.in = pools;
    a.n = n;
    a.ctl = reinterpret_cast<uint32_t *>(ws);
    a.hist = reinterpret_cast<uint32_t *>(ws + w.hist);
    a.ticket = reinterpret_cast<uint32_t *>(ws + w.ticket);
    a.plans = reinterpret_cast<uint8_t *>(d_plans);
    a.paged = src;
    return launch_plan(a, stream);
}

sz_status sz_encode_paged_batched(sz_dtype dtype, int T, const sz_plan_t *d_plans, const sz_paged_t *src,
                                  const uint64_t *n, void *const *d_out, const size_t *out_cap, void *d_ws,
                                  size_t ws_bytes, cudaStream_t stream) {
    if (!dtype_ok(dtype)) return SZ_ERR_UNSUPPORTED_DTYPE;
    const void *pools[SZ_MAX_BATCH];
    sz_status s = check_paged(dtype, T, src, n, pools);
    if (s != SZ_OK) return s;
    return encode_common(dtype, T, d_plans, pools, n, d_out, out_cap, nullptr, false, src, d_ws, ws_bytes, stream);
}

sz_status sz_decode_paged_batched(sz_dtype dtype, int T, const void *const *d_comp, const size_t *comp_bytes,
                                  const sz_paged_t *dst, const uint64_t *n, void *d_ws, size_t ws_bytes,
                                  cudaStream_t stream) {
    if (!dtype_ok(dtype)) return SZ_ERR_UNSUPPORTED_DTYPE;
    const void *pools[SZ_MAX_BATCH];
    sz_status s = check_paged(dtype, T, dst, n, pools);
    if (s != SZ_OK) return s;
    void *outs[SZ_MAX_BATCH];
    for (int t = 0; t < T; ++t) outs[t] = const_cast<void *>(pools[t]);
    return decode_common(dtype, T, d_comp, comp_bytes, outs, n, dst, d_ws, ws_bytes, stream);
}

sz_status sz_encode_reuse_paged_batched(sz_dtype dtype, int T, const sz_plan_t *d_codebooks,
                                        const sz_paged_t *src, const uint64_t *n, void *const *d_out,
                                        const size_t *out_cap, uint64_t *d_totals, void *d_ws, size_t ws_bytes,
                                        cudaStream_t stream) {
    if (!dtype_ok(dtype)) return SZ_ERR_UNSUPPORTED_DTYPE;
    const void *pools[SZ_MAX_BATCH];
    sz_status s = check_paged(dtype, T, src, n, pools);
    if (s != SZ_OK) return s;
    return encode_common(dtype, T, d_codebooks, pools, n, d_out, out_cap, d_totals, true, src, d_ws, ws_bytes,
                         stream);
}
