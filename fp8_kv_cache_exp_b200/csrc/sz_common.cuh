// sz_common.cuh -- definitions shared by the libsplitzip kernels and host layer:
// stream-format layout (format v1), workspace layout, launch parameter blocks
// and small device helpers.
//
// Method: "SplitZip: Ultra-Fast Lossless KV Compression for Disaggregated LLM
// Serving" (project page), Abstract: frequent exponents -> fixed 4-bit codes,
// sign and mantissa exact, rare exponents -> sparse escape stream.  The byte
// layout is this library's own (the page prints none); it is described in
// include/splitzip.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "splitzip.h"

namespace sz {

constexpr uint32_t kMagic = 0x564B5A53u;  // "SZKV" little-endian
constexpr uint32_t kVersion = 1;
constexpr uint32_t kBlockLog2 = 12;
constexpr uint32_t kBlock = 1u << kBlockLog2;  // elements per escape-offset block (= one tile)
constexpr uint32_t kCodes = 15;                // codes 0..14 name codebook entries
constexpr uint32_t kEscape = 15;               // code 15 marks an escaped exponent
constexpr uint32_t kFlagRawBlocks = 1;         // header byte 39, bit 0: raw blocks allowed
constexpr int kTileThreads = 256;              // threads per encode/decode tile CTA
constexpr int kSmallBatch = 8;                 // parameter blocks sized for <= 8 tensors ...
constexpr int kLargeBatch = SZ_MAX_BATCH;      // ... or for up to SZ_MAX_BATCH tensors

// Control words at the start of every workspace (u32 each).
enum : int {
    kCtlErr = 0,         // first device error (sz_status), 0 if none
    kCtlErrDetail = 1,   // error detail (e.g. the tile that failed)
    kCtlEpoch = 2,       // encode launch counter, tags look-back status words
    kCtlTileCtr = 3,     // encode job counter (tile ids in launch order)
    kCtlDone = 4,        // encode CTAs finished
    kCtlDecodeDone = 5,  // decode CTAs finished
    kCtlWords = 64       // 256 bytes reserved
};
// Decode's per-tensor block counters live in word 0 of each tensor's
// histogram slot (plan leaves the histograms zero; decode zeroes its counters
// before it returns), one 1 KB slot apart.
constexpr uint32_t kClaimStride = 256;

// Resident CTAs per SM of a kernel launched with `threads` threads and `smem`
// bytes of dynamic shared memory, on the current device; the first call per
// device also raises the kernel's dynamic shared-memory limit.  `cache` holds
// one entry per device (a function-local static of the launcher).  0 on error.
constexpr int kMaxDevices = 64;
inline int resident_per_sm(const void *kern, int threads, size_t smem, std::atomic<int> *cache) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    const int known = cache[dev].load(std::memory_order_acquire);
    if (known > 0) return known;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return 0;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess || per_sm < 1)
        return 0;
    cache[dev].store(per_sm, std::memory_order_release);
    return per_sm;
}

__host__ __device__ constexpr uint64_t align256(uint64_t x) { return (x + 255u) & ~uint64_t(255); }
__host__ __device__ constexpr uint64_t cdiv(uint64_t a, uint64_t b) { return (a + b - 1) / b; }

template <int DT> struct Dt;
template <> struct Dt<SZ_BF16> {
    static constexpr int kBins = 256;      // 8-bit exponent
    static constexpr int kElemBytes = 2;
};
template <> struct Dt<SZ_FP8_E5M2> {
    static constexpr int kBins = 32;       // 5-bit exponent
    static constexpr int kElemBytes = 1;
};

// Escape-section bytes of a raw block of m elements: the exponent bits above
// the low four, which its code nibbles hold (four per BF16 element, one per
// E5M2 element).  With raw blocks allowed, a block whose escapes would fill at
// least this many bytes is stored raw, and a coded block has fewer escapes, so
// its offsets-table count tells which it is.
template <int DT>
__host__ __device__ constexpr uint32_t raw_block_bytes(uint32_t m) {
    return DT == SZ_BF16 ? (m + 1) / 2 : (m + 7) / 8;
}

// Section offsets of a stream with n elements and E escapes.
struct Layout {
    uint64_t nb;         // 4096-element blocks
    uint64_t tab_end;    // end of the offsets table: 64 + 4(nb+1)
    uint64_t plane[3];   // BF16: sm, code ; E5M2: sign, mantissa, code
    uint64_t plane_len[3];
    int nplanes;
    uint64_t code;       // code-plane start (the last plane)
    uint64_t esc;        // escape-stream start
    uint64_t total;      // stream length
};

__host__ __device__ inline Layout stream_layout(int dtype, uint64_t n, uint64_t E) {
    Layout L;
    L.nb = cdiv(n, kBlock);
    L.tab_end = 64 + 4 * (L.nb + 1);
    if (dtype == SZ_BF16) {
        L.nplanes = 2;
        L.plane_len[0] = n;
        L.plane_len[1] = cdiv(n, 2);
        L.plane_len[2] = 0;
    } else {
        L.nplanes = 3;
        L.plane_len[0] = cdiv(n, 8);
        L.plane_len[1] = cdiv(n, 4);
        L.plane_len[2] = cdiv(n, 2);
    }
    uint64_t pos = align256(L.tab_end);
#if defined(__CUDA_ARCH__)
#pragma unroll
#endif
    for (int s = 0; s < 3; ++s) {
        L.plane[s] = pos;
        if (s < L.nplanes) pos = align256(pos + L.plane_len[s]);
    }
    L.code = L.plane[L.nplanes - 1];
    L.esc = pos;
    L.total = pos + E;
    return L;
}

// Encode's look-back works on two levels: one status word per chunk and one
// per group of kLbGroup consecutive chunks of a tensor.
constexpr int kLbGroupLog2 = 5;
constexpr uint32_t kLbGroup = 1u << kLbGroupLog2;

// Workspace partition: control block, per-tensor histograms and tickets
// (plan), per-tile look-back status words and per-group words (encode; a
// tensor's groups start at word (its first chunk >> kLbGroupLog2) + its index,
// so total_tiles / kLbGroup + T + 1 words hold every launch's groups).
struct WsLayout {
    size_t hist, ticket, status, group, bytes;
};
constexpr WsLayout ws_layout(int T, uint64_t total_tiles) {
    WsLayout w{};
    w.hist = kCtlWords * 4;
    w.ticket = w.hist + size_t(T) * 256 * 4;
    w.status = w.ticket + align256(size_t(T) * 4);
    w.group = w.status + align256(size_t(total_tiles) * 8);
    w.bytes = w.group + (size_t(total_tiles >> kLbGroupLog2) + size_t(T) + 1) * 8;
    return w;
}

// ------------------------------------------------------------- parameters
// Passed by value as __grid_constant__ kernel parameters: no descriptor copy.

// Where a tensor's elements live: contiguous at its base pointer (pages ==
// nullptr), or in pages of a pool at that base -- element i at
// base + pages[i / page_elems] * page_bytes + (i % page_elems) * element bytes.
struct PageRef {
    const int32_t *pages;
    uint64_t pool_pages;
    uint64_t page_bytes;
    uint32_t page_elems;  // a multiple of 1024 (a quarter block never straddles pages), <= 2^18
};

template <int MAXB>
struct PlanParams {
    uint32_t *ctl;
    uint32_t *hist;      // T x 256 counts
    uint32_t *ticket;    // T items-done counters
    uint8_t *plans;      // T x 64-byte plans
    uint64_t total_items;
    int T;
    const uint8_t *in[MAXB];
    uint64_t n[MAXB];
    uint64_t item_begin[MAXB + 1];  // prefix over tensors of ceil(n / item elements)
    PageRef pg[MAXB];
};

// Encode works in chunks of 1 << chunk_log2 consecutive 4096-element blocks of
// one tensor (chunk_log2 <= kMaxChunkLog2).  One look-back status word per
// chunk; the workspace holds one per block, enough for any chunk size.
constexpr int kMaxChunkLog2 = 3;
constexpr int kMaxChunkBlocks = 1 << kMaxChunkLog2;

template <int MAXB>
struct EncodeParams {
    uint32_t *ctl;
    unsigned long long *status;  // one look-back word per global chunk
    unsigned long long *group;   // one look-back word per group of kLbGroup chunks of a tensor
    const uint8_t *plans;
    unsigned long long *totals;  // per-tensor stream bytes out (may be null)
    int reuse;                   // plans give codebooks only: E and the total are found here
    uint32_t total_chunks;
    uint32_t total_jobs;         // chunks + empty tensors
    int T;
    int n_empty;
    int chunk_log2;              // blocks per chunk = 1 << chunk_log2
    const uint8_t *in[MAXB];
    uint8_t *out[MAXB];
    uint64_t n[MAXB];
    uint64_t cap[MAXB];
    uint32_t chunk_begin[MAXB + 1];  // prefix over tensors of their chunk counts
    uint16_t empty[MAXB];
    PageRef pg[MAXB];                // input pages
};

template <int MAXB>
struct DecodeParams {
    uint32_t *ctl;
    uint32_t *claim;     // per-tensor block counters, word t * kClaimStride (zero between calls)
    uint32_t total_blocks;
    int T;
    const uint8_t *comp[MAXB];
    uint64_t comp_bytes[MAXB];
    uint8_t *out[MAXB];
    uint64_t n[MAXB];
    uint32_t block_begin[MAXB + 1];  // prefix over tensors of their 4096-element blocks
    PageRef pg[MAXB];                // output pages
};

// Blocks per chunk for a launch.  Every chunk costs a claim, a look-back and a
// ring restart, so chunks are as long as the launch allows: 8 blocks if that
// still gives at least one chunk per two resident warps, else 2 blocks -- 1 if
// even that leaves fewer chunks than half the resident warps.  Measured: the
// Llama-3-8B and E5M2 batches and a cold Qwen3-32B layer are fastest in
// 8-block chunks; one Llama-3-8B or E5M2 layer (4096 or 8192 blocks) in 2-block
// chunks (1-block: 13% slower for Llama-3-8B; 4-block: 8% slower for E5M2).
inline int pick_chunk_log2(uint64_t total_blocks, uint64_t resident_warps) {
    if ((total_blocks >> kMaxChunkLog2) >= resident_warps / 2) return kMaxChunkLog2;
    return (total_blocks >> 1) >= resident_warps / 2 ? 1 : 0;
}

// ------------------------------------------------ programmatic dependent launch
// The plan and decode kernels are launched with programmatic stream
// serialization: each may start while the kernel before it on the stream is
// still running (after that kernel's CTAs have all called
// pdl_launch_dependents, or exited).  Before griddepcontrol.wait returns, a
// kernel touches nothing but its parameters and its shared memory; the wait
// returns once every kernel before it on the stream has completed and its
// memory is visible.  So a launch's fixed costs (launch, CTA placement,
// shared-memory set-up) overlap the previous kernel's tail, and the order of
// memory effects is that of plain stream order.  The encode kernel waits in
// the same way, so it is safe under either kind of launch; it is launched the
// ordinary way (see its launcher).

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// Launch kern<<<grid, block, smem, stream>>>(args...) with programmatic stream
// serialization allowed.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
                              cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------- device helpers

// Record the first device error; later errors keep the first one.
__device__ inline void set_error(uint32_t *ctl, uint32_t code, uint32_t detail) {
    if (atomicCAS(&ctl[kCtlErr], 0u, code) == 0u) atomicExch(&ctl[kCtlErrDetail], detail);
}

// Byte offset of element e from its tensor's base (PageRef above), or
// kBadOffset when the page id is outside the pool.  For paged tensors this
// reads one page id (read-only path).
constexpr uint64_t kBadOffset = ~0ull;
template <int EB>
__device__ __forceinline__ uint64_t elem_offset(const PageRef &pr, uint64_t e) {
    if (!pr.pages) return e * EB;
    const uint32_t page = uint32_t(e) / pr.page_elems;  // e < 2^32: tensors hold fewer than 2^32 elements
    const int64_t id = __ldg(pr.pages + page);
    if (id < 0 || uint64_t(id) >= pr.pool_pages) return kBadOffset;
    return uint64_t(id) * pr.page_bytes + (e - uint64_t(page) * pr.page_elems) * EB;
}

__device__ inline uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ inline unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ inline void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ inline uint32_t ld_relaxed_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ------------------------------------------------ bulk copies and mbarriers
// One-dimensional bulk copies global -> shared (the TMA engine, no tensor map),
// completed on an mbarrier by transaction bytes.  Addresses and sizes must be
// multiples of 16 bytes.  Every wait is bounded.

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the bulk-copy engine.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier shared-memory accesses before later bulk copies.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Pull [p, p + bytes) into L2 ahead of use (bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Shared-memory accesses by 32-bit shared address.
__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds_u64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds_u128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts_u8(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u8 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

__device__ __forceinline__ void sts_u64(uint32_t a, uint64_t v) {
    asm volatile("st.shared.u64 [%0], %1;" ::"r"(a), "l"(v) : "memory");
}

// Wait for the phase of the given parity to complete; false after limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > limit_ns) return false;
    return true;
}

// Index t with begin[t] <= x < begin[t+1] (begin non-decreasing, begin[0] = 0).
template <typename U, int MAXB>
__device__ inline int find_tensor(const U (&begin)[MAXB + 1], int T, U x) {
    int lo = 0, hi = T;  // invariant: begin[lo] <= x < begin[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (begin[mid] <= x) lo = mid; else hi = mid;
    }
    return lo;
}

// prmt.b32 in its default mode (PTX ISA, "prmt"): byte i of the result is
// byte (s_i & 7) of the pair {b, a} (a = bytes 0-3) when selector nibble s_i
// (bits 4i..4i+3 of s) is below 8, and that byte's top bit copied into all
// 8 bits when s_i >= 8.  Four table lookups of up to 8 bytes in one
// instruction.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
    return d;
}

// Exclusive prefix of c over the lanes of a warp; *total receives the warp's
// sum.  When no lane has c > 1 (escapes are rare) the prefix is a popcount of
// the lanes below with c = 1; otherwise a shuffle scan.
__device__ __forceinline__ uint32_t warp_exclusive_prefix(uint32_t c, uint32_t *total) {
    const uint32_t any = __ballot_sync(0xffffffffu, c != 0);
    if (any == 0) {
        *total = 0;
        return 0;
    }
    const int lane = threadIdx.x & 31;
    if (__ballot_sync(0xffffffffu, c > 1) == 0) {
        *total = __popc(any);
        return __popc(any & ((1u << lane) - 1u));
    }
    uint32_t x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    *total = __shfl_sync(0xffffffffu, x, 31);
    return x - c;
}

// Lanes below this one (bit i set for lane i < this lane).
__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Nibble flags of the escape code 15 among 8 packed 4-bit codes: bit 4j set
// when code j is 15.
__device__ __forceinline__ uint32_t escape_nibbles(uint32_t cw) {
    const uint32_t t = cw & (cw >> 1);
    return t & (t >> 2) & 0x11111111u;
}

// Exclusive prefix sum over the CTA (NT threads); *total receives the sum.
template <int NT>
__device__ inline uint32_t block_exclusive_scan(uint32_t v, uint32_t *s_warp, uint32_t *total) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        uint32_t s = s_warp[w];
        before += (w < warp) ? s : 0u;
        all += s;
    }
    *total = all;
    return before + x - v;
}

// w[i] for a small runtime index without spilling the array to local memory.
__device__ __forceinline__ uint32_t pick4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t i) {
    const uint32_t lo = (i & 1u) ? w1 : w0;
    const uint32_t hi = (i & 1u) ? w3 : w2;
    return (i & 2u) ? hi : lo;
}

// Plan words (the 64-byte header as 16 little-endian u32 words).
struct Header {
    uint32_t magic, vtag;  // vtag = version | dtype << 16 | block_log2 << 24
    uint64_t n, E, total;
    uint32_t cbw[4];       // cb[0..14] in bytes 0..14, byte 15 the flags
};

__device__ inline Header load_header(const uint8_t *h) {
    const uint32_t *w = reinterpret_cast<const uint32_t *>(h);
    Header H;
    H.magic = w[0];
    H.vtag = w[1];
    H.n = uint64_t(w[2]) | (uint64_t(w[3]) << 32);
    H.E = uint64_t(w[4]) | (uint64_t(w[5]) << 32);
    H.cbw[0] = w[6];
    H.cbw[1] = w[7];
    H.cbw[2] = w[8];
    H.cbw[3] = w[9];
    H.total = uint64_t(w[10]) | (uint64_t(w[11]) << 32);
    return H;
}

__device__ inline uint32_t header_vtag(int dtype) {
    return kVersion | (uint32_t(dtype) << 16) | (kBlockLog2 << 24);
}

__device__ inline uint32_t cb_byte(const uint32_t (&cbw)[4], int c) {
    return (pick4(cbw[0], cbw[1], cbw[2], cbw[3], uint32_t(c) >> 2) >> (8 * (c & 3))) & 0xFFu;
}

}  // namespace sz
