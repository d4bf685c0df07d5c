// sz_plan.cu -- plan kernel: exponent histogram + top-15 codebook selection.
//
// SplitZip project page, Abstract: the codec gives fixed 4-bit codes to "the
// most frequent exponent values".  This kernel counts every exponent value of
// each tensor and, in the last CTA to finish a tensor, ranks the values by
// (count descending, value ascending), takes the first 15 as the codebook and
// writes the 64-byte plan (= stream header: n, E, codebook, total bytes).
//
// Histogram design (B200): counters live in shared memory as 16-bit halves of
// 32-bit words.  Word (e, c) at s_cols[e * NT/2 + c] holds two counts of
// exponent value e: the low half belongs to thread c, the high half to thread
// c + NT/2.  A thread therefore adds a constant (1 or 1 << 16) to one word per
// element: a shift, a mask and one shared-memory atomic.  Lane l of any warp
// always hits bank l % 32 and no two lanes of a warp share a word, so the
// atomics never conflict and never contend, whatever the exponent
// distribution (an all-zero tensor costs the same as a spread one).  Counters
// are flushed to the tensor's global histogram (one atomic per non-zero bin
// per CTA) before any thread can have counted 65535 elements.  Input is
// streamed with 16-byte read-only loads, a software-pipelined batch of U
// vectors per thread in flight.
#include "sz_common.cuh"
#include "sz_internal.h"

namespace sz {

namespace {

constexpr int kPlanThreads = 256;
// 16-byte vectors in flight per thread: the kernel has one CTA of 8 warps per
// SM, so its loads in flight decide how close it gets to the HBM bandwidth.
// BF16 runs fastest with 16 (242 registers), E5M2 with 12 (measured).
template <int DT>
constexpr int plan_unroll() { return DT == SZ_BF16 ? 16 : 12; }
constexpr uint32_t kItemBytes = 16384;        // partition unit of the input
constexpr uint32_t kMaxPerThread = 65535;     // 16-bit counter limit

template <int DT>
struct PlanCfg {
    static constexpr int kBins = Dt<DT>::kBins;
    static constexpr int kElemBytes = Dt<DT>::kElemBytes;
    static constexpr int kVecElems = 16 / kElemBytes;       // elements per 16-byte vector
    static constexpr uint32_t kItemElems = kItemBytes / kElemBytes;
};

// Add inc to the shared-memory word at addr (no return value needed).
__device__ __forceinline__ void red_shared_add(uint32_t addr, uint32_t inc) {
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(addr), "r"(inc) : "memory");
}

// Count the elements of one 16-byte vector.  col = shared address of this
// thread's column (s_cols + tid % (NT/2)); inc = its half (1 or 1 << 16).
template <int DT, int NT>
__device__ __forceinline__ void count_vec(uint32_t col, uint32_t inc, uint4 v) {
    constexpr uint32_t kRowBytes = NT / 2 * 4;  // bytes per exponent value
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if constexpr (DT == SZ_BF16) {
            // two elements per word: exponent bits 7..14 and 23..30
            red_shared_add(col + ((w[k] >> 7) & 0xFFu) * kRowBytes, inc);
            red_shared_add(col + ((w[k] >> 23) & 0xFFu) * kRowBytes, inc);
        } else {
            // four elements per word: exponent bits 2..6 of each byte, all four
            // extracted by one shift and mask, then each moved to byte 0 by a
            // byte permute (about 2.5 integer ops per element instead of 3)
            const uint32_t x = (w[k] >> 2) & 0x1F1F1F1Fu;
#pragma unroll
            for (int b = 0; b < 4; ++b)
                red_shared_add(col + __byte_perm(x, 0u, 0x4440u + uint32_t(b)) * kRowBytes, inc);
        }
    }
}

template <int DT>
__device__ __forceinline__ uint32_t exponent_scalar(const uint8_t *in, uint64_t i) {
    if constexpr (DT == SZ_BF16) {
        const uint32_t b = reinterpret_cast<const uint16_t *>(in)[i];
        return (b >> 7) & 0xFFu;
    } else {
        return (uint32_t(in[i]) >> 2) & 0x1Fu;
    }
}

// Count elements [a, b) of one tensor (a is a multiple of the vector size).
// Batches of U vectors per thread are software-pipelined: the next batch is
// loaded while the current one is counted.  Only the last, partial batch needs
// bounds checks.
template <int DT, int NT>
__device__ void count_range(uint32_t col, uint32_t inc, const uint8_t *in, uint64_t a, uint64_t b) {
    using C = PlanCfg<DT>;
    constexpr int U = plan_unroll<DT>();
    constexpr uint32_t kBatch = uint32_t(U) * NT;
    const int tid = threadIdx.x;
    const uint4 *src = reinterpret_cast<const uint4 *>(in) + a / C::kVecElems + tid;
    const uint32_t nvec = uint32_t((b - a) / C::kVecElems);  // < 2^29: sub-ranges are short
    const uint32_t full = nvec / kBatch;                       // batches with every vector in range
    auto load_checked = [&](uint4 (&dst)[U], uint32_t base) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t k = base + uint32_t(tid) + uint32_t(u) * NT;
            dst[u] = k < nvec ? __ldg(src + (base + uint32_t(u) * NT)) : make_uint4(0, 0, 0, 0);
        }
    };
    uint4 cur[U];
    if (full > 0) {
#pragma unroll
        for (int u = 0; u < U; ++u) cur[u] = __ldg(src + uint32_t(u) * NT);
    } else {
        load_checked(cur, 0);
    }
    for (uint32_t bi = 0; bi < full; ++bi) {
        uint4 nxt[U];
        const uint32_t nbase = (bi + 1) * kBatch;
        if (bi + 1 < full) {
#pragma unroll
            for (int u = 0; u < U; ++u) nxt[u] = __ldg(src + (nbase + uint32_t(u) * NT));
        } else {
            load_checked(nxt, nbase);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) count_vec<DT, NT>(col, inc, cur[u]);
#pragma unroll
        for (int u = 0; u < U; ++u) cur[u] = nxt[u];
    }
    // the partial batch (already loaded, zero past the end)
    const uint32_t tail = full * kBatch;
#pragma unroll
    for (int u = 0; u < U; ++u)
        if (tail + uint32_t(tid) + uint32_t(u) * NT < nvec) count_vec<DT, NT>(col, inc, cur[u]);
    // ragged end (< one vector): thread 0 counts it element by element
    if (tid == 0) {
        for (uint64_t i = a + uint64_t(nvec) * C::kVecElems; i < b; ++i)
            red_shared_add(col + exponent_scalar<DT>(in, i) * (NT / 2 * 4), inc);
    }
}

// Page ids cached in shared memory per pass of count_range_paged.
constexpr uint32_t kPageCache = 4096;

// Count elements [a, b) of a paged tensor (a a multiple of the vector size);
// called by the whole CTA.  The range's page ids are first copied into shared
// memory (s_ids, kPageCache at a time).  Each warp then streams whole pages of
// the range, U vectors per lane ahead, so that an SM reads several pages at
// once wherever they lie in the pool.  A page id outside the pool sets *bad and
// that page is not counted.
template <int DT, int NT>
__device__ void count_range_paged(uint32_t col, uint32_t inc, const uint8_t *pool, const PageRef &pr,
                                  uint64_t a, uint64_t b, int32_t *s_ids, bool *bad) {
    using C = PlanCfg<DT>;
    constexpr int U = plan_unroll<DT>();
    const int tid = threadIdx.x;
    const uint64_t pe = pr.page_elems;
    // whole vectors only; the ragged end (< one vector) is counted below
    const uint64_t b_vec = a + (b - a) / C::kVecElems * C::kVecElems;
    for (uint64_t p0 = a / pe; p0 * pe < b_vec; p0 += kPageCache) {
        const uint64_t lo = max(a, p0 * pe), hi = min(b_vec, (p0 + kPageCache) * pe);
        const uint32_t npg = uint32_t((hi - 1) / pe - p0 + 1);
        __syncthreads();  // the previous pass is done with s_ids
        for (uint32_t i = tid; i < npg; i += NT) s_ids[i] = __ldg(pr.pages + p0 + i);
        __syncthreads();
        // warp w takes pages w, w + NW, ... of the pass: every warp streams its own
        // page, so an SM has NW pages in flight (pages lie anywhere in the pool)
        constexpr int NW = NT / 32;
        const int warp = tid >> 5, lane = tid & 31;
        for (uint32_t j = uint32_t(warp); j < npg; j += NW) {
            const uint64_t ps = (p0 + j) * pe;
            const uint64_t x = max(lo, ps), y = min(hi, ps + pe);
            const int32_t id = s_ids[j];
            if (id < 0 || uint64_t(id) >= pr.pool_pages) {
                *bad = true;
                continue;
            }
            const uint4 *src = reinterpret_cast<const uint4 *>(pool + uint64_t(id) * pr.page_bytes +
                                                                (x - ps) * C::kElemBytes);
            const uint32_t nvec = uint32_t((y - x) / C::kVecElems);
            uint4 cur[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t k = uint32_t(lane) + uint32_t(u) * 32;
                cur[u] = k < nvec ? __ldg(src + k) : make_uint4(0, 0, 0, 0);
            }
            for (uint32_t base = 0; base < nvec; base += uint32_t(U) * 32) {
                uint4 nxt[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const uint32_t k = base + uint32_t(U) * 32 + uint32_t(lane) + uint32_t(u) * 32;
                    nxt[u] = k < nvec ? __ldg(src + k) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (base + uint32_t(lane) + uint32_t(u) * 32 < nvec) count_vec<DT, NT>(col, inc, cur[u]);
#pragma unroll
                for (int u = 0; u < U; ++u) cur[u] = nxt[u];
            }
        }
    }
    // ragged end (< one vector): thread 0 counts it element by element
    if (tid == 0) {
        for (uint64_t i = b_vec; i < b; ++i) {
            const uint64_t off = elem_offset<C::kElemBytes>(pr, i);
            if (off == kBadOffset) {
                *bad = true;
                continue;
            }
            red_shared_add(col + exponent_scalar<DT>(pool + off, 0) * (NT / 2 * 4), inc);
        }
    }
}

// Add every column into the global histogram g_hist and clear them: a warp
// takes one exponent row at a time, one 16-byte load and store per lane.
template <int DT, int NT>
__device__ void flush_columns(uint32_t *s_cols, uint32_t *g_hist) {
    using C = PlanCfg<DT>;
    constexpr int kRowVecs = NT / 2 / 4;  // 16-byte vectors per exponent row
    static_assert(kRowVecs == 32, "one vector per lane per row");
    uint4 *rows = reinterpret_cast<uint4 *>(s_cols);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    for (int e = warp; e < C::kBins; e += NT / 32) {
        const uint4 w = rows[e * kRowVecs + lane];
        rows[e * kRowVecs + lane] = make_uint4(0, 0, 0, 0);
        uint32_t sum = (w.x & 0xFFFFu) + (w.x >> 16) + (w.y & 0xFFFFu) + (w.y >> 16) + (w.z & 0xFFFFu) +
                       (w.z >> 16) + (w.w & 0xFFFFu) + (w.w >> 16);
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0 && sum) atomicAdd(g_hist + e, sum);
    }
    __threadfence();
    __syncthreads();
}

// Write a 64-byte plan (16 words) from thread-0 values kept in shared memory.
__device__ inline void store_plan(uint8_t *plan, const uint32_t *s_words) {
    if (threadIdx.x < 16) reinterpret_cast<uint32_t *>(plan)[threadIdx.x] = s_words[threadIdx.x];
}

__device__ inline void make_plan_words(uint32_t *s_words, int dtype, uint64_t n, uint64_t E,
                                       const uint8_t *cb) {
    const Layout L = stream_layout(dtype, n, E);
    s_words[0] = kMagic;
    s_words[1] = header_vtag(dtype);
    s_words[2] = uint32_t(n);
    s_words[3] = uint32_t(n >> 32);
    s_words[4] = uint32_t(E);
    s_words[5] = uint32_t(E >> 32);
    for (int q = 0; q < 4; ++q) {
        uint32_t w = 0;
        for (int b = 0; b < 4; ++b) {
            const int c = 4 * q + b;
            if (c < int(kCodes)) w |= uint32_t(cb[c]) << (8 * b);
        }
        s_words[6 + q] = w;
    }
    s_words[10] = uint32_t(L.total);
    s_words[11] = uint32_t(L.total >> 32);
    s_words[12] = s_words[13] = s_words[14] = s_words[15] = 0;
}

// Shared scratch of the codebook selection.
template <int DT>
struct SelectSmem {
    uint32_t cnt[Dt<DT>::kBins];   // the tensor's histogram
    uint32_t list_cnt[Dt<DT>::kBins];  // its non-zero bins, in no particular order
    uint8_t list_val[Dt<DT>::kBins];
    uint32_t nnz, sum;
    uint8_t cb[16];
    uint32_t words[16];
};

// Rank every exponent value by (count desc, value asc); write the plan of a
// tensor of n elements; leave its histogram and ticket zeroed for reuse.  A
// value's rank counts the values ahead of it in that order; only the non-zero
// bins are compared (a zero bin comes after all of them, and among zero bins
// the smaller value first), so the work follows the number of distinct
// exponents, not the 256 possible ones.
template <int DT, int NT>
__device__ void select_codebook(uint32_t *g_hist, uint32_t *g_ticket, uint64_t n, uint8_t *plan, uint32_t *ctl,
                                SelectSmem<DT> &S) {
    using C = PlanCfg<DT>;
    static_assert(C::kBins <= NT, "one bin per thread");
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) S.nnz = S.sum = 0;
    __syncthreads();
    const uint32_t c = tid < C::kBins ? __ldcg(g_hist + tid) : 0u;
    if (tid < C::kBins) {
        S.cnt[tid] = c;
        if (c) {
            const uint32_t pos = atomicAdd(&S.nnz, 1u);
            S.list_cnt[pos] = c;
            S.list_val[pos] = uint8_t(tid);
        }
    }
    const uint32_t wsum = __reduce_add_sync(0xffffffffu, c);  // n < 2^32: no overflow
    if (lane == 0 && wsum) atomicAdd(&S.sum, wsum);
    __syncthreads();
    if (tid < C::kBins) {
        const uint32_t nnz = S.nnz, v = uint32_t(tid);
        uint32_t rank = kCodes;
        if (c) {
            rank = 0;
            for (uint32_t j = 0; j < nnz; ++j) {
                const uint32_t cu = S.list_cnt[j], u = S.list_val[j];
                rank += (cu > c) | ((cu == c) & (u < v));
            }
        } else if (nnz < kCodes) {
            uint32_t below = 0;  // non-zero bins of smaller value
            for (uint32_t j = 0; j < nnz; ++j) below += S.list_val[j] < v;
            rank = nnz + (v - below);
        }
        if (rank < kCodes) S.cb[rank] = uint8_t(v);
    }
    __syncthreads();
    if (tid == 0) {
        uint64_t covered = 0;
        for (int k = 0; k < int(kCodes); ++k) covered += S.cnt[S.cb[k]];
        if (S.sum != n) set_error(ctl, SZ_ERR_INTERNAL, 1);
        make_plan_words(S.words, DT, n, n - covered, S.cb);
    }
    __syncthreads();
    store_plan(plan, S.words);
    if (tid < C::kBins) g_hist[tid] = 0;
    if (tid == 0) *g_ticket = 0;
}

template <int DT, int NT, int MAXB>
__global__ void __launch_bounds__(NT, 1) plan_kernel(const __grid_constant__ PlanParams<MAXB> p) {
    using C = PlanCfg<DT>;
    extern __shared__ uint32_t s_cols[];  // C::kBins * NT/2 words of two 16-bit counters, then page ids
    int32_t *s_ids = reinterpret_cast<int32_t *>(s_cols + C::kBins * (NT / 2));
    __shared__ SelectSmem<DT> s_sel;
    __shared__ uint32_t s_last;
    const int tid = threadIdx.x;
    const uint32_t col = smem_u32(s_cols + (tid % (NT / 2)));
    const uint32_t inc = 1u << (16 * (tid / (NT / 2)));
    const uint64_t lo = p.total_items * blockIdx.x / gridDim.x;
    const uint64_t hi = p.total_items * (blockIdx.x + 1) / gridDim.x;
    // shared-memory set-up overlaps the previous kernel (programmatic launch)
    if (lo < hi) {
        for (int i = tid; i < C::kBins * (NT / 2) / 4; i += NT)
            reinterpret_cast<uint4 *>(s_cols)[i] = make_uint4(0, 0, 0, 0);
    }
    pdl_wait();
    pdl_launch_dependents();

    // Plans of empty tensors: codebook of the 15 smallest values, E = 0.
    if (blockIdx.x == 0) {
        for (int t = 0; t < p.T; ++t) {
            if (p.n[t] != 0) continue;
            if (tid == 0) {
                uint8_t cb[kCodes];
                for (int c = 0; c < int(kCodes); ++c) cb[c] = uint8_t(c);
                make_plan_words(s_sel.words, DT, 0, 0, cb);
            }
            __syncthreads();
            store_plan(p.plans + 64 * size_t(t), s_sel.words);
            __syncthreads();
        }
    }

    if (lo >= hi) return;
    __syncthreads();

    int t = find_tensor<uint64_t, MAXB>(p.item_begin, p.T, lo);
    uint64_t i = lo;
    while (i < hi) {
        while (p.item_begin[t + 1] <= i) ++t;  // skip tensors without items
        const uint64_t i_end = min(hi, p.item_begin[t + 1]);
        const uint64_t a = (i - p.item_begin[t]) * C::kItemElems;
        const uint64_t b = min(p.n[t], (i_end - p.item_begin[t]) * C::kItemElems);
        uint32_t *g_hist = p.hist + size_t(t) * 256;
        // sub-ranges short enough that no 16-bit counter can overflow
        constexpr uint64_t kSub = uint64_t(kMaxPerThread / C::kVecElems) * C::kVecElems * NT;
        const PageRef &pr = p.pg[t];
        // Paged ranges are counted page by page per warp, so one lane may see up to
        // range / NT + 1.25 page / 32 elements: half-size sub-ranges keep that below
        // 65535 for pages of up to 2^18 elements (the host's limit).
        constexpr uint64_t kSubPaged = uint64_t(kMaxPerThread / 2) * NT;
        const uint64_t sub = pr.pages ? kSubPaged : kSub;
        for (uint64_t s = a; s < b; s += sub) {
            const uint64_t e = min(b, s + sub);
            if (!pr.pages) {
                count_range<DT, NT>(col, inc, p.in[t], s, e);
            } else {
                bool bad = false;
                count_range_paged<DT, NT>(col, inc, p.in[t], pr, s, e, s_ids, &bad);
                if (bad) set_error(p.ctl, SZ_ERR_INVALID_ARG, uint32_t(t));
            }
            flush_columns<DT, NT>(s_cols, g_hist);
        }
        // ticket: the CTA that completes the tensor's last item selects its codebook
        if (tid == 0) {
            const uint32_t items = uint32_t(i_end - i);
            const uint32_t need = uint32_t(p.item_begin[t + 1] - p.item_begin[t]);
            const uint32_t done = atomicAdd(p.ticket + t, items) + items;
            s_last = (done == need);
            __threadfence();
        }
        __syncthreads();
        if (s_last) {
            select_codebook<DT, NT>(g_hist, p.ticket + t, p.n[t], p.plans + 64 * size_t(t), p.ctl, s_sel);
            __syncthreads();
        }
        i = i_end;
    }
}

template <int DT, int MAXB>
sz_status launch_plan_t(const PlanArgs &a, cudaStream_t stream) {
    using C = PlanCfg<DT>;
    constexpr int NT = kPlanThreads;
    PlanParams<MAXB> p;
    p.ctl = a.ctl;
    p.hist = a.hist;
    p.ticket = a.ticket;
    p.plans = a.plans;
    p.T = a.T;
    p.item_begin[0] = 0;
    for (int t = 0; t < a.T; ++t) p.pg[t] = page_ref(a.paged ? a.paged + t : nullptr);
    for (int t = 0; t < a.T; ++t) {
        p.in[t] = static_cast<const uint8_t *>(a.in[t]);
        p.n[t] = a.n[t];
        p.item_begin[t + 1] = p.item_begin[t] + cdiv(a.n[t], C::kItemElems);
    }
    p.total_items = p.item_begin[a.T];
    bool any_paged = false;
    for (int t = 0; t < a.T; ++t) any_paged = any_paged || (a.paged && a.paged[t].pages && a.n[t]);
    const size_t smem = size_t(C::kBins) * (NT / 2) * 4 + (any_paged ? size_t(kPageCache) * 4 : 0);
    auto kern = plan_kernel<DT, NT, MAXB>;
    // the kernel's shared-memory limit is set once, for the larger (paged) need
    const size_t smem_max = size_t(C::kBins) * (NT / 2) * 4 + size_t(kPageCache) * 4;
    static std::atomic<int> cache[kMaxDevices];
    const int per_sm = resident_per_sm(reinterpret_cast<const void *>(kern), NT, smem_max, cache);
    if (per_sm < 1) return SZ_ERR_CUDA;
    uint64_t grid = uint64_t(a.num_sms) * per_sm;
    if (p.total_items < grid) grid = p.total_items;
    if (grid == 0) grid = 1;  // only empty tensors: block 0 writes their plans
    return launch_pdl(kern, unsigned(grid), NT, smem, stream, p) == cudaSuccess ? SZ_OK : SZ_ERR_CUDA;
}

}  // namespace

sz_status launch_plan(const PlanArgs &a, cudaStream_t stream) {
    if (a.dtype == SZ_BF16)
        return a.T <= kSmallBatch ? launch_plan_t<SZ_BF16, kSmallBatch>(a, stream)
                                  : launch_plan_t<SZ_BF16, kLargeBatch>(a, stream);
    return a.T <= kSmallBatch ? launch_plan_t<SZ_FP8_E5M2, kSmallBatch>(a, stream)
                              : launch_plan_t<SZ_FP8_E5M2, kLargeBatch>(a, stream);
}

}  // namespace sz
