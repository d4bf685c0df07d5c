// sz_encode.cu -- encode kernel: split, code, pack, escape offsets and scatter.
//
// SplitZip project page, Abstract: sign and mantissa bits are kept exactly,
// frequent exponents get fixed 4-bit codes, rare exponents go to a sparse
// escape stream.  Persistent CTAs of independent warps (8 per CTA for BF16, 12
// for E5M2; no CTA barrier on the path).  Each warp takes chunks -- 1 to 8 consecutive 4096-element blocks of
// one tensor, short chunks for small batches -- in launch order from an atomic
// counter:
//   1. the chunk's input arrives by 1-D bulk copies of 2 KB units into the
//      warp's 3-stage shared-memory ring (bounded mbarrier waits);
//   2. per step a lane codes 8 (BF16) or 16 (E5M2) elements from one 16-byte
//      shared load: exponent -> code through a 256-byte table whose entry
//      address one prmt forms, sign|mantissa planes and 4-bit codes written
//      with coalesced stores; escapes ranked by ballots (a fast path when no
//      lane has two; E5M2's takes one flag bit per escape and the exponent
//      with one byte permute) and staged in element order in the warp's stage;
//   3. the chunk's escape offset comes from a single-pass decoupled look-back
//      over the chunks of its tensor, on two levels (the chunk's own group of
//      32 chunks, then whole groups, 32 per round); a chunk whose predecessors
//      have not yet published is finished once the warp has coded its next
//      chunk; every wait is bounded: SZ_ERR_TIMEOUT instead of a hang;
//   4. the chunk's offsets-table entries and escapes are written contiguously
//      (a chunk whose escapes overflow the stage re-codes its input and writes
//      them directly); the tensor's last chunk writes the header, offsets[nb]
//      and the zero padding;
//   5. with raw blocks allowed (header flag), a block whose escapes reach its
//      raw size is stored raw: its chunk re-reads the input, writes the low
//      exponent nibbles over the codes and the high bits to the escape
//      section, and the last chunk writes the exact E and total.
#include <type_traits>

#include "sz_common.cuh"
#include "sz_internal.h"

namespace sz {

namespace {

// Persistent CTAs of independent warps, 24 per SM at 80 registers: 3 CTAs of
// 8 warps for BF16, 2 CTAs of 12 for E5M2 (measured best among 2 x 8 warps at
// 128 registers, 2 x 10 at 96, 3 x 7 at 96 and 2 x 12 at 80, with the E5M2
// step loop rolled).  One CTA of 24 warps per SM was the same on large batches
// and slower on one Qwen3-32B layer (0.70 against 0.76 of the HBM peak).
template <int DT>
constexpr int enc_threads() { return DT == SZ_BF16 ? kTileThreads : 384; }
template <int DT>
constexpr int enc_ctas_per_sm() { return DT == SZ_BF16 ? 3 : 2; }
constexpr int kChunkBlocks = kMaxChunkBlocks;         // a warp's unit of work: up to 8 consecutive blocks
constexpr uint32_t kWarpStage = 1024;                 // staged escape bytes per chunk (two chunks)
constexpr int kRing = 3;                              // input-unit stages per warp
constexpr uint32_t kUnitBytes = 2048;                 // one input unit: a quarter block (BF16) or half a block (E5M2)
constexpr uint64_t kLookbackLimitNs = 1000000000ull;  // 1 s: far above any legitimate wait
constexpr uint64_t kWaitLimitNs = 1000000000ull;      // bulk-copy wait limit
constexpr unsigned long long kFlagAgg = 1ull << 32;   // chunk aggregate published
constexpr unsigned long long kFlagInc = 2ull << 32;   // inclusive prefix published

// Each warp works alone: its own input ring (bulk copies of 2 KB units),
// plan header, exponent -> code table, and two escape stages (the chunk being
// coded and one whose offset is still being looked up).
struct alignas(128) WarpShared {
    uint8_t ring[kRing][kUnitBytes];
    uint64_t bar[kRing];
    uint32_t hdr[16];
    uint32_t blk_off[2][kChunkBlocks];  // escapes before each block, within the chunk
    uint8_t lut_raw[512];  // holds the 256-byte-aligned code table (lut_addr)
    uint8_t esc[2][kWarpStage];
};

template <int DT>
struct Geo {
    static constexpr int LE = (DT == SZ_BF16) ? 8 : 16;    // elements per lane per step
    static constexpr int IT = int(kBlock) / (32 * LE);      // steps per block
    static constexpr int kAhead = 3;                        // steps of loads in flight
};

// Decoupled look-back of one chunk, run by one warp and resumable, on two
// levels.  Status words (per chunk, and per group of kLbGroup consecutive
// chunks of a tensor): epoch (30 bits) << 34 | flag << 32 | value; words of
// earlier launches carry an older epoch and read as "not published".  A chunk
// word holds the chunk's escape count (flag kFlagAgg) or its inclusive prefix
// (kFlagInc); a group word holds the sum of its chunks (kFlagAgg) or the
// inclusive prefix through its last chunk (kFlagInc).
//   Phase 1: the chunk's own group -- the up to 31 predecessors in it, one per
//   lane -- summed back to the nearest inclusive prefix.
//   Phase 2: whole groups, 32 per round (1024 chunks), summed back to the
//   nearest inclusive group word; the start of the tensor counts as an
//   inclusive prefix of 0.  A needed group word not yet published is made by
//   the warp itself from the group's chunk words, once they are all published.
// Group words are also published by the last chunk of each group, right after
// its own aggregate (if the group's other chunks are done) and with its own
// inclusive prefix.  Every chunk publishes its aggregate as soon as it has
// coded its chunk, without waiting on anything, so a look-back always ends;
// the total wait is still bounded (SZ_ERR_TIMEOUT).  When every chunk of a
// launch finishes at about the same time (one chunk per warp), a one-level
// look-back needs some j / 256 dependent rounds for chunk j; two levels need
// two or three.  Measured variants: 512 predecessors per one-level round made
// every encode slower; retrying a deferred look-back between the blocks of
// the warp's next chunk (each try stalls the warp for an L2 round trip) made
// the Llama-3-8B batch encode 4% and one Qwen3-32B layer 8% slower than
// settling it once, after that chunk.
struct Lookback {
    int32_t j;      // phase 1: nearest unsummed predecessor; phase 2: nearest unsummed group
    uint32_t excl;  // escapes summed so far
    uint32_t t0;    // low bits of the time a predecessor was first found unpublished
    uint32_t flags; // kLbDone | kLbTimedOut | kLbWaiting | kLbGroups
};
constexpr uint32_t kLbDone = 1, kLbTimedOut = 2, kLbWaiting = 4, kLbGroups = 8;

// A tensor's look-back words: its chunk words, its group words, its chunk count.
struct LbWords {
    unsigned long long *st, *gs;
    uint32_t nchunks;
};

// Flag (0: not published in this launch) and value of a status word.
__device__ __forceinline__ uint32_t lb_flag(unsigned long long w, unsigned long long tag) {
    return ((w >> 34) == (tag >> 34)) ? uint32_t(w >> 32) & 3u : 0u;
}

// Publish word w (flag f) for group g unless it already holds as much (an
// inclusive prefix beats an aggregate); one compare-and-swap, losing a race
// to another publisher is fine (both words are true).
__device__ __forceinline__ void publish_group(const LbWords &c, uint32_t g, unsigned long long w,
                                              unsigned long long tag) {
    const unsigned long long cur = ld_relaxed_u64(c.gs + g);
    if (lb_flag(cur, tag) < lb_flag(w, tag)) atomicCAS(c.gs + g, cur, w);
}

// Try to make group g's word from its chunk words (one round, warp-wide):
// true if it is published now.
__device__ bool make_group(const LbWords &c, uint32_t g, unsigned long long tag) {
    const int lane = threadIdx.x & 31;
    const uint32_t k = (g << kLbGroupLog2) + uint32_t(lane);
    uint32_t f = 2, v = 0;  // chunks past the tensor's end: nothing to add
    if (k < c.nchunks) {
        const unsigned long long w = ld_relaxed_u64(c.st + k);
        f = lb_flag(w, tag);
        v = uint32_t(w);
    }
    if (!__all_sync(0xffffffffu, f != 0)) return false;
    // the last inclusive prefix among the group's chunks, then the aggregates after it
    const uint32_t inc = __ballot_sync(0xffffffffu, k < c.nchunks && f == 2);
    const int L = inc ? 31 - __clz(inc) : -1;
    const uint32_t sum = __reduce_add_sync(0xffffffffu, (lane >= L && k < c.nchunks) ? v : 0u);
    if (lane == 0)
        publish_group(c, g, tag | (L >= 0 ? kFlagInc : kFlagAgg) | sum, tag);
    return true;
}

__device__ __forceinline__ void lookback_start(Lookback &lb, const LbWords &c, uint32_t chunk, uint32_t agg,
                                               unsigned long long tag) {
    const int lane = threadIdx.x & 31;
    lb.excl = 0;
    lb.t0 = 0;
    lb.flags = chunk == 0 ? kLbDone : 0u;
    lb.j = int32_t(chunk) - 1;
    if (chunk != 0 && (chunk & (kLbGroup - 1)) == 0) {  // first chunk of its group: no phase 1
        lb.flags |= kLbGroups;
        lb.j = int32_t(chunk >> kLbGroupLog2) - 1;
    }
    if (lane == 0) st_relaxed_u64(c.st + chunk, tag | (chunk == 0 ? kFlagInc : kFlagAgg) | agg);
    // the last chunk of a group publishes the group's word if the others are done
    if ((chunk & (kLbGroup - 1)) == kLbGroup - 1 || chunk + 1 == c.nchunks) {
        __syncwarp();
        make_group(c, chunk >> kLbGroupLog2, tag);
    }
}

// Sum published predecessors of chunk (own count agg); with `block`, wait
// until done.  Returns true once the chunk's offset is known.
__device__ bool lookback_advance(Lookback &lb, const LbWords &c, uint32_t chunk, uint32_t agg,
                                 unsigned long long tag, bool block) {
    const int lane = threadIdx.x & 31;
    uint32_t backoff = 32;
    while (!(lb.flags & kLbDone)) {
        const bool groups = (lb.flags & kLbGroups) != 0;
        // phase 1: predecessor lb.j - lane of the own group; phase 2: group lb.j - lane
        const int32_t first = groups ? 0 : int32_t(chunk & ~(kLbGroup - 1));
        const int32_t idx = lb.j - lane;
        uint32_t f = 2, v = 0;  // before the group's (phase 1) or tensor's (phase 2) start: inclusive 0
        if (idx >= first) {
            const unsigned long long w = ld_relaxed_u64((groups ? c.gs : c.st) + idx);
            f = lb_flag(w, tag);
            v = uint32_t(w);
        } else if (!groups) {
            f = 3;  // phase 1 past the own group's start: not needed, ends the phase
        }
        const uint32_t stop = __ballot_sync(0xffffffffu, f >= 2);
        const int L = stop ? __ffs(stop) - 1 : 32;  // nearest inclusive prefix (or phase end)
        const bool need = lane < L || (lane == L && f == 2);
        if (__all_sync(0xffffffffu, !need || f != 0)) {
            lb.excl += __reduce_add_sync(0xffffffffu, need ? v : 0u);
            if (L < 32 && __shfl_sync(0xffffffffu, f, L) == 2) {
                lb.flags |= kLbDone;
                break;
            }
            if (groups) {
                lb.j -= 32;
            } else {  // own group summed: continue with the groups before it
                lb.flags |= kLbGroups;
                lb.j = int32_t(chunk >> kLbGroupLog2) - 1;
                if (lb.j < 0) {
                    lb.flags |= kLbDone;
                    break;
                }
            }
            continue;
        }
        if (groups) {
            // make the nearest missing group word, then try again at once
            const uint32_t miss = __ballot_sync(0xffffffffu, need && f == 0);
            if (make_group(c, uint32_t(lb.j - (__ffs(miss) - 1)), tag)) continue;
        }
        const uint32_t now = __shfl_sync(0xffffffffu, uint32_t(global_ns()), 0);
        if (!(lb.flags & kLbWaiting)) {
            lb.flags |= kLbWaiting;
            lb.t0 = now;
        } else if (now - lb.t0 > uint32_t(kLookbackLimitNs)) {  // unsigned: correct across wrap
            lb.flags |= kLbDone | kLbTimedOut;
            break;
        }
        if (!block) return false;
        __nanosleep(backoff);
        if (backoff < 256) backoff <<= 1;
    }
    if (chunk != 0 && lane == 0) {
        const unsigned long long w = tag | kFlagInc | (lb.excl + agg);
        st_relaxed_u64(c.st + chunk, w);
        // the last chunk of a group: its inclusive prefix is the group's
        if ((chunk & (kLbGroup - 1)) == kLbGroup - 1 || chunk + 1 == c.nchunks)
            publish_group(c, chunk >> kLbGroupLog2, w, tag);
    }
    return true;
}

// Header flags (byte 39).
__device__ __forceinline__ uint32_t header_flags(const Header &H) { return H.cbw[3] >> 24; }

// The plan's codebook: 15 distinct values inside the exponent range, and
// flags no other than kFlagRawBlocks (one lane per entry; warp-wide).
template <int DT>
__device__ __forceinline__ bool codebook_ok(const Header &H) {
    const int lane = threadIdx.x & 31;
    bool ok = (header_flags(H) & ~kFlagRawBlocks) == 0;
    if (lane < int(kCodes)) {
        const uint32_t v = cb_byte(H.cbw, lane);
        ok = ok && v < uint32_t(Dt<DT>::kBins);
        for (int d = 0; d < lane; ++d) ok = ok && cb_byte(H.cbw, d) != v;
    }
    return __all_sync(0xffffffffu, ok);
}

// Check a tensor's plan before coding it (warp-wide).  Ordinary encode: the
// plan is this tensor's header (n, E, codebook, total) and its total must fit
// the output.  Codebook reuse: only the codebook is taken from the plan; the
// smallest stream for n must fit (escapes are bounded by the capacity later).
template <int DT>
__device__ __forceinline__ bool plan_ok(const Header &H, uint64_t n, uint64_t cap, bool reuse,
                                        uint32_t *why) {
    const bool cb = codebook_ok<DT>(H);
    if (reuse) {
        if (!cb) {
            *why = SZ_ERR_PLAN_MISMATCH;
            return false;
        }
        if (stream_layout(DT, n, 0).total > cap) {
            *why = SZ_ERR_BUFFER_TOO_SMALL;
            return false;
        }
        return true;
    }
    if (!cb || H.magic != kMagic || H.vtag != header_vtag(DT) || H.n != n || H.E > n ||
        H.total != stream_layout(DT, n, H.E).total) {
        *why = SZ_ERR_PLAN_MISMATCH;
        return false;
    }
    if (H.total > cap) {
        *why = SZ_ERR_BUFFER_TOO_SMALL;
        return false;
    }
    return true;
}

// Word `lane` (< 16) of the 64-byte stream header for n elements, E escapes
// and codebook words cbw.
template <int DT>
__device__ __forceinline__ uint32_t header_word(int lane, uint64_t n, uint64_t E, uint64_t total,
                                                const uint32_t (&cbw)[4]) {
    uint32_t w = 0;
    w = lane == 0 ? kMagic : w;
    w = lane == 1 ? header_vtag(DT) : w;
    w = lane == 2 ? uint32_t(n) : w;
    w = lane == 3 ? uint32_t(n >> 32) : w;
    w = lane == 4 ? uint32_t(E) : w;
    w = lane == 5 ? uint32_t(E >> 32) : w;
    w = (lane >= 6 && lane < 10) ? pick4(cbw[0], cbw[1], cbw[2], cbw[3], uint32_t(lane - 6)) : w;
    w = lane == 10 ? uint32_t(total) : w;
    w = lane == 11 ? uint32_t(total >> 32) : w;
    return w;
}

__device__ __forceinline__ void zero_bytes(uint8_t *out, uint64_t a, uint64_t b) {
    for (uint64_t x = a + (threadIdx.x & 31); x < b; x += 32) out[x] = 0;
}

// Header (lane l < 16 holds word l), offsets[nb] and the zero gaps between
// sections (once per stream, one warp).
__device__ void write_stream_frame(uint8_t *out, const Layout &L, uint32_t hdr_word, uint64_t E) {
    const int lane = threadIdx.x & 31;
    if (lane < 16) reinterpret_cast<uint32_t *>(out)[lane] = hdr_word;
    if (lane == 0) *reinterpret_cast<uint32_t *>(out + 64 + 4 * L.nb) = uint32_t(E);
    zero_bytes(out, L.tab_end, L.plane[0]);
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        if (s < L.nplanes) {
            const uint64_t end = L.plane[s] + L.plane_len[s];
            const uint64_t next = (s + 1 < L.nplanes) ? L.plane[s + 1] : L.esc;
            zero_bytes(out, end, next);
        }
    }
}

// Up to `valid` elements of one lane's 16-byte step at src (byte by byte
// past the end of the tensor).
template <int DT>
__device__ __forceinline__ uint4 load_step(const uint8_t *src, int valid) {
    if (valid >= Geo<DT>::LE) return __ldcs(reinterpret_cast<const uint4 *>(src));
    uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < Geo<DT>::LE; ++j) {
        if (j < valid) {
            if constexpr (DT == SZ_BF16) {
                const uint32_t b = reinterpret_cast<const uint16_t *>(src)[j];
                w[j >> 1] |= b << (16 * (j & 1));
            } else {
                w[j >> 2] |= uint32_t(src[j]) << (8 * (j & 3));
            }
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void store_bytes(uint8_t *p, uint32_t lo, uint32_t hi, int nbytes) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < nbytes) p[j] = uint8_t(((j < 4) ? lo : hi) >> (8 * (j & 3)));
}

// Per-lane output pointers of one block; each step advances them by a fixed stride.
struct EPtr {
    uint8_t *a, *b, *code;  // BF16: sm plane, -, codes ; E5M2: sign, mantissa, codes
};

template <int DT> struct EStride;
template <> struct EStride<SZ_BF16> {
    static constexpr int a = 256, code = 128;
};
template <> struct EStride<SZ_FP8_E5M2> {
    static constexpr int a = 64, b = 128, code = 256;
};

template <int DT>
__device__ __forceinline__ EPtr block_out(uint8_t *out, const Layout &L, uint64_t e_lane) {
    EPtr q;
    q.code = out + L.code + e_lane / 2;
    if constexpr (DT == SZ_BF16) {
        q.a = out + L.plane[0] + e_lane;
        q.b = nullptr;
    } else {
        q.a = out + L.plane[0] + e_lane / 8;
        q.b = out + L.plane[1] + e_lane / 4;
    }
    return q;
}

// Escape flags of one lane's step: bit 4j for element j (32 bits hold BF16's 8
// elements, 64 bits E5M2's 16).
template <int DT>
using EMask = typename std::conditional<DT == SZ_BF16, uint32_t, uint64_t>::type;

// Shared address of the warp's code table: 256 one-byte entries starting on a
// 256-byte boundary, so that one prmt forms an entry's address from the table
// address (bytes 1-3) and an index byte of the data (byte 0).  BF16 entries
// are indexed by the exponent, E5M2 entries by the whole element byte.
__device__ __forceinline__ uint32_t lut_addr(const WarpShared &W) {
    return (smem_u32(W.lut_raw) + 255u) & ~255u;
}

__device__ __forceinline__ uint32_t popc_mask(uint32_t m) { return __popc(m); }
__device__ __forceinline__ uint32_t popc_mask(uint64_t m) { return __popcll(m); }
__device__ __forceinline__ uint32_t first_bit(uint32_t m) { return __ffs(m) - 1; }
__device__ __forceinline__ uint32_t first_bit(uint64_t m) { return __ffsll(m) - 1; }

// Code one lane's step (LE elements in v); when STORE, write its planes and
// codes.  Returns escape flags: bit 4j for element j.
template <int DT, bool STORE>
__device__ __forceinline__ EMask<DT> code_step(uint32_t lut, uint4 v, int valid, const EPtr &q,
                                              int it) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    if constexpr (DT == SZ_BF16) {
        uint32_t cw = 0, x[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t ws = w[k] << 1;  // exponents in bytes 1 and 3
            const uint32_t c0 = lds_u8(prmt(ws, lut, 0x7651u));
            const uint32_t c1 = lds_u8(prmt(ws, lut, 0x7653u));
            cw += (c0 << (8 * k)) + (c1 << (8 * k + 4));
            // bytes 0 and 2: sign<<7 | mantissa of the two elements (bytes 1, 3 unused)
            x[k] = ((w[k] >> 8) & 0x00800080u) | (w[k] & 0xFF7FFF7Fu);
        }
        if (valid < 8) cw &= (1u << (4 * valid)) - 1u;  // codes past n are 0
        if (STORE) {
            const uint32_t sm_lo = __byte_perm(x[0], x[1], 0x6420);
            const uint32_t sm_hi = __byte_perm(x[2], x[3], 0x6420);
            uint8_t *sm_dst = q.a + it * EStride<DT>::a;
            uint8_t *cd_dst = q.code + it * EStride<DT>::code;
            if (valid == 8) {
                *reinterpret_cast<uint2 *>(sm_dst) = make_uint2(sm_lo, sm_hi);
                *reinterpret_cast<uint32_t *>(cd_dst) = cw;
            } else if (valid > 0) {
                store_bytes(sm_dst, sm_lo, sm_hi, valid);
                store_bytes(cd_dst, cw, 0, (valid + 1) / 2);
            }
        }
        return escape_nibbles(cw);
    } else {
        uint32_t cw[2] = {0, 0}, sign = 0, mant = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t c = lds_u8(prmt(w[k], lut, 0x7650u + uint32_t(b)));
                cw[k >> 1] += c << (4 * (4 * (k & 1) + b));
            }
        }
        if (STORE) {
            // Gathers by multiplication, in which no two partial products share
            // a bit.  The sign bits of two words, the first word's shifted down
            // by 4, land in order in the top byte of one product; the four 2-bit
            // mantissas of a word land in order in the top byte of its product.
            // Byte permutes then set the top bytes side by side.
            const uint32_t s01 = (((w[0] & 0x80808080u) >> 4) | (w[1] & 0x80808080u)) * 0x00204081u;
            const uint32_t s23 = (((w[2] & 0x80808080u) >> 4) | (w[3] & 0x80808080u)) * 0x00204081u;
            sign = __byte_perm(s01, s23, 0x0073u);
            uint32_t mt[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) mt[k] = (w[k] & 0x03030303u) * 0x01041040u;
            mant = __byte_perm(__byte_perm(mt[0], mt[1], 0x0073u), __byte_perm(mt[2], mt[3], 0x0073u), 0x5410u);
        }
        if (valid < 16) {
            if (valid < 8) {
                cw[0] &= (1u << (4 * valid)) - 1u;
                cw[1] = 0;
            } else {
                cw[1] &= (valid == 8) ? 0u : ((1u << (4 * (valid - 8))) - 1u);
            }
        }
        if (STORE) {
            uint8_t *sg_dst = q.a + it * EStride<DT>::a;
            uint8_t *mt_dst = q.b + it * EStride<DT>::b;
            uint8_t *cd_dst = q.code + it * EStride<DT>::code;
            if (valid == 16) {
                *reinterpret_cast<uint16_t *>(sg_dst) = uint16_t(sign);
                *reinterpret_cast<uint32_t *>(mt_dst) = mant;
                *reinterpret_cast<uint2 *>(cd_dst) = make_uint2(cw[0], cw[1]);
            } else if (valid > 0) {
                store_bytes(sg_dst, sign, 0, (valid + 7) / 8);
                store_bytes(mt_dst, mant, 0, (valid + 3) / 4);
                store_bytes(cd_dst, cw[0], cw[1], (valid + 1) / 2);
            }
        }
        return uint64_t(escape_nibbles(cw[0])) | (uint64_t(escape_nibbles(cw[1])) << 32);
    }
}

// Exponent of element j (runtime) of a lane's step.
template <int DT>
__device__ __forceinline__ uint32_t exponent_at(uint4 v, uint32_t j) {
    if constexpr (DT == SZ_BF16) {
        const uint32_t wj = pick4(v.x, v.y, v.z, v.w, j >> 1);
        return (wj >> (16 * (j & 1) + 7)) & 0xFFu;
    } else {
        const uint32_t wj = pick4(v.x, v.y, v.z, v.w, j >> 2);
        return (wj >> (8 * (j & 3) + 2)) & 0x1Fu;
    }
}

// A rank no escape has (ranks within a block are below 4096): a put given it
// stores nothing.
constexpr uint32_t kNoRank = 0x80000000u;

// Escapes of a step in which some lane has two or more (rare on KV data):
// a warp prefix of the per-lane counts c, then each lane hands its escapes
// over in element order.  (Inline: as a call it made KV encode 23% slower,
// measured.)
template <int DT, typename Put>
__device__ __forceinline__ void rank_general(EMask<DT> m, uint4 v, uint32_t c, uint32_t &running, Put put) {
    uint32_t tot;
    const uint32_t prefix = warp_exclusive_prefix(c, &tot);
    if (tot) {
        uint32_t r = running + prefix;
        while (m) {
            const uint32_t j = first_bit(m) >> 2;  // element, in element order
            m &= m - 1;
            put(r++, exponent_at<DT>(v, j));
        }
        running += tot;
    }
}

// Rank one step's escapes within the block and hand each to put(rank,
// exponent).  With `wanted` false the escapes of a step with several per lane
// are only counted: the caller has no room left for them (a chunk whose
// escapes overflow its stage is coded again when it is finished, and its
// escapes are written then).
template <int DT, typename Put>
__device__ __forceinline__ void rank_step(EMask<DT> m, uint4 v, uint32_t &running, Put put, bool wanted = true) {
    if constexpr (DT == SZ_FP8_E5M2) {
        // one flag bit per escaped element: 4j for element j < 8, 4(j - 8) + 1 above
        const uint32_t fl = uint32_t(m) | (uint32_t(m >> 32) << 1);
        const uint32_t any = __ballot_sync(0xffffffffu, fl != 0u);
        const uint32_t multi = __ballot_sync(0xffffffffu, (fl & (fl - 1u)) != 0u);
        if (multi == 0u) {
            // the escaped element's byte: byte (p >> 2) of words x, y (p even) or z, w (p odd)
            const uint32_t p = __ffs(fl) - 1u;
            const uint32_t odd = p & 1u;
            const uint32_t e = (__byte_perm(odd ? v.z : v.x, odd ? v.w : v.y, p >> 2) >> 2) & 0x1Fu;
            put(fl ? running + __popc(any & lanemask_lt()) : kNoRank, e);
            running += __popc(any);
            return;
        }
    }
    const uint32_t c = popc_mask(m);
    const uint32_t any = __ballot_sync(0xffffffffu, c != 0);
    if (any == 0) return;
    if (__ballot_sync(0xffffffffu, c > 1) == 0) {
        // at most one escape per lane: its rank counts the lanes before it that have one
        const uint32_t lane = threadIdx.x & 31;
        // without a divergent branch (1% faster, measured): a lane without an
        // escape passes kNoRank, which every put rejects
        put(c ? running + __popc(any & ((1u << lane) - 1u)) : kNoRank, exponent_at<DT>(v, first_bit(m) >> 2));
        running += __popc(any);
        return;
    }
    if (!wanted) {
        running += __reduce_add_sync(0xffffffffu, c);
        return;
    }
    rank_general<DT>(m, v, c, running, put);
}

// One warp codes block blk of a tensor of n elements: planes and codes go to
// out; escapes (exponents in element order) go to put(rank, exponent).
// Returns the block's escape count.
template <int DT, bool STORE, bool PAGED, typename Put>
__device__ __forceinline__ uint32_t code_block(uint32_t lut, const uint8_t *in, const PageRef &pr, uint64_t n,
                                               uint64_t blk, const Layout &L, uint8_t *out, Put put) {
    using G = Geo<DT>;
    const int lane = threadIdx.x & 31;
    const uint64_t e_lane = blk * kBlock + uint64_t(lane) * G::LE;
    const uint8_t *src = in + e_lane * Dt<DT>::kElemBytes;
    const EPtr q = block_out<DT>(out, L, e_lane);
    uint32_t running = 0;
    if (PAGED && pr.pages) {
        // paged input: each step's 16 bytes from its own page (a step never straddles one)
        for (int it = 0; it < G::IT; ++it) {
            const int64_t left = int64_t(n) - int64_t(e_lane) - int64_t(it) * 32 * G::LE;
            const int valid = left <= 0 ? 0 : (left >= G::LE ? G::LE : int(left));
            uint4 v = make_uint4(0, 0, 0, 0);
            if (valid > 0) {
                const uint64_t off = elem_offset<Dt<DT>::kElemBytes>(pr, e_lane + uint64_t(it) * 32 * G::LE);
                if (off != kBadOffset) v = load_step<DT>(in + off, valid);
            }
            const EMask<DT> m = code_step<DT, STORE>(lut, v, valid, q, it);
            rank_step<DT>(m, v, running, put);
        }
    } else if ((blk + 1) * kBlock <= n) {
        uint4 ring[G::kAhead + 1];
#pragma unroll
        for (int i = 0; i < G::kAhead; ++i) ring[i] = __ldcs(reinterpret_cast<const uint4 *>(src + i * 512));
#pragma unroll
        for (int it = 0; it < G::IT; ++it) {
            if (it + G::kAhead < G::IT)
                ring[(it + G::kAhead) % (G::kAhead + 1)] =
                    __ldcs(reinterpret_cast<const uint4 *>(src + (it + G::kAhead) * 512));
            const uint4 v = ring[it % (G::kAhead + 1)];
            const EMask<DT> m = code_step<DT, STORE>(lut, v, G::LE, q, it);
            rank_step<DT>(m, v, running, put);
        }
    } else {
        for (int it = 0; it < G::IT; ++it) {
            const int64_t left = int64_t(n) - int64_t(e_lane) - int64_t(it) * 32 * G::LE;
            const int valid = left <= 0 ? 0 : (left >= G::LE ? G::LE : int(left));
            const uint4 v = valid > 0 ? load_step<DT>(src + it * 512, valid) : make_uint4(0, 0, 0, 0);
            const EMask<DT> m = code_step<DT, STORE>(lut, v, valid, q, it);
            rank_step<DT>(m, v, running, put);
        }
    }
    return running;
}

// One lane's share of one step of a raw block (v: its up to LE elements, only
// `valid` of them in the tensor): the low four bits of each exponent to the
// code plane at cd (the bytes code_step wrote for this lane), the bits above
// them to the escape section at h (BF16: a high nibble per element, E5M2: bit
// 4 per element), bytes at or past bound not written.  A full step writes its
// code bytes with one aligned store and its high bits with one store when h
// is aligned for it.
template <int DT>
__device__ __forceinline__ void raw_step(uint4 v, int valid, uint8_t *cd, uint8_t *out, uint64_t h, uint64_t bound) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t lo[2] = {0, 0}, hi = 0;
    if constexpr (DT == SZ_BF16) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            // exponents of elements 2k, 2k+1 in bytes 0 and 2
            const uint32_t x = (w[k] >> 7) & 0x00FF00FFu;
            lo[0] |= ((x & 0xFu) | ((x >> 12) & 0xF0u)) << (8 * k);
            hi |= (((x >> 4) & 0xFu) | ((x >> 16) & 0xF0u)) << (8 * k);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t x = (w[j >> 2] >> (8 * (j & 3) + 2)) & 0x1Fu;
            lo[j >> 3] |= (x & 0xFu) << (4 * (j & 7));
            hi |= (x >> 4) << j;
        }
    }
    constexpr int kHiBytes = (DT == SZ_BF16) ? 4 : 2;
    if (valid == Geo<DT>::LE) {
        if constexpr (DT == SZ_BF16) *reinterpret_cast<uint32_t *>(cd) = lo[0];
        else *reinterpret_cast<uint2 *>(cd) = make_uint2(lo[0], lo[1]);
        if (h + kHiBytes <= bound && (h & (kHiBytes - 1)) == 0) {
            if constexpr (DT == SZ_BF16) *reinterpret_cast<uint32_t *>(out + h) = hi;
            else *reinterpret_cast<uint16_t *>(out + h) = uint16_t(hi);
            return;
        }
    } else {
        store_bytes(cd, lo[0], lo[1], (valid + 1) / 2);
    }
    const int hbytes = (DT == SZ_BF16) ? (valid + 1) / 2 : (valid + 7) / 8;
    for (int b = 0; b < hbytes; ++b)
        if (h + b < bound) out[h + b] = uint8_t(hi >> (8 * b));
}

// One warp stores block blk raw (raw blocks allowed and its escapes would
// fill at least raw_block_bytes): the low four bits of each exponent
// overwrite the block's code nibbles, the remaining bits go to the escape
// section at byte d (BF16: high nibbles, element j of the block in nibble j%2
// of byte j/2; E5M2: bit 4 at bit j%8 of byte j/8), bytes at or past bound
// not written.  Planes are as coded.  The block's input is read again, with
// G::kAhead loads per lane in flight for a full contiguous block.  Out of line:
// inlined into the kernel it slowed the coded path by 1-2% (measured).
template <int DT, bool PAGED>
__device__ __noinline__ void raw_block(const uint8_t *in, const PageRef &pr, uint64_t n, uint64_t blk, const Layout &L,
                          uint8_t *out, uint64_t d, uint64_t bound) {
    using G = Geo<DT>;
    constexpr int EB = Dt<DT>::kElemBytes;
    const int lane = threadIdx.x & 31;
    const uint64_t e_lane = blk * kBlock + uint64_t(lane) * G::LE;
    const bool paged = PAGED && pr.pages != nullptr;
    uint8_t *code = out + L.code + e_lane / 2;
    // this lane's high bits of step it start at h0 + it * kHiStride
    const uint64_t h0 = d + ((DT == SZ_BF16) ? uint64_t(lane) * G::LE / 2 : uint64_t(lane) * G::LE / 8);
    constexpr uint32_t kHiStride = (DT == SZ_BF16) ? 32 * G::LE / 2 : 32 * G::LE / 8;
    if (!paged && (blk + 1) * kBlock <= n) {
        const uint8_t *src = in + e_lane * EB;
        uint4 ring[G::kAhead + 1];
#pragma unroll
        for (int i = 0; i < G::kAhead; ++i) ring[i] = __ldcs(reinterpret_cast<const uint4 *>(src + i * 512));
#pragma unroll
        for (int it = 0; it < G::IT; ++it) {
            if (it + G::kAhead < G::IT)
                ring[(it + G::kAhead) % (G::kAhead + 1)] =
                    __ldcs(reinterpret_cast<const uint4 *>(src + (it + G::kAhead) * 512));
            raw_step<DT>(ring[it % (G::kAhead + 1)], G::LE, code + it * EStride<DT>::code, out,
                         h0 + uint64_t(it) * kHiStride, bound);
        }
        return;
    }
#pragma unroll 1
    for (int it = 0; it < G::IT; ++it) {
        const int64_t left = int64_t(n) - int64_t(e_lane) - int64_t(it) * 32 * G::LE;
        const int valid = left <= 0 ? 0 : (left >= G::LE ? G::LE : int(left));
        if (valid <= 0) continue;
        const uint64_t e = e_lane + uint64_t(it) * 32 * G::LE;
        const uint64_t off = paged ? elem_offset<EB>(pr, e) : e * EB;
        const uint4 v = off != kBadOffset ? load_step<DT>(in + off, valid) : make_uint4(0, 0, 0, 0);
        raw_step<DT>(v, valid, code + it * EStride<DT>::code, out, h0 + uint64_t(it) * kHiStride, bound);
    }
}

// The warp's input ring: units (Units below) of the chunk being coded,
// stage = unit % kRing; units of a partial (last) block are not copied and
// are read from global memory instead.
struct RingState {
    uint32_t issued;  // bit s: stage s holds a copy not yet waited for
    uint32_t parity;  // bit s: parity of stage s's next completion
    uint32_t vi, vc;  // units issued / consumed
};

// Units per 4096-element block of the input ring: 2 KB units, i.e. quarter
// blocks for BF16 and half blocks for E5M2 -- but quarter blocks for paged E5M2
// input, whose pages are only known to hold multiples of 1024 elements.
template <int DT, bool PAGED>
struct Units {
    static constexpr int kPerBlock = (DT == SZ_BF16 || PAGED) ? 4 : 2;
    static constexpr uint32_t kElems = kBlock / kPerBlock;
    static constexpr uint32_t kBytes = kElems * Dt<DT>::kElemBytes;
    static_assert(kBytes <= kUnitBytes, "a unit must fit a ring stage");
};

template <int DT, bool PAGED>
__device__ __forceinline__ void ring_issue(WarpShared &W, RingState &R, const uint8_t *in, uint64_t n,
                                           uint64_t b0, uint32_t x, bool paged, uint64_t paged_off, uint32_t *ctl) {
    using U = Units<DT, PAGED>;
    const int st = int(R.vi % kRing);
    const uint64_t blk = b0 + x / U::kPerBlock;
    if ((blk + 1) * kBlock <= n) {
        // byte offset of the unit from the input base (paged: looked up by the caller)
        const uint64_t off = paged ? paged_off
                                   : (blk * kBlock + (x % U::kPerBlock) * U::kElems) * Dt<DT>::kElemBytes;
        if (off != kBadOffset) {
            if ((threadIdx.x & 31) == 0) {
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&W.bar[st], U::kBytes);
                bulk_g2s(W.ring[st], in + off, U::kBytes, &W.bar[st]);
            }
            R.issued |= 1u << st;
        } else if ((threadIdx.x & 31) == 0) {
            set_error(ctl, SZ_ERR_INVALID_ARG, uint32_t(blk));  // page id outside the pool: not read
        }
    }
    ++R.vi;
}

// Wait for the unit about to be consumed; false if its copy never landed.
__device__ __forceinline__ bool ring_take(WarpShared &W, RingState &R, int *stage) {
    const int st = int(R.vc % kRing);
    *stage = st;
    ++R.vc;
    if (!(R.issued & (1u << st))) return true;
    const bool ok = mbar_wait(&W.bar[st], (R.parity >> st) & 1u, kWaitLimitNs);
    R.parity ^= 1u << st;
    R.issued &= ~(1u << st);
    return ok;
}

// Load tensor t's plan into the warp's shared area and build its exponent ->
// code table.
template <int DT, int MAXB>
__device__ __forceinline__ void warp_load_plan(const EncodeParams<MAXB> &p, int t, WarpShared &W) {
    const int lane = threadIdx.x & 31;
    if (lane < 16)
        W.hdr[lane] = lane < 12 ? reinterpret_cast<const uint32_t *>(p.plans + 64 * size_t(t))[lane] : 0u;
    __syncwarp();
    const Header H = load_header(reinterpret_cast<const uint8_t *>(W.hdr));
    const uint32_t lut = lut_addr(W);
    // every entry escapes (8 bytes per lane) ...
    sts_u64(lut + uint32_t(lane) * 8u, 0x0F0F0F0F0F0F0F0Full);
    __syncwarp();
    // ... except those of the codebook's values: lane c writes code c.  A value
    // outside the exponent range writes nothing (plan_ok then rejects the plan).
    if (lane < int(kCodes)) {
        const uint32_t e = cb_byte(H.cbw, lane);
        if (e < uint32_t(Dt<DT>::kBins)) {
            if constexpr (DT == SZ_BF16) {
                sts_u8(lut + e, uint32_t(lane));  // BF16 entries are indexed by the exponent
            } else {
#pragma unroll
                for (uint32_t sm = 0; sm < 8; ++sm)  // E5M2 entries by the element byte: sign, mantissa
                    sts_u8(lut + ((sm >> 2) << 7 | e << 2 | (sm & 3u)), uint32_t(lane));
            }
        }
    }
    __syncwarp();
}

// Geometry of a chunk (job) of the launch.
struct ChunkGeo {
    int t;
    uint32_t chunk;
    uint64_t n, nb, b0;
    int nbk;
};

// LG: blocks per chunk as a log2 fixed at compile time (the full-size chunk of
// large batches), or -1 to read it from the launch (small batches).
template <int MAXB, int LG>
__device__ __forceinline__ ChunkGeo chunk_geo(const EncodeParams<MAXB> &p, uint32_t job) {
    const int lg = LG >= 0 ? LG : p.chunk_log2;
    ChunkGeo g;
    g.t = find_tensor<uint32_t, MAXB>(p.chunk_begin, p.T, job);
    g.chunk = job - p.chunk_begin[g.t];
    g.n = p.n[g.t];
    g.nb = cdiv(g.n, kBlock);
    g.b0 = uint64_t(g.chunk) << lg;
    g.nbk = int(min(uint64_t(1) << lg, g.nb - g.b0));
    return g;
}

// One warp codes a chunk: planes and codes go out, escapes are staged in
// esc[slot] (element order) with per-block offsets in blk_off[slot].  Returns
// the chunk's escape-section bytes, or
// 0xFFFFFFFF if the plan does not fit the data (reported; nothing to finish).
// With raw blocks allowed, bit k of *raw is set for each block k of the chunk
// that is to be stored raw; it counts raw_block_bytes.
template <int DT, int MAXB, bool PAGED>
__device__ uint32_t code_chunk(const EncodeParams<MAXB> &p, uint32_t job, const ChunkGeo &g, int slot,
                               WarpShared &W, RingState &R, int &plan_tensor, bool *lost, uint32_t *raw) {
    const int lane = threadIdx.x & 31;
    const uint8_t *in = p.in[g.t];
    uint8_t *out = p.out[g.t];
    const uint64_t n = g.n, b0 = g.b0;
    const int nbk = g.nbk;
    if (g.t != plan_tensor) {
        warp_load_plan<DT, MAXB>(p, g.t, W);
        plan_tensor = g.t;
    }
    const Header H = load_header(reinterpret_cast<const uint8_t *>(W.hdr));
    uint32_t why = 0;
    if (!plan_ok<DT>(H, n, p.cap[g.t], p.reuse != 0, &why)) {
        if (lane == 0 && g.chunk == 0) set_error(p.ctl, why, uint32_t(g.t));
        return 0xFFFFFFFFu;  // every chunk of this tensor takes this branch: no look-back waits on it
    }
    const Layout L = stream_layout(DT, n, p.reuse ? 0 : H.E);  // section starts do not depend on E
    const bool raw_ok = (header_flags(H) & kFlagRawBlocks) != 0;
    *raw = 0;

    using G = Geo<DT>;
    using UN = Units<DT, PAGED>;
    constexpr int QIT = G::IT / UN::kPerBlock;  // steps per unit
    const uint32_t lut = lut_addr(W), stage = smem_u32(W.esc[slot]);
    const uint32_t nunits = uint32_t(UN::kPerBlock) * uint32_t(nbk);
    // paged input: lane x looks up where unit x (a quarter block) of the chunk lives
    const PageRef &pr = p.pg[g.t];
    const bool paged = PAGED && pr.pages != nullptr;
    uint64_t unit_off = 0;
    if (paged && uint32_t(lane) < nunits && b0 * kBlock + uint64_t(lane) * UN::kElems < n)
        unit_off = elem_offset<Dt<DT>::kElemBytes>(pr, b0 * kBlock + uint64_t(lane) * UN::kElems);
    auto issue = [&](uint32_t x) {
        const uint64_t off = paged ? __shfl_sync(0xffffffffu, unit_off, int(x)) : 0ull;
        ring_issue<DT, PAGED>(W, R, in, n, b0, x, paged, off, p.ctl);
    };
    uint32_t next_x = 0;
    for (; next_x < uint32_t(kRing - 1) && next_x < nunits; ++next_x) issue(next_x);
    uint32_t running = 0;
#pragma unroll 1
    for (int k = 0; k < nbk; ++k) {
        const uint64_t blk = b0 + k;
        if (lane == 0) W.blk_off[slot][k] = running;
        const bool full = (blk + 1) * kBlock <= n;
        const uint64_t e_lane = blk * kBlock + uint64_t(lane) * G::LE;
        const EPtr q = block_out<DT>(out, L, e_lane);
        const uint32_t base = running;
        auto put = [&](uint32_t r, uint32_t e) {  // base + kNoRank does not wrap: base < kWarpStage
            if (base + r < kWarpStage) sts_u8(stage + base + r, e);
        };
        uint32_t blk_run = 0;
#pragma unroll 1
        for (int qq = 0; qq < UN::kPerBlock; ++qq) {
            if (next_x < nunits) issue(next_x++);
            int st;
            *lost = !ring_take(W, R, &st) || *lost;
            if (full) {
                const uint32_t src = smem_u32(W.ring[st]) + uint32_t(lane) * 16;
                // escapes that can no longer be staged are only counted (checked per unit)
                const bool staged = base + blk_run < kWarpStage;
                // E5M2 runs this loop rolled: 3% faster than unrolled (measured)
                if constexpr (DT == SZ_BF16) {
#pragma unroll
                    for (int it = 0; it < QIT; ++it) {
                        const uint4 v = lds_u128(src + it * 512);
                        const EMask<DT> m = code_step<DT, true>(lut, v, G::LE, q, qq * QIT + it);
                        rank_step<DT>(m, v, blk_run, put, staged);
                    }
                } else {
#pragma unroll 1
                    for (int it = 0; it < QIT; ++it) {
                        const uint4 v = lds_u128(src + it * 512);
                        const EMask<DT> m = code_step<DT, true>(lut, v, G::LE, q, qq * QIT + it);
                        rank_step<DT>(m, v, blk_run, put, staged);
                    }
                }
            } else {
                for (int it = qq * QIT; it < (qq + 1) * QIT; ++it) {
                    const int64_t left = int64_t(n) - int64_t(e_lane) - int64_t(it) * 32 * G::LE;
                    const int valid = left <= 0 ? 0 : (left >= G::LE ? G::LE : int(left));
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (valid > 0) {
                        const uint64_t e = e_lane + uint64_t(it) * 32 * G::LE;
                        const uint64_t off = paged ? elem_offset<Dt<DT>::kElemBytes>(pr, e) : e * Dt<DT>::kElemBytes;
                        if (off != kBadOffset) v = load_step<DT>(in + off, valid);
                    }
                    const EMask<DT> m = code_step<DT, true>(lut, v, valid, q, it);
                    rank_step<DT>(m, v, blk_run, put);
                }
            }
            __syncwarp();  // the stage just read may be refilled from here on
        }
        if (raw_ok) {
            const uint32_t m = full ? kBlock : uint32_t(n - blk * kBlock);
            if (blk_run >= raw_block_bytes<DT>(m)) {
                blk_run = raw_block_bytes<DT>(m);
                *raw |= 1u << k;
            }
        }
        running += blk_run;
    }
    __syncwarp();
    return running;
}

// Once the chunk's offset excl is known: its offsets-table entries, its
// escapes (from the stage, or re-coded from the input when they overflowed
// it or the chunk has raw blocks -- the warp's code table is then still the
// chunk's), and the stream frame if it is the tensor's last chunk.
// hdr_here: the warp's shared copy of the plan (W.hdr) is this chunk's tensor's,
// so it is read instead of the plan in global memory.
template <int DT, int MAXB, bool PAGED>
__device__ void finish_chunk(const EncodeParams<MAXB> &p, uint32_t job, const ChunkGeo &g, int slot,
                             uint32_t total, uint32_t raw, const Lookback &lb, WarpShared &W, bool hdr_here) {
    const int lane = threadIdx.x & 31;
    const Header H = load_header(hdr_here ? reinterpret_cast<const uint8_t *>(W.hdr) : p.plans + 64 * size_t(g.t));
    const bool reuse = p.reuse != 0;
    // the plan's E counts every escape; raw blocks store fewer bytes, so with
    // raw blocks allowed E is known only at the end, as with a reused codebook
    const bool raw_ok = (header_flags(H) & kFlagRawBlocks) != 0;
    const Layout L = stream_layout(DT, g.n, reuse ? 0 : H.E);
    uint8_t *out = p.out[g.t];
    const uint32_t excl = lb.excl;
    const bool last = g.b0 + g.nbk == g.nb;
    if (lane == 0) {
        if (lb.flags & kLbTimedOut) set_error(p.ctl, SZ_ERR_TIMEOUT, job);
        if (!reuse) {
            if (uint64_t(excl) + total > H.E) set_error(p.ctl, SZ_ERR_PLAN_MISMATCH, job);
            if (!raw_ok && last && uint64_t(excl) + total != H.E) set_error(p.ctl, SZ_ERR_PLAN_MISMATCH, job);
        }
    }
    if (lane < g.nbk) *reinterpret_cast<uint32_t *>(out + 64 + 4 * (g.b0 + lane)) = excl + W.blk_off[slot][lane];
    // escapes past the stream's end (ordinary encode) or the buffer's (reuse) are not written
    const uint64_t bound = reuse ? p.cap[g.t] : L.total;
    const uint64_t dst = L.esc + excl;
    if (total <= kWarpStage && raw == 0) {
        for (uint32_t x = lane; x < total; x += 32)
            if (dst + x < bound) out[dst + x] = W.esc[slot][x];
    } else {
        const uint32_t lut = lut_addr(W);
#pragma unroll 1
        for (int k = 0; k < g.nbk; ++k) {
            const uint64_t d = dst + W.blk_off[slot][k];
            if ((raw >> k) & 1u) {
                raw_block<DT, PAGED>(p.in[g.t], p.pg[g.t], g.n, g.b0 + k, L, out, d, bound);
            } else {
                code_block<DT, false, PAGED>(lut, p.in[g.t], p.pg[g.t], g.n, g.b0 + k, L, out,
                                             [&](uint32_t r, uint32_t e) {
                                                 if (r < kNoRank && d + r < bound) out[d + r] = uint8_t(e);
                                             });
            }
        }
    }
    if (last) {
        // the tensor's escape-section length is now known: excl + total
        const uint64_t E = (reuse || raw_ok) ? uint64_t(excl) + total : H.E;
        const uint64_t stream_total = stream_layout(DT, g.n, E).total;
        if (reuse && stream_total > p.cap[g.t] && lane == 0) set_error(p.ctl, SZ_ERR_BUFFER_TOO_SMALL, job);
        write_stream_frame(out, L, header_word<DT>(lane, g.n, E, stream_total, H.cbw), E);
        if (p.totals && lane == 0) p.totals[g.t] = stream_total;
    }
    __syncwarp();
}

// Stream of an empty tensor: header, offsets[0] = 0, zero padding (one warp).
template <int DT, int MAXB>
__device__ void encode_empty(const EncodeParams<MAXB> &p, int t, WarpShared &W, int &plan_tensor) {
    const int lane = threadIdx.x & 31;
    warp_load_plan<DT, MAXB>(p, t, W);
    plan_tensor = t;
    const Header H = load_header(reinterpret_cast<const uint8_t *>(W.hdr));
    uint32_t why = 0;
    if (!plan_ok<DT>(H, 0, p.cap[t], p.reuse != 0, &why)) {
        if (lane == 0) set_error(p.ctl, why, uint32_t(t));
        return;
    }
    const Layout L = stream_layout(DT, 0, 0);
    write_stream_frame(p.out[t], L, header_word<DT>(lane, 0, 0, L.total, H.cbw), 0);
    if (p.totals && lane == 0) p.totals[t] = L.total;
}

// A chunk whose offset is still being looked up.
struct Pending {
    bool valid;
    uint32_t job, total;
    int slot;
    Lookback lb;
};

// Tensor t's look-back words.
template <int MAXB>
__device__ __forceinline__ LbWords lb_words(const EncodeParams<MAXB> &p, int t) {
    LbWords c;
    c.st = p.status + p.chunk_begin[t];
    c.gs = p.group + (p.chunk_begin[t] >> kLbGroupLog2) + uint32_t(t);
    c.nchunks = p.chunk_begin[t + 1] - p.chunk_begin[t];
    return c;
}

template <int DT, int MAXB, bool PAGED, int LG>
__global__ void __launch_bounds__(enc_threads<DT>(), enc_ctas_per_sm<DT>()) encode_kernel(const __grid_constant__ EncodeParams<MAXB> p) {
    extern __shared__ __align__(128) uint8_t s_raw[];
    WarpShared *s_warp = reinterpret_cast<WarpShared *>(s_raw);
    __shared__ uint32_t s_epoch;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WarpShared &W = s_warp[warp];
    if (lane == 0) {
        for (int i = 0; i < kRing; ++i) mbar_init(&W.bar[i], 1);
        fence_mbar_init();
    }
    pdl_wait();  // nothing above touches global memory (programmatic launch)
    pdl_launch_dependents();
    if (tid == 0) s_epoch = ld_relaxed_u32(&p.ctl[kCtlEpoch]);
    __syncthreads();
    const uint32_t epoch = s_epoch;
    const unsigned long long tag = (unsigned long long)(epoch & 0x3FFFFFFFu) << 34;
    RingState R = {0u, 0u, 0u, 0u};
    int plan_tensor = -1;
    Pending pend;
    pend.valid = false;
    // finish the pending chunk (its look-back waits, bounded, until done)
    auto settle = [&]() {
        if (!pend.valid) return;
        const ChunkGeo pg = chunk_geo<MAXB, LG>(p, pend.job);
        lookback_advance(pend.lb, lb_words(p, pg.t), pg.chunk, pend.total, tag, true);
        finish_chunk<DT, MAXB, PAGED>(p, pend.job, pg, pend.slot, pend.total, 0u, pend.lb, W, pg.t == plan_tensor);
        pend.valid = false;
    };
    // every warp claims chunks in launch order until none is left
    while (true) {
        uint32_t job = 0;
        if (lane == 0) job = atomicAdd(&p.ctl[kCtlTileCtr], 1u);
        job = __shfl_sync(0xffffffffu, job, 0);
        if (job >= p.total_jobs) break;
        if (job >= p.total_chunks) {
            encode_empty<DT, MAXB>(p, p.empty[job - p.total_chunks], W, plan_tensor);
            continue;
        }
        const ChunkGeo g = chunk_geo<MAXB, LG>(p, job);
        const int slot = pend.valid ? (pend.slot ^ 1) : 0;
        bool lost = false;
        uint32_t raw = 0;
        const uint32_t total = code_chunk<DT, MAXB, PAGED>(p, job, g, slot, W, R, plan_tensor, &lost, &raw);
        if (lost && lane == 0) set_error(p.ctl, SZ_ERR_TIMEOUT, job);
        if (total == 0xFFFFFFFFu) continue;  // plan rejected for this tensor
        const LbWords st = lb_words(p, g.t);
        Lookback lb;
        lookback_start(lb, st, g.chunk, total, tag);
        settle();  // at most one chunk waits for its offset
        // chunks that re-read their input (escape overflow, raw blocks) finish at once
        if (total > kWarpStage || raw != 0 || lookback_advance(lb, st, g.chunk, total, tag, false)) {
            lookback_advance(lb, st, g.chunk, total, tag, true);
            finish_chunk<DT, MAXB, PAGED>(p, job, g, slot, total, raw, lb, W, g.t == plan_tensor);
        } else {
            pend.valid = true;
            pend.job = job;
            pend.total = total;
            pend.slot = slot;
            pend.lb = lb;
        }
    }
    settle();
    // The last CTA to retire leaves the counters ready for the next launch.
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(&p.ctl[kCtlDone], 1u) == gridDim.x - 1) {
            atomicExch(&p.ctl[kCtlTileCtr], 0u);
            atomicExch(&p.ctl[kCtlDone], 0u);
            atomicExch(&p.ctl[kCtlEpoch], epoch + 1);
        }
    }
}

template <int DT, int MAXB, bool PAGED>
sz_status launch_encode_t(const EncodeArgs &a, cudaStream_t stream) {
    // Full-size chunks (large batches) run an instantiation with the chunk size
    // fixed at compile time; shorter chunks read it from the launch.  Both have
    // the same launch bounds and shared memory.
    constexpr int NT = enc_threads<DT>(), NW = NT / 32;
    auto kern_full = encode_kernel<DT, MAXB, PAGED, kMaxChunkLog2>;
    auto kern_any = encode_kernel<DT, MAXB, PAGED, -1>;
    const size_t smem = sizeof(WarpShared) * NW;
    static std::atomic<int> cache_full[kMaxDevices], cache_any[kMaxDevices];
    const int per_sm = resident_per_sm(reinterpret_cast<const void *>(kern_full), NT, smem, cache_full);
    if (per_sm < 1) return SZ_ERR_CUDA;
    const uint64_t resident = uint64_t(a.num_sms) * per_sm;
    EncodeParams<MAXB> p;
    p.ctl = a.ctl;
    p.status = a.status;
    p.group = a.group;
    p.plans = a.plans;
    p.totals = a.totals;
    p.reuse = a.reuse;
    for (int t = 0; t < a.T; ++t) p.pg[t] = page_ref(a.paged ? a.paged + t : nullptr);
    p.T = a.T;
    p.n_empty = 0;
    uint64_t total_blocks = 0;
    for (int t = 0; t < a.T; ++t) total_blocks += cdiv(a.n[t], kBlock);
    p.chunk_log2 = pick_chunk_log2(total_blocks, resident * NW);
    p.chunk_begin[0] = 0;
    for (int t = 0; t < a.T; ++t) {
        p.in[t] = static_cast<const uint8_t *>(a.in[t]);
        p.out[t] = static_cast<uint8_t *>(a.out[t]);
        p.n[t] = a.n[t];
        p.cap[t] = a.cap[t];
        const uint64_t nb = cdiv(a.n[t], kBlock);
        p.chunk_begin[t + 1] = p.chunk_begin[t] + uint32_t(cdiv(nb, uint64_t(1) << p.chunk_log2));
        if (a.n[t] == 0) p.empty[p.n_empty++] = uint16_t(t);
    }
    p.total_chunks = p.chunk_begin[a.T];
    p.total_jobs = p.total_chunks + uint32_t(p.n_empty);
    if (p.total_jobs == 0) return SZ_OK;
    const uint64_t need = cdiv(p.total_jobs, NW);
    const uint64_t grid = need < resident ? need : resident;
    auto kern = kern_full;
    if (p.chunk_log2 != kMaxChunkLog2) {
        kern = kern_any;
        if (resident_per_sm(reinterpret_cast<const void *>(kern_any), NT, smem, cache_any) < 1) return SZ_ERR_CUDA;
    }
    // An ordinary launch: with a programmatic one, a small launch's CTAs pile
    // onto the SMs that the previous kernel frees first (3 per SM), and one
    // Llama-3-8B layer's encode took 45% longer (measured).
    kern<<<unsigned(grid), NT, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? SZ_OK : SZ_ERR_CUDA;
}

}  // namespace

sz_status launch_encode(const EncodeArgs &a, cudaStream_t stream) {
    // paged inputs get their own instantiation: contiguous ones carry no paging code
    if (a.paged) {
        if (a.dtype == SZ_BF16)
            return a.T <= kSmallBatch ? launch_encode_t<SZ_BF16, kSmallBatch, true>(a, stream)
                                      : launch_encode_t<SZ_BF16, kLargeBatch, true>(a, stream);
        return a.T <= kSmallBatch ? launch_encode_t<SZ_FP8_E5M2, kSmallBatch, true>(a, stream)
                                  : launch_encode_t<SZ_FP8_E5M2, kLargeBatch, true>(a, stream);
    }
    if (a.dtype == SZ_BF16)
        return a.T <= kSmallBatch ? launch_encode_t<SZ_BF16, kSmallBatch, false>(a, stream)
                                  : launch_encode_t<SZ_BF16, kLargeBatch, false>(a, stream);
    return a.T <= kSmallBatch ? launch_encode_t<SZ_FP8_E5M2, kSmallBatch, false>(a, stream)
                              : launch_encode_t<SZ_FP8_E5M2, kLargeBatch, false>(a, stream);
}

}  // namespace sz
