// sz_decode.cu -- decode kernel: code -> exponent, escape gather, reassembly.
//
// SplitZip project page, FAQ "Is SplitZip lossy?": decoded tensors are
// bitwise identical to the originals; FAQ "How can I reduce KV cache transfer
// time ...": decompression runs on the decode GPU.  The stored per-block
// escape offsets make decode a pure gather with no dependency between blocks,
// so one warp decodes one 4096-element block on its own, with no CTA barrier
// on the way (one closes the kernel, before the last CTA resets the claims):
//   - warps claim blocks one at a time from per-tensor counters (claiming the
//     next block while decoding the current one), so they all finish within
//     about one block of each other; a warp stays in one tensor while it has
//     blocks and checks a tensor's header (and builds its code-pair table)
//     when it moves to it; a stream that fails a check sets
//     SZ_ERR_CORRUPT_STREAM and is not written;
//   - the block's code and plane bytes (6 KB BF16, 3.5 KB E5M2) arrive by 1-D
//     bulk copies of 1.5-1.8 KB units into a 4-stage shared-memory ring that
//     runs 2-3 units ahead of the decoding, across into the claimed next block
//     (waits are bounded); the next block's offsets-table entries and first 32
//     escape bytes are prefetched into registers;
//   - per 256-element (BF16) or 512-element (E5M2) step: BF16 code bytes (two
//     4-bit codes) select pre-spread exponent pairs from a 256-entry shared
//     table, E5M2 codes select exponents from a 16-byte table in registers
//     with prmt; escape ranks come from ballots (a fast path when no lane has
//     two: in E5M2 it runs straight through, with one flag bit per escape and
//     no per-lane counts) and the escape bytes from a shuffle -- an E5M2 lane's
//     escape enters through its table's code-15 byte; the elements are reassembled
//     with byte permutes and integer multiply-adds and written with 16-byte
//     stores (512 contiguous bytes per warp instruction);
//   - a raw block (header flag set and an offsets-table count equal to the
//     block's raw size) is rebuilt from its low exponent nibbles and the high
//     bits in its escape section: step by step in the contiguous BF16 kernel,
//     and by a second kernel (raw_pass_kernel) after the others.
#include <type_traits>

#include "sz_common.cuh"
#include "sz_internal.h"

namespace sz {

namespace {

// One CTA per SM of independent warps, so that every SM gets the same number
// of warps however the CTAs are placed (a launch that starts while the previous
// kernel holds some SMs places several small CTAs on the SMs freed first): 24
// warps at 80 registers for BF16, 20 warps at 96 registers for E5M2, which
// does more integer work per byte (measured: 7% faster than 24 warps; 16 warps
// are slower for both).
template <int DT>
constexpr int dec_threads() { return DT == SZ_BF16 ? 768 : 640; }
// The raw-block pass: one ordinary CTA per tensor.
constexpr int kRawThreads = kTileThreads;
constexpr int kRawWarps = kRawThreads / 32;
constexpr int kStages = 4;                            // ring of input-unit stages per warp
constexpr uint64_t kWaitLimitNs = 1000000000ull;      // 1 s

// Input units of the ring: quarter blocks for BF16 (1536 bytes of codes and
// planes) and for paged E5M2 (whose pages are only known to hold multiples of
// 1024 elements), half blocks for contiguous E5M2 (1792 bytes) -- so that a
// unit is some 1.5-2 KB and its per-unit work covers several steps.
template <int DT, bool PAGED = false>
struct DGeo {
    static constexpr int LE = (DT == SZ_BF16) ? 8 : 16;   // elements per lane per step
    static constexpr int IT = int(kBlock) / (32 * LE);     // steps per block
    static constexpr int kUnits = (DT == SZ_BF16 || PAGED) ? 4 : 2;
    static constexpr int QIT = IT / kUnits;                // steps per unit
    static constexpr uint32_t kUnitElems = kBlock / kUnits;
    // stage layout: codes, then plane a, then plane b
    static constexpr uint32_t kCodeBytes = kUnitElems / 2;
    static constexpr uint32_t kABytes = (DT == SZ_BF16) ? kUnitElems : kUnitElems / 8;
    static constexpr uint32_t kBBytes = (DT == SZ_BF16) ? 0 : kUnitElems / 4;
    static constexpr uint32_t kA = kCodeBytes, kB = kCodeBytes + kABytes;
    static constexpr uint32_t kBytes = kCodeBytes + kABytes + kBBytes;
    // units issued ahead of the one being decoded; the unit of a block at which
    // the next block's claim must be known (its first unit gets issued there),
    // and the one after, where the next block's first escapes are fetched
    static constexpr int kAhead = kUnits == 4 ? 3 : 2;
    static constexpr int kResolveQ = kUnits - kAhead;
    static constexpr int kEscQ = kResolveQ + 1;
    static_assert(kAhead < kStages && kEscQ < kUnits, "ring geometry");
};

template <uint32_t kStageBytes>
struct alignas(128) WarpSmem {
    uint8_t stage[kStages][kStageBytes];
    uint32_t tab[256];       // code byte -> pre-spread exponent pair
    uint64_t bar[kStages];   // one mbarrier per stage
};

// One lane's share of one step: codes and planes.
struct DFrag {
    uint32_t c0, c1;  // nibble codes (BF16: c0 only)
    uint32_t a, b;    // BF16: sm bytes 0-3, 4-7 ; E5M2: 16 sign bits, 16 x 2 mantissa bits
};

// Per-warp decode state for the tensor it is working on.
struct WarpStream {
    int t;                        // tensor, -1 if none yet
    bool ok;                      // header passed every check
    bool raw_ok;                  // the stream may hold raw blocks (header flag)
    uint32_t nb;                  // 4096-element blocks
    uint64_t n, E;
    uint64_t code, pa, pb, esc;   // section offsets in the stream
    uint32_t xt[4];               // E5M2: byte c = exponent of code c, times 4 (byte 15: 0)
};

// Step `it` (within a unit) from the shared-memory stage at address st.
template <int DT, typename G>
__device__ __forceinline__ DFrag read_stage(uint32_t st, int it) {
    const uint32_t lane = threadIdx.x & 31;
    DFrag f;
    if constexpr (DT == SZ_BF16) {
        f.c0 = lds_u32(st + it * 128 + lane * 4);
        f.c1 = 0;
        const uint2 s = lds_u64(st + G::kA + it * 256 + lane * 8);
        f.a = s.x;
        f.b = s.y;
    } else {
        const uint2 c = lds_u64(st + it * 256 + lane * 8);
        f.c0 = c.x;
        f.c1 = c.y;
        f.a = lds_u16(st + G::kA + it * 64 + lane * 2);
        f.b = lds_u32(st + G::kB + it * 128 + lane * 4);
    }
    return f;
}

__device__ __forceinline__ uint32_t load_le(const uint8_t *p, int nbytes) {
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (j < nbytes) v |= uint32_t(p[j]) << (8 * j);
    return v;
}

// Step `it` of a partial block straight from global memory: only `valid`
// (< LE) elements of this lane exist.
template <int DT>
__device__ __forceinline__ DFrag read_partial(const uint8_t *comp, const WarpStream &ws, uint64_t blk,
                                              int it, int valid) {
    DFrag f = {0, 0, 0, 0};
    if (valid <= 0) return f;
    const int lane = threadIdx.x & 31;
    const uint64_t e0 = blk * kBlock + uint64_t(it) * 32 * DGeo<DT>::LE + uint64_t(lane) * DGeo<DT>::LE;
    const uint8_t *cd = comp + ws.code + e0 / 2;
    const int cbytes = (valid + 1) / 2;
    f.c0 = load_le(cd, cbytes < 4 ? cbytes : 4);
    if (cbytes > 4) f.c1 = load_le(cd + 4, cbytes - 4);
    if constexpr (DT == SZ_BF16) {
        const uint8_t *sm = comp + ws.pa + e0;
        f.a = load_le(sm, valid < 4 ? valid : 4);
        if (valid > 4) f.b = load_le(sm + 4, valid - 4);
    } else {
        f.a = load_le(comp + ws.pa + e0 / 8, (valid + 7) / 8);
        f.b = load_le(comp + ws.pb + e0 / 4, (valid + 3) / 4);
    }
    // codes of elements past n are ignored
    if (valid < 8) {
        f.c0 &= (1u << (4 * valid)) - 1u;
        f.c1 = 0;
    } else if (valid < 16) {
        f.c1 &= (valid == 8) ? 0u : ((1u << (4 * (valid - 8))) - 1u);
    }
    return f;
}

// Check tensor t's header with the warp; on success fill the code tables.
// BF16: the shared code-pair table, tab[b] = exponents of the two codes in
// byte b pre-spread for reassembly (e_even | e_odd << 16); E5M2: the register
// table ws.xt.  Code 15 gives 0 in both.
template <int DT, int MAXB>
__device__ __forceinline__ void warp_open_stream(const DecodeParams<MAXB> &p, int t, uint32_t *tab, WarpStream &ws) {
    const int lane = threadIdx.x & 31;
    const uint8_t *comp = p.comp[t];
    const uint32_t hw = lane < 12 ? reinterpret_cast<const uint32_t *>(comp)[lane] : 0u;
    uint32_t w[12];
#pragma unroll
    for (int i = 0; i < 12; ++i) w[i] = __shfl_sync(0xffffffffu, hw, i);
    const uint64_t n = p.n[t];
    const uint64_t hn = uint64_t(w[2]) | (uint64_t(w[3]) << 32);
    const uint64_t E = uint64_t(w[4]) | (uint64_t(w[5]) << 32);
    const uint64_t total = uint64_t(w[10]) | (uint64_t(w[11]) << 32);
    const uint32_t cbw[4] = {w[6], w[7], w[8], w[9]};
    bool ok = w[0] == kMagic && (w[1] & 0xFF00FFFFu) == (header_vtag(DT) & 0xFF00FFFFu) &&
              ((w[1] >> 16) & 0xFFu) == uint32_t(DT) && hn == n && E <= n && ((w[9] >> 24) & ~kFlagRawBlocks) == 0 &&
              total == stream_layout(DT, n, E).total && total <= p.comp_bytes[t];
    // codebook: 15 distinct values inside the exponent range
    bool cb_ok = true;
    if (lane < int(kCodes)) {
        const uint32_t c = cb_byte(cbw, lane);
        cb_ok = c < uint32_t(Dt<DT>::kBins);
        for (int d = 0; d < lane; ++d) cb_ok = cb_ok && cb_byte(cbw, d) != c;
    }
    ok = __all_sync(0xffffffffu, ok && cb_ok);
    if (!ok && lane == 0) {
        const bool dtype_mismatch = w[0] == kMagic && ((w[1] >> 16) & 0xFFu) != uint32_t(DT);
        set_error(p.ctl, dtype_mismatch ? SZ_ERR_UNSUPPORTED_DTYPE : SZ_ERR_CORRUPT_STREAM, uint32_t(t));
    }
    if (ok && DT == SZ_BF16) {
        for (int b = lane; b < 256; b += 32) {
            const uint32_t c0 = b & 15, c1 = b >> 4;
            const uint32_t e0 = c0 < kCodes ? cb_byte(cbw, int(c0)) : 0u;
            const uint32_t e1 = c1 < kCodes ? cb_byte(cbw, int(c1)) : 0u;
            tab[b] = e0 | (e1 << 16);
        }
    }
    __syncwarp();
    const Layout L = stream_layout(DT, n, ok ? E : 0);
    ws.t = t;
    ws.ok = ok;
    ws.raw_ok = ((w[9] >> 24) & kFlagRawBlocks) != 0;
    ws.nb = uint32_t(L.nb);
    ws.n = n;
    ws.E = E;
    ws.code = L.code;
    ws.pa = L.plane[0];
    ws.pb = L.plane[1];
    ws.esc = L.esc;
    // E5M2 exponents are below 32, so every byte of the x4 table stays below
    // 128: a selector nibble with its top bit set reads as zero (see prmt).
    // Byte 15 (code 15) is 0: the flags byte is masked off.
#pragma unroll
    for (int i = 0; i < 4; ++i) ws.xt[i] = ok ? ((i == 3 ? (cbw[i] & 0x00FFFFFFu) : cbw[i]) << 2) : 0u;
}

// Section offsets of a tensor's stream; they depend on n only.
struct StreamGeo {
    const uint8_t *comp;
    uint64_t code, pa, pb;
};

template <int DT, int MAXB>
__device__ __forceinline__ StreamGeo stream_geo(const DecodeParams<MAXB> &p, int t) {
    const Layout L = stream_layout(DT, p.n[t], 0);
    StreamGeo g;
    g.comp = p.comp[t];
    g.code = L.code;
    g.pa = L.plane[0];
    g.pb = L.plane[1];
    return g;
}

// Lane 0 starts the bulk copies of unit q of block blk into a stage.
template <typename G>
__device__ __forceinline__ void issue_unit(uint8_t *st, uint64_t *bar, const StreamGeo &sg, uint64_t blk, int q) {
    const uint64_t u = blk * G::kUnits + q;  // unit index within the tensor
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, G::kBytes);
    bulk_g2s(st, sg.comp + sg.code + u * G::kCodeBytes, G::kCodeBytes, bar);
    bulk_g2s(st + G::kA, sg.comp + sg.pa + u * G::kABytes, G::kABytes, bar);
    if (G::kBBytes) bulk_g2s(st + G::kB, sg.comp + sg.pb + u * G::kBBytes, G::kBBytes, bar);
}

// Add escape exponent e of element j (of this lane's LE elements) into o.
template <int DT>
__device__ __forceinline__ void patch(uint32_t (&o)[4], uint32_t j, uint32_t e) {
    uint32_t k, add;
    if constexpr (DT == SZ_BF16) {
        k = j >> 1;
        add = e << (7 + 16 * (j & 1));
    } else {
        k = j >> 2;
        add = e << (2 + 8 * (j & 3));
    }
    o[0] += (k == 0) ? add : 0u;
    o[1] += (k == 1) ? add : 0u;
    o[2] += (k == 2) ? add : 0u;
    o[3] += (k == 3) ? add : 0u;
}

// Escapes of one step by the general path: warp prefix of the per-lane counts c
// and a per-lane loop over the escape flags m (bit 4j: element j), patching
// each escape's exponent into o.
template <int DT, typename M>
__device__ __forceinline__ void patch_escapes(uint32_t (&o)[4], M m, uint32_t c, uint32_t &running,
                                              uint32_t esc_reg, const uint8_t *esc_g, uint32_t cnt, bool &bad) {
    uint32_t tot;
    const uint32_t prefix = warp_exclusive_prefix(c, &tot);
    const uint32_t maxc = __reduce_max_sync(0xffffffffu, c);
    M mm = m;
    for (uint32_t i = 0; i < maxc; ++i) {
        const uint32_t r = running + prefix + i;
        const uint32_t v = __shfl_sync(0xffffffffu, esc_reg, r & 31);
        if (i < c) {
            // element, in element order
            const uint32_t j = uint32_t((DT == SZ_BF16) ? __ffs(uint32_t(mm)) - 1 : __ffsll(uint64_t(mm)) - 1) >> 2;
            mm &= mm - 1;
            uint32_t e = 0;
            if (r < cnt) e = (r < 32) ? v : uint32_t(esc_g[r]);
            else bad = true;
            if (DT == SZ_FP8_E5M2 && e >= 32u) bad = true;
            patch<DT>(o, j, e & (Dt<DT>::kBins - 1));
        }
    }
    running += tot;
}

// Decode one step.  running: escapes of the block before this step (updated);
// esc_reg: lane i holds the block's escape i (i < 32); esc_g: the block's
// escapes in global memory; cnt: escapes the offsets table gives the block.
template <int DT, bool PARTIAL, bool CHECKED = false>
__device__ __forceinline__ void decode_step(const DFrag &f, uint32_t tab, const uint32_t (&xt)[4],
                                            uint8_t *dst, int valid, uint32_t &running, uint32_t esc_reg,
                                            const uint8_t *esc_g, uint32_t cnt, bool &bad, bool store = true) {
    uint32_t o[4];
    if constexpr (DT == SZ_BF16) {
        const uint32_t cw = f.c0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t e2 = lds_u32(tab + (((cw >> (8 * k)) & 0xFFu) << 2));
            const uint32_t x = __byte_perm((k < 2) ? f.a : f.b, 0, (k & 1) ? 0x4342 : 0x4140);
            o[k] = x + (x & 0x00800080u) * 0xFFu + (e2 << 7);
        }
        const uint32_t m = escape_nibbles(cw);  // bit 4j: element j is escaped
        const uint32_t c = __popc(m);
        const uint32_t any = __ballot_sync(0xffffffffu, c != 0);
        if (any == 0) {
            // no escape in this step
        } else if (__ballot_sync(0xffffffffu, c > 1) == 0) {
            // at most one escape per lane: its rank counts the lanes before it that have one
            const uint32_t lane = threadIdx.x & 31;
            const uint32_t r = running + __popc(any & ((1u << lane) - 1u));
            const uint32_t v = __shfl_sync(0xffffffffu, esc_reg, r & 31);
            if (c) {
                const uint32_t j = uint32_t(__ffs(m) - 1) >> 2;
                uint32_t e = 0;
                if (r < cnt) e = (r < 32) ? v : uint32_t(esc_g[r]);
                else bad = true;
                patch<DT>(o, j, e & 0xFFu);
            }
            running += __popc(any);
        } else {
            patch_escapes<DT>(o, m, c, running, esc_reg, esc_g, cnt, bad);
        }
    } else {
        // Escapes first.  With one escape in a lane (the usual case) its exponent
        // takes the place of code 15's byte in this lane's table, so the lookups
        // below produce it directly.  The common step -- at most one escape per
        // lane, in a block with at most 32 -- runs straight through: the rank
        // counts the lanes before this one that have an escape, the exponent
        // comes from esc_reg (masked to 5 bits for the block), and a lane
        // without an escape loads some other lane's byte into a slot it never
        // selects.  Otherwise: with two escapes in a lane both read that byte
        // and the second (in element order) is corrected by the difference of
        // the two exponents, which never carries out of its byte; ranks come
        // from the ballots of "has one" and "has two".  Three or more (rare)
        // take the general path.  Escapes read from global memory (rank 32 and
        // up) are checked here; a stream with more escapes than the block's
        // count gives a count mismatch at the block's end.
        const uint32_t n0 = escape_nibbles(f.c0), n1 = escape_nibbles(f.c1);
        const uint64_t m = uint64_t(n0) | (uint64_t(n1) << 32);
        const uint32_t fl = n0 | (n1 << 1);  // one bit per escaped element
        const uint32_t any = __ballot_sync(0xffffffffu, fl != 0u);
        const uint32_t multi = __ballot_sync(0xffffffffu, (fl & (fl - 1u)) != 0u);
        uint32_t xt3 = xt[3];
        bool general = false;
        uint32_t two = 0, fix_k = 0, fix_add = 0, c = 0;
        if (multi == 0u && cnt <= 32u) {
            const uint32_t r = running + __popc(any & lanemask_lt());
            xt3 += __shfl_sync(0xffffffffu, esc_reg, r) << 26;  // source lane r mod 32
            running += __popc(any);
        } else {
            c = __popc(n0) + __popc(n1);
            two = multi;
            if (__ballot_sync(0xffffffffu, c > 2) == 0) {
                const uint32_t lt = lanemask_lt();
                const uint32_t r = running + __popc(any & lt) + __popc(two & lt);
                const uint32_t v = __shfl_sync(0xffffffffu, esc_reg, r & 31);
                if (c) {
                    uint32_t e = v;
                    if (r >= 32) {
                        e = r < cnt ? uint32_t(esc_g[r]) : 0u;
                        bad = bad || e >= 32u;
                    }
                    xt3 = (xt3 & 0x00FFFFFFu) | ((e & 31u) << 26);  // table byte 15 = exponent x 4 (< 128)
                    fix_add = e;
                }
                if (two) {
                    const uint32_t v2 = __shfl_sync(0xffffffffu, esc_reg, (r + 1) & 31);
                    if (c == 2) {
                        uint32_t e2 = v2;
                        if (r + 1 >= 32) {
                            e2 = r + 1 < cnt ? uint32_t(esc_g[r + 1]) : 0u;
                            bad = bad || e2 >= 32u;
                        }
                        // the second escape: the highest flagged nibble
                        const uint32_t j = n1 ? 8u + ((31u - __clz(n1)) >> 2) : (31u - __clz(n0)) >> 2;
                        fix_k = j >> 2;
                        fix_add = ((e2 & 31u) - (fix_add & 31u)) << (2 + 8 * (j & 3));
                    } else {
                        fix_add = 0;
                    }
                }
                running += __popc(any) + __popc(two);
            } else {
                general = true;
                two = 0;
            }
        }
        // four codes per word select their exponents from the register table:
        // codes 0-7 from bytes 0-7, codes 8-15 from bytes 8-15 (selector with
        // the top bit flipped, so each half reads zero for the other's codes)
        const uint32_t x0 = f.c0 ^ 0x88888888u, x1 = f.c1 ^ 0x88888888u;
        const uint32_t ev = f.b & 0x33333333u, od = f.b & 0xCCCCCCCCu;  // mantissas 0, 2 / 1, 3 of each byte
        const uint32_t ahi = f.a >> 8;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t cw = (k < 2) ? f.c0 : f.c1, cx = (k < 2) ? x0 : x1;
            const uint32_t sl = (k & 1) ? (cw >> 16) : cw, sh = (k & 1) ? (cx >> 16) : cx;
            const uint32_t e_lo = prmt(xt[0], xt[1], sl), e_hi = prmt(xt[2], xt3, sh);
            // Spreads by multiplication (the partial products never overlap a
            // kept bit): sign bits 4k..4k+3 of plane a to bit 7 of bytes 0-3,
            // the four 2-bit mantissas of byte k of plane b to bits 0-1.
            const uint32_t sa = (k < 2) ? f.a : ahi;
            const uint32_t sg = (k & 1) ? (sa & 0xF0u) * 0x01020408u : (sa & 0x0Fu) * 0x10204080u;
            const uint32_t mn = prmt(ev, 0u, 0x4440u + uint32_t(k)) * 0x1001u +
                                prmt(od, 0u, 0x4440u + uint32_t(k)) * 0x40040u;
            o[k] = ((sg & 0x80808080u) | e_hi) | ((mn & 0x03030303u) | e_lo);
        }
        if (two != 0u || general) {
            if (two) {
#pragma unroll
                for (int k = 0; k < 4; ++k) o[k] += (fix_k == uint32_t(k)) ? fix_add : 0u;
            } else {
                patch_escapes<DT>(o, m, c, running, esc_reg, esc_g, cnt, bad);
            }
        }
    }
    if (CHECKED && !store) {
        // an output page outside the pool: nothing is written
    } else if (!PARTIAL) {
        *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    } else if constexpr (DT == SZ_BF16) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < valid) reinterpret_cast<uint16_t *>(dst)[j] = uint16_t(o[j >> 1] >> (16 * (j & 1)));
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < valid) dst[j] = uint8_t(o[j >> 2] >> (8 * (j & 3)));
    }
}

// Decode one step of a raw block: the code nibbles are the low four exponent
// bits; hs points at this lane's share of the block's high bits in the escape
// section (BF16: a high nibble per element, E5M2: bit 4 per element).  Only
// `valid` elements exist (LE for a full step).  Rare by construction: plain
// per-element code.
template <int DT, bool PARTIAL, bool CHECKED>
__device__ __forceinline__ void raw_step_body(const DFrag &f, const uint8_t *hs, uint8_t *dst, int valid,
                                              bool store) {
    constexpr int LE = DGeo<DT>::LE;
    const int hbytes = (DT == SZ_BF16) ? (valid + 1) / 2 : (valid + 7) / 8;
    uint32_t hi = 0;
    for (int b = 0; b < hbytes; ++b) hi |= uint32_t(hs[b]) << (8 * b);
    uint32_t o[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < LE; ++j) {
        const uint32_t lo = (((j < 8) ? f.c0 : f.c1) >> (4 * (j & 7))) & 0xFu;
        if constexpr (DT == SZ_BF16) {
            const uint32_t e = lo | (((hi >> (4 * j)) & 0xFu) << 4);
            const uint32_t sm = (((j < 4) ? f.a : f.b) >> (8 * (j & 3))) & 0xFFu;
            const uint32_t v = ((sm & 0x80u) << 8) | (e << 7) | (sm & 0x7Fu);
            o[j >> 1] |= v << (16 * (j & 1));
        } else {
            const uint32_t e = lo | (((hi >> j) & 1u) << 4);
            const uint32_t sg = (f.a >> j) & 1u, mt = (f.b >> (2 * j)) & 3u;
            o[j >> 2] |= ((sg << 7) | (e << 2) | mt) << (8 * (j & 3));
        }
    }
    if (CHECKED && !store) {
        // an output page outside the pool: nothing is written
    } else if (!PARTIAL) {
        *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    } else if constexpr (DT == SZ_BF16) {
        for (int j = 0; j < valid; ++j) reinterpret_cast<uint16_t *>(dst)[j] = uint16_t(o[j >> 1] >> (16 * (j & 1)));
    } else {
        for (int j = 0; j < valid; ++j) dst[j] = uint8_t(o[j >> 2] >> (8 * (j & 3)));
    }
}

template <int DT, bool PARTIAL>
__device__ __noinline__ void raw_step_outlined(const DFrag &f, const uint8_t *hs, uint8_t *dst, int valid) {
    raw_step_body<DT, PARTIAL, false>(f, hs, dst, valid, true);
}

// A raw step inside the coded loop of the contiguous BF16 kernel, as a call:
// that leaves its coded path fastest (measured).
template <int DT, bool PARTIAL>
__device__ __forceinline__ void decode_step_raw(const DFrag &f, const uint8_t *hs, uint8_t *dst, int valid) {
    if constexpr (DT == SZ_BF16) raw_step_outlined<DT, PARTIAL>(f, hs, dst, valid);
    else raw_step_body<DT, PARTIAL, false>(f, hs, dst, valid, true);
}

// This lane's high bits of step `it` of a raw block within the block's escape
// section esc_g.
template <int DT>
__device__ __forceinline__ const uint8_t *raw_high(const uint8_t *esc_g, int it) {
    const uint32_t local = uint32_t(it) * 32 * DGeo<DT>::LE + (threadIdx.x & 31) * DGeo<DT>::LE;
    return esc_g + ((DT == SZ_BF16) ? local / 2 : local / 8);
}

// Offsets-table entries of a block and their checks.
struct BlockEsc {
    uint32_t lo, hi;
};

__device__ __forceinline__ BlockEsc load_offsets(const uint8_t *comp, uint64_t blk) {
    const uint32_t *tabw = reinterpret_cast<const uint32_t *>(comp + 64);
    BlockEsc b;
    b.lo = tabw[blk];
    b.hi = tabw[blk + 1];
    return b;
}

__device__ __forceinline__ bool offsets_ok(const BlockEsc &b, const WarpStream &ws, uint64_t blk) {
    return b.lo <= b.hi && b.hi <= ws.E && b.hi - b.lo <= kBlock && (blk != 0 || b.lo == 0) &&
           (blk + 1 != ws.nb || b.hi == ws.E);
}

__device__ __forceinline__ uint32_t load_escape_reg(const uint8_t *comp, const WarpStream &ws,
                                                    const BlockEsc &b) {
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t cnt = b.hi >= b.lo ? b.hi - b.lo : 0u;
    return (lane < cnt && b.hi <= ws.E) ? uint32_t(comp[ws.esc + b.lo + lane]) : 0u;
}

// Decode raw block blk of tensor t (the warp, from global memory): codes and
// planes as read_partial gives them, high bits from the block's escape section
// esc_g.  Used by raw_pass_kernel, over what the decode kernel's coded pass
// wrote.
template <int DT, int MAXB, bool PAGED>
__device__ __forceinline__ void decode_raw_block(const DecodeParams<MAXB> &p, int t, const WarpStream &ws, uint32_t blk,
                                                 const uint8_t *esc_g) {
    using G = DGeo<DT, PAGED>;
    constexpr int EB = Dt<DT>::kElemBytes;
    const int lane = threadIdx.x & 31;
    for (int it = 0; it < G::IT; ++it) {
        const int64_t e = int64_t(blk) * kBlock + int64_t(it) * 32 * G::LE + int64_t(lane) * G::LE;
        const int64_t left = int64_t(ws.n) - e;
        const int valid = left <= 0 ? 0 : (left >= G::LE ? G::LE : int(left));
        if (valid == 0) continue;
        const DFrag f = read_partial<DT>(p.comp[t], ws, blk, it, valid);
        uint8_t *dst = p.out[t] + uint64_t(e) * EB;
        bool store = true;
        if constexpr (PAGED) {
            const uint64_t off = elem_offset<EB>(p.pg[t], uint64_t(e));
            store = off != kBadOffset;  // reported by the coded pass
            dst = p.out[t] + off;
        }
        raw_step_body<DT, true, PAGED>(f, raw_high<DT>(esc_g, it), dst, valid, store);
    }
}

template <int MAXB>
__device__ __forceinline__ uint32_t nblocks(const DecodeParams<MAXB> &p, int t) {
    return p.block_begin[t + 1] - p.block_begin[t];
}

// Warp-wide block claim.  `first` (valid in lane 0) is the result of an
// atomicAdd that lane 0 already made on tensor t's counter; if that block
// exists it is the claim.  Otherwise the other tensors are scanned, 32 per
// step starting after t, and each one whose counter is still below its block
// count is tried with an atomicAdd.  Returns the block and sets t to its
// tensor; t = -1 once every tensor's blocks are taken (counters only grow, so
// a tensor seen exhausted stays exhausted).
template <int MAXB>
__device__ __forceinline__ uint32_t claim_resolve(const DecodeParams<MAXB> &p, int &t, uint32_t first) {
    const int lane = threadIdx.x & 31;
    const uint32_t r = __shfl_sync(0xffffffffu, first, 0);
    if (r < nblocks(p, t)) return r;
    for (int base = 1; base <= p.T; base += 32) {
        const int k = base + lane;  // tensors t+1 .. t+T (mod T), t itself last
        int u = 0;
        bool open = false;
        if (k <= p.T) {
            u = t + k >= p.T ? t + k - p.T : t + k;
            open = ld_relaxed_u32(p.claim + u * kClaimStride) < nblocks(p, u);
        }
        uint32_t m = __ballot_sync(0xffffffffu, open);
        while (m) {
            const int src = __ffs(m) - 1;
            m &= m - 1;
            const int uu = __shfl_sync(0xffffffffu, u, src);
            uint32_t rr = 0;
            if (lane == 0) rr = atomicAdd(p.claim + uu * kClaimStride, 1u);
            rr = __shfl_sync(0xffffffffu, rr, 0);
            if (rr < nblocks(p, uu)) {
                t = uu;
                return rr;
            }
        }
    }
    t = -1;
    return 0;
}

// The warp's input units in claim order; the producer side of its ring.  It
// runs G::kAhead units ahead of the consumer, so it reaches the next block's
// first unit while the consumer is on unit G::kResolveQ of the current block:
// the next block is handed over (set_next) just before that.
template <int DT, int MAXB, typename G, typename WS>
struct UnitFeed {
    static constexpr int kAwait = -2;
    int t;          // tensor of the next unit to issue; -1: no more units, kAwait: next block not yet known
    uint32_t blk;   // its block within the tensor
    int q;          // its unit within the block
    bool full;      // the block has all 4096 elements (partial blocks are read directly)
    int sg_t;       // tensor whose geometry sg holds
    StreamGeo sg;
    uint32_t v;     // units issued so far

    __device__ __forceinline__ void start(const DecodeParams<MAXB> &p, int t0, uint32_t blk0) {
        sg_t = -1;
        v = 0;
        set_next(p, t0, blk0);
    }
    __device__ __forceinline__ void set_next(const DecodeParams<MAXB> &p, int tn, uint32_t bn) {
        t = tn;
        blk = bn;
        q = 0;
        full = false;
        if (tn >= 0) {
            if (tn != sg_t) {
                sg = stream_geo<DT, MAXB>(p, tn);
                sg_t = tn;
            }
            full = (uint64_t(bn) + 1) * kBlock <= p.n[tn];
        }
    }
    // Issue the next unit into stage v % kStages (if it is part of a full
    // block); returns the bit to set in the issued mask.
    __device__ __forceinline__ uint32_t issue_next(WS &W) {
        if (t < 0) return 0;
        const int st = int(v % kStages);
        uint32_t bit = 0;
        if (full) {
            if ((threadIdx.x & 31) == 0) issue_unit<G>(W.stage[st], &W.bar[st], sg, blk, q);
            bit = 1u << st;
        }
        ++v;
        if (++q == G::kUnits) t = kAwait;
        return bit;
    }
};

template <int DT, int MAXB, bool PAGED>
__device__ __forceinline__ void decode_body(const DecodeParams<MAXB> &p) {
    constexpr int NW = dec_threads<DT>() / 32;
    using G = DGeo<DT, PAGED>;
    using WS = WarpSmem<G::kBytes>;
    extern __shared__ __align__(128) uint8_t s_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WS &W = reinterpret_cast<WS *>(s_raw)[warp];
    const uint32_t tab_addr = smem_u32(W.tab);
    if (lane == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(&W.bar[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    pdl_wait();  // nothing above touches global memory (programmatic launch)
    pdl_launch_dependents();

    // Blocks are claimed one at a time from per-tensor counters, one block
    // ahead of the one being decoded.  Each warp starts in the tensor that
    // holds its proportional share of the launch's blocks, stays there while
    // it has blocks, then moves to any tensor that still has some.
    const uint64_t nwarps = uint64_t(gridDim.x) * NW;
    const uint64_t gw = uint64_t(blockIdx.x) * NW + warp;
    int t = find_tensor<uint32_t, MAXB>(p.block_begin, p.T, uint32_t(uint64_t(p.total_blocks) * gw / nwarps));
    uint32_t first = 0;
    if (lane == 0) first = atomicAdd(p.claim + t * kClaimStride, 1u);
    uint32_t blk = claim_resolve<MAXB>(p, t, first);

    uint32_t issued = 0;  // bit s: stage s holds an issued unit not yet waited for
    uint32_t parity = 0;  // bit s: parity of stage s's next completion
    if (t >= 0) {
        UnitFeed<DT, MAXB, G, WS> feed;
        feed.start(p, t, blk);
        for (int k = 0; k < G::kAhead; ++k) issued |= feed.issue_next(W);

        WarpStream ws;
        // BF16 reads the block's offsets-table entries (inside the buffer: the
        // host checked its size) beside the header, not after it (per-layer
        // decode 1.4% faster; E5M2 0.8% slower, so it keeps the other order)
        BlockEsc be;
        if constexpr (DT == SZ_BF16) be = load_offsets(p.comp[t], blk);
        warp_open_stream<DT, MAXB>(p, t, W.tab, ws);
        if constexpr (DT != SZ_BF16) be = load_offsets(p.comp[t], blk);
        uint32_t esc_reg = ws.ok ? load_escape_reg(p.comp[t], ws, be) : 0u;
        uint32_t v = 0;  // units consumed

        while (true) {
            const uint8_t *comp = p.comp[t];
            uint32_t pend = 0;  // claim of the next block, resolved at unit G::kResolveQ
            if (lane == 0) pend = atomicAdd(p.claim + t * kClaimStride, 1u);
            int t_n = t;
            uint32_t blk_n = 0;
            BlockEsc be_n = {0, 0};
            uint32_t esc_n = 0;

            const bool ok = ws.ok && offsets_ok(be, ws, blk);
            const uint32_t cnt = ok ? be.hi - be.lo : 0u;
            const uint8_t *esc_g = comp + ws.esc + be.lo;
            constexpr int EB = Dt<DT>::kElemBytes;
            uint8_t *out = p.out[t] + (uint64_t(blk) * kBlock + uint64_t(lane) * G::LE) * EB;
            const bool full = (uint64_t(blk) + 1) * kBlock <= ws.n;
            // a raw block: its count is exactly raw_block_bytes (a coded block has fewer escapes)
            const bool raw = ok && ws.raw_ok &&
                             cnt == raw_block_bytes<DT>(full ? kBlock : uint32_t(ws.n - uint64_t(blk) * kBlock));
            // paged output: lane q < G::kUnits looks up where unit q of the block goes
            uint64_t qoff = 0;
            if constexpr (PAGED) {
                if (lane < G::kUnits && uint64_t(blk) * kBlock + uint64_t(lane) * G::kUnitElems < ws.n)
                    qoff = elem_offset<EB>(p.pg[t], uint64_t(blk) * kBlock + uint64_t(lane) * G::kUnitElems);
            }
            uint32_t running = 0;
            // E5M2: the block's first 32 escape bytes, held in esc_reg, must be exponents
            bool bad = DT == SZ_FP8_E5M2 && __any_sync(0xffffffffu, esc_reg >= 32u), timed_out = false;
            if (DT == SZ_FP8_E5M2) esc_reg &= 31u;
            for (int q = 0; q < G::kUnits; ++q, ++v) {
                if (q == G::kResolveQ) {
                    blk_n = claim_resolve<MAXB>(p, t_n, pend);
                    feed.set_next(p, t_n, blk_n);
                    if (t_n == t && ws.ok) be_n = load_offsets(comp, blk_n);
                }
                issued |= feed.issue_next(W);
                const int st = int(v % kStages);
                if (issued & (1u << st)) {
                    timed_out = timed_out || !mbar_wait(&W.bar[st], (parity >> st) & 1u, kWaitLimitNs);
                    parity ^= 1u << st;
                    issued &= ~(1u << st);
                }
                if (q == G::kEscQ && t_n == t && ws.ok) esc_n = load_escape_reg(comp, ws, be_n);
                if (ok && !timed_out) {
                    if (full) {
                        const uint32_t st_addr = smem_u32(W.stage[st]);
                        if constexpr (PAGED) {
                            const uint64_t off = __shfl_sync(0xffffffffu, qoff, q);
                            const bool store = off != kBadOffset;
                            uint8_t *out_q = p.out[t] + off + uint64_t(lane) * G::LE * EB;
                            if (!store && lane == 0) set_error(p.ctl, SZ_ERR_INVALID_ARG, p.block_begin[t] + blk);
#pragma unroll
                            for (int it = 0; it < G::QIT; ++it) {
                                const DFrag f = read_stage<DT, G>(st_addr, it);
                                decode_step<DT, false, true>(f, tab_addr, ws.xt, out_q + it * 512, G::LE, running,
                                                             esc_reg, esc_g, cnt, bad, store);
                            }
                        } else if (DT == SZ_BF16 && raw) {
                            for (int it = 0; it < G::QIT; ++it)
                                decode_step_raw<DT, false>(read_stage<DT, G>(st_addr, it),
                                                           raw_high<DT>(esc_g, q * G::QIT + it),
                                                           out + (q * G::QIT + it) * 512, G::LE);
                        } else {
#pragma unroll
                            for (int it = 0; it < G::QIT; ++it) {
                                const DFrag f = read_stage<DT, G>(st_addr, it);
                                decode_step<DT, false>(f, tab_addr, ws.xt, out + (q * G::QIT + it) * 512, G::LE,
                                                       running, esc_reg, esc_g, cnt, bad);
                            }
                        }
                    } else {
                        for (int it = q * G::QIT; it < (q + 1) * G::QIT; ++it) {
                            const int64_t e = int64_t(blk) * kBlock + int64_t(it) * 32 * G::LE + int64_t(lane) * G::LE;
                            const int64_t left = int64_t(ws.n) - e;
                            const int valid = left <= 0 ? 0 : (left >= G::LE ? G::LE : int(left));
                            const DFrag f = read_partial<DT>(comp, ws, blk, it, valid);
                            if constexpr (PAGED) {
                                uint8_t *dst = out;
                                bool store = valid > 0;
                                if (valid > 0) {
                                    const uint64_t off = elem_offset<EB>(p.pg[t], uint64_t(e));
                                    store = off != kBadOffset;
                                    dst = p.out[t] + off;
                                    if (!store) set_error(p.ctl, SZ_ERR_INVALID_ARG, p.block_begin[t] + blk);
                                }
                                decode_step<DT, true, true>(f, tab_addr, ws.xt, dst, valid, running, esc_reg, esc_g,
                                                            cnt, bad, store);
                            } else if (DT == SZ_BF16 && raw) {
                                decode_step_raw<DT, true>(f, raw_high<DT>(esc_g, it), out + it * 512, valid);
                            } else {
                                decode_step<DT, true>(f, tab_addr, ws.xt, out + it * 512, valid, running, esc_reg,
                                                      esc_g, cnt, bad);
                            }
                        }
                    }
                }
                __syncwarp();  // the stage just read may be refilled from here on
            }
            if constexpr (PAGED || DT == SZ_FP8_E5M2) {
                // A raw block.  The coded pass above took its low exponent nibbles
                // for codes (its escape reads stayed inside the block's section);
                // raw_pass_kernel, launched next, decodes it from its planes and
                // high bits.
                if (raw) bad = false;
            }
            if (raw) running = cnt;  // a raw block's high bits fill its count exactly
            if (ok && !timed_out) bad = __any_sync(0xffffffffu, bad) || running != cnt;
            if (lane == 0) {
                const uint32_t g = p.block_begin[t] + blk;
                if (timed_out) set_error(p.ctl, SZ_ERR_TIMEOUT, g);
                else if (ws.ok && (!ok || bad)) set_error(p.ctl, SZ_ERR_CORRUPT_STREAM, g);
            }
            if (timed_out || t_n < 0) break;  // a copy that never landed stops this warp

            // ---- advance to the claimed block
            if (t_n == t) {
                be = be_n;
                esc_reg = esc_n;
            } else {
                t = t_n;
                if constexpr (DT == SZ_BF16) be = load_offsets(p.comp[t], blk_n);
                warp_open_stream<DT, MAXB>(p, t, W.tab, ws);
                if constexpr (DT != SZ_BF16) be = load_offsets(p.comp[t], blk_n);
                esc_reg = ws.ok ? load_escape_reg(p.comp[t], ws, be) : 0u;
            }
            blk = blk_n;
        }
    }
    // wait for copies still in flight before the warp's shared memory goes away
    for (int st = 0; st < kStages; ++st)
        if (issued & (1u << st)) mbar_wait(&W.bar[st], (parity >> st) & 1u, kWaitLimitNs);

    // the last CTA out zeroes the claim counters for the next call
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&p.ctl[kCtlDecodeDone], 1u) == gridDim.x - 1) {
            for (int u = 0; u < p.T; ++u) atomicExch(p.claim + u * kClaimStride, 0u);
            atomicExch(&p.ctl[kCtlDecodeDone], 0u);
        }
    }
}

// Contiguous outputs (80 registers: 24 warps per SM).
template <int DT, int MAXB>
__global__ void __launch_bounds__(dec_threads<DT>(), 1) decode_kernel(const __grid_constant__ DecodeParams<MAXB> p) {
    decode_body<DT, MAXB, false>(p);
}

// Paged outputs: capped at 80 registers like the contiguous kernel.
template <int DT, int MAXB>
__global__ void __launch_bounds__(dec_threads<DT>(), 1) decode_kernel_paged(const __grid_constant__ DecodeParams<MAXB> p) {
    decode_body<DT, MAXB, true>(p);
}

// Second pass of the paged kernels and of the E5M2 one: one CTA per tensor
// re-reads the stream's header and, if it allows raw blocks, decodes each raw
// block from its planes and high bits over what the coded pass wrote.  A
// stream without the flag costs one header read.  Keeping raw blocks out of
// those kernels' loops keeps the loops as fast as without them (measured).
template <int DT, int MAXB, bool PAGED>
__global__ void __launch_bounds__(kRawThreads) raw_pass_kernel(const __grid_constant__ DecodeParams<MAXB> p) {
    __shared__ uint32_t s_tab[kRawWarps][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = int(blockIdx.x);
    pdl_wait();
    pdl_launch_dependents();
    if (t >= p.T || p.n[t] == 0) return;
    WarpStream ws;
    warp_open_stream<DT, MAXB>(p, t, s_tab[warp], ws);  // each warp, for its own copy of ws
    if (!ws.ok || !ws.raw_ok) return;
    const uint8_t *comp = p.comp[t];
    const uint32_t *tabw = reinterpret_cast<const uint32_t *>(comp + 64);
    for (uint32_t b0 = uint32_t(warp) * 32; b0 < ws.nb; b0 += kRawWarps * 32) {
        const uint32_t b = b0 + uint32_t(lane);
        bool raw = false;
        uint32_t lo = 0;
        if (b < ws.nb) {
            lo = tabw[b];
            const uint32_t hi = tabw[b + 1];
            const uint64_t first = uint64_t(b) * kBlock;
            const uint32_t m = uint32_t(min(uint64_t(kBlock), ws.n - first));
            raw = lo <= hi && hi <= ws.E && hi - lo == raw_block_bytes<DT>(m);
        }
        uint32_t mask = __ballot_sync(0xffffffffu, raw);
        while (mask) {
            const int l = __ffs(mask) - 1;
            mask &= mask - 1;
            const uint32_t blo = __shfl_sync(0xffffffffu, lo, l);
            decode_raw_block<DT, MAXB, PAGED>(p, t, ws, b0 + uint32_t(l), comp + ws.esc + blo);
        }
    }
}

template <int DT, int MAXB, bool PAGED>
sz_status launch_decode_t(const DecodeArgs &a, cudaStream_t stream) {
    constexpr int NT = dec_threads<DT>(), NW = NT / 32;
    auto kern = PAGED ? decode_kernel_paged<DT, MAXB> : decode_kernel<DT, MAXB>;
    const size_t smem = sizeof(WarpSmem<DGeo<DT, PAGED>::kBytes>) * NW;
    static std::atomic<int> cache[kMaxDevices];
    const int per_sm = resident_per_sm(reinterpret_cast<const void *>(kern), NT, smem, cache);
    if (per_sm < 1) return SZ_ERR_CUDA;
    DecodeParams<MAXB> p;
    p.ctl = a.ctl;
    p.claim = a.ctl + kCtlWords;  // the histogram slots
    for (int t = 0; t < a.T; ++t) p.pg[t] = page_ref(a.paged ? a.paged + t : nullptr);
    p.T = a.T;
    p.block_begin[0] = 0;
    for (int t = 0; t < a.T; ++t) {
        p.comp[t] = static_cast<const uint8_t *>(a.comp[t]);
        p.comp_bytes[t] = a.comp_bytes[t];
        p.out[t] = static_cast<uint8_t *>(a.out[t]);
        p.n[t] = a.n[t];
        p.block_begin[t + 1] = p.block_begin[t] + uint32_t(cdiv(a.n[t], kBlock));
    }
    p.total_blocks = p.block_begin[a.T];
    if (p.total_blocks == 0) return SZ_OK;
    // a CTA per SM (fewer only if there are fewer blocks than SMs); warps claim blocks
    const uint64_t resident = uint64_t(a.num_sms) * per_sm;
    const uint64_t grid = p.total_blocks < resident ? p.total_blocks : resident;
    if (launch_pdl(kern, unsigned(grid), NT, smem, stream, p) != cudaSuccess) return SZ_ERR_CUDA;
    if (PAGED || DT == SZ_FP8_E5M2)
        return launch_pdl(raw_pass_kernel<DT, MAXB, PAGED>, unsigned(a.T), kRawThreads, 0, stream, p) == cudaSuccess
                   ? SZ_OK
                   : SZ_ERR_CUDA;
    return SZ_OK;
}

}  // namespace

sz_status launch_decode(const DecodeArgs &a, cudaStream_t stream) {
    // paged outputs get their own instantiation: contiguous ones carry no paging code
    if (a.paged) {
        if (a.dtype == SZ_BF16)
            return a.T <= kSmallBatch ? launch_decode_t<SZ_BF16, kSmallBatch, true>(a, stream)
                                      : launch_decode_t<SZ_BF16, kLargeBatch, true>(a, stream);
        return a.T <= kSmallBatch ? launch_decode_t<SZ_FP8_E5M2, kSmallBatch, true>(a, stream)
                                  : launch_decode_t<SZ_FP8_E5M2, kLargeBatch, true>(a, stream);
    }
    if (a.dtype == SZ_BF16)
        return a.T <= kSmallBatch ? launch_decode_t<SZ_BF16, kSmallBatch, false>(a, stream)
                                  : launch_decode_t<SZ_BF16, kLargeBatch, false>(a, stream);
    return a.T <= kSmallBatch ? launch_decode_t<SZ_FP8_E5M2, kSmallBatch, false>(a, stream)
                              : launch_decode_t<SZ_FP8_E5M2, kLargeBatch, false>(a, stream);
}

}  // namespace sz
