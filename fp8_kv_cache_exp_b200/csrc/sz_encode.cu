// sz_encode.cu -- encode kernel: split, code, pack, escape offsets and scatter.
//
// SplitZip project page, Abstract: sign and mantissa bits are kept exactly,
// frequent exponents get fixed 4-bit codes, rare exponents go to a sparse
// escape stream.  One CTA encodes one 4096-element tile:
//   1. 16-byte loads of the tile, exponent -> code through a 256-entry
//      shared-memory table built from the plan's codebook;
//   2. sign|mantissa bytes (BF16) or sign bits + 2-bit mantissas (E5M2) and
//      the 4-bit codes stored with 4-16 byte coalesced stores;
//   3. escapes counted per thread, ranked by a CTA prefix sum, and staged in
//      shared memory in element order;
//   4. the tile's escape offset found by a single-pass decoupled look-back
//      over the tiles of its tensor (tile ids taken from an atomic counter in
//      launch order, so every predecessor is already running; every wait is
//      bounded and reports SZ_ERR_TIMEOUT instead of hanging);
//   5. staged escapes written contiguously at that offset; the tile's entry
//      of the offsets table written; the tensor's last tile also writes the
//      header, offsets[nb] and the zero padding between sections.
#include "sz_common.cuh"
#include "sz_internal.h"

namespace sz {

namespace {

constexpr int NT = kTileThreads;
constexpr uint64_t kLookbackLimitNs = 1000000000ull;  // 1 s: far above any legitimate wait
constexpr unsigned long long kFlagAgg = 1ull << 32;    // tile aggregate published
constexpr unsigned long long kFlagInc = 2ull << 32;    // inclusive prefix published

struct TileShared {
    uint32_t hdr[16];
    uint32_t warp[NT / 32];
    uint32_t excl;
    uint8_t lut[256];
    alignas(16) uint8_t esc[kBlock];
};

// Decoupled look-back, run by warp 0.  Returns the number of escapes in the
// tensor's tiles before `tile`; publishes this tile's aggregate at once and
// its inclusive prefix when known.  Status word: epoch (30 bits) << 34 |
// flag << 32 | value; words from earlier launches carry an older epoch and
// read as "not published".
__device__ uint32_t lookback(unsigned long long *st, uint32_t tile, uint32_t agg, uint32_t epoch,
                             bool *timed_out) {
    const int lane = threadIdx.x & 31;
    const unsigned long long tag = (unsigned long long)(epoch & 0x3FFFFFFFu) << 34;
    *timed_out = false;
    if (tile == 0) {
        if (lane == 0) st_relaxed_u64(st, tag | kFlagInc | agg);
        return 0;
    }
    if (lane == 0) st_relaxed_u64(st + tile, tag | kFlagAgg | agg);
    uint32_t excl = 0;
    int64_t j = int64_t(tile) - 1;  // nearest predecessor, read by lane 0
    uint64_t t0 = 0;
    uint32_t backoff = 32;
    while (true) {
        const int64_t idx = j - lane;
        uint32_t flag = 2, val = 0;  // before tile 0: a virtual inclusive 0
        if (idx >= 0) {
            const unsigned long long w = ld_relaxed_u64(st + idx);
            flag = ((w >> 34) == (tag >> 34)) ? uint32_t(w >> 32) & 3u : 0u;
            val = uint32_t(w);
        }
        const uint32_t ready = __ballot_sync(0xffffffffu, flag != 0);
        const uint32_t inc = __ballot_sync(0xffffffffu, flag == 2);
        // lanes up to and including the nearest inclusive prefix must be ready
        const uint32_t need = inc ? (((inc & (0u - inc)) << 1) - 1u) : 0xffffffffu;
        if ((ready & need) == need) {
            excl += __reduce_add_sync(0xffffffffu, ((need >> lane) & 1u) ? val : 0u);
            if (inc) break;
            j -= 32;
            continue;
        }
        uint64_t now = __shfl_sync(0xffffffffu, global_ns(), 0);
        if (t0 == 0) {
            t0 = now;
        } else if (now - t0 > kLookbackLimitNs) {
            *timed_out = true;
            break;
        }
        __nanosleep(backoff);
        if (backoff < 1024) backoff <<= 1;
    }
    if (lane == 0) st_relaxed_u64(st + tile, tag | kFlagInc | (excl + agg));
    return excl;
}

template <int DT>
__device__ __forceinline__ bool header_ok(const Header &H, uint64_t n, uint64_t cap,
                                          uint32_t *why) {
    if (H.magic != kMagic || H.vtag != header_vtag(DT) || H.n != n || H.E > n ||
        (H.cbw[3] >> 24) != 0 || H.total != stream_layout(DT, n, H.E).total) {
        *why = SZ_ERR_PLAN_MISMATCH;
        return false;
    }
    if (H.total > cap) {
        *why = SZ_ERR_BUFFER_TOO_SMALL;
        return false;
    }
    return true;
}

// Zero [a, b) of out with the whole CTA.
__device__ __forceinline__ void zero_bytes(uint8_t *out, uint64_t a, uint64_t b) {
    for (uint64_t x = a + threadIdx.x; x < b; x += NT) out[x] = 0;
}

// Header, offsets[nb] and the zero gaps between sections (done once per stream).
template <int DT>
__device__ void write_stream_frame(uint8_t *out, const Layout &L, const uint32_t *hdr, uint64_t n,
                                   uint64_t E) {
    if (threadIdx.x < 16) reinterpret_cast<uint32_t *>(out)[threadIdx.x] = hdr[threadIdx.x];
    if (threadIdx.x == 0) *reinterpret_cast<uint32_t *>(out + 64 + 4 * L.nb) = uint32_t(E);
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

// Load up to `valid` elements of 16 bytes starting at byte offset `off` of in.
template <int DT>
__device__ __forceinline__ uint4 load_group(const uint8_t *in, uint64_t off, int valid) {
    constexpr int kVec = 16 / Dt<DT>::kElemBytes;
    if (valid >= kVec) return __ldcs(reinterpret_cast<const uint4 *>(in + off));
    uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kVec; ++j) {
        if (j < valid) {
            if constexpr (DT == SZ_BF16) {
                const uint32_t b = reinterpret_cast<const uint16_t *>(in + off)[j];
                w[j >> 1] |= b << (16 * (j & 1));
            } else {
                w[j >> 2] |= uint32_t(in[off + j]) << (8 * (j & 3));
            }
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Store the low `nbytes` bytes of (lo, hi) at p; full width when nbytes == width.
__device__ __forceinline__ void store_bytes(uint8_t *p, uint32_t lo, uint32_t hi, int nbytes) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < nbytes) p[j] = uint8_t(((j < 4) ? lo : hi) >> (8 * (j & 3)));
}

template <int DT, int MAXB>
__device__ void encode_tile(const EncodeParams<MAXB> &p, uint32_t job, uint32_t epoch,
                            TileShared &S) {
    const int tid = threadIdx.x;
    const int t = find_tensor<uint32_t, MAXB>(p.tile_begin, p.T, job);
    const uint32_t tile = job - p.tile_begin[t];
    const uint64_t n = p.n[t];
    const uint8_t *in = p.in[t];
    uint8_t *out = p.out[t];
    if (tid < 16) S.hdr[tid] = tid < 12 ? reinterpret_cast<const uint32_t *>(p.plans + 64 * size_t(t))[tid] : 0u;

    // ---- 1. loads (issued before the header arrives)
    constexpr int G = (DT == SZ_BF16) ? 2 : 1;          // 16-byte groups per thread
    constexpr int kGE = (DT == SZ_BF16) ? 8 : 16;       // elements per group
    const uint64_t e_tile = uint64_t(tile) * kBlock;
    uint64_t e0[G];
    int valid[G];
    uint4 v[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        e0[g] = e_tile + uint64_t(g) * (kBlock / 2) + uint64_t(tid) * kGE;
        valid[g] = n > e0[g] ? int(min(uint64_t(kGE), n - e0[g])) : 0;
        v[g] = valid[g] > 0 ? load_group<DT>(in, e0[g] * Dt<DT>::kElemBytes, valid[g])
                            : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    Header H = load_header(reinterpret_cast<const uint8_t *>(S.hdr));
    uint32_t why = 0;
    if (!header_ok<DT>(H, n, p.cap[t], &why)) {
        if (tid == 0 && tile == 0) set_error(p.ctl, why, uint32_t(t));
        return;  // every tile of this tensor takes this branch: no look-back waits on it
    }
    // exponent -> code table
    if (tid < Dt<DT>::kBins) {
        uint32_t code = kEscape;
#pragma unroll
        for (int c = 0; c < int(kCodes); ++c)
            if (cb_byte(H.cbw, c) == uint32_t(tid)) code = uint32_t(c);
        S.lut[tid] = uint8_t(code);
    }
    __syncthreads();
    const Layout L = stream_layout(DT, n, H.E);

    // ---- 2. code, split, store
    uint32_t codes[G][2];   // nibbles of the group's elements (BF16 uses [g][0])
    uint32_t emask[G];      // escape flags, bit j = element j of the group
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const uint32_t w[4] = {v[g].x, v[g].y, v[g].z, v[g].w};
        if constexpr (DT == SZ_BF16) {
            uint32_t cw = 0, smp[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t c0 = S.lut[(w[k] >> 7) & 0xFFu];
                const uint32_t c1 = S.lut[(w[k] >> 23) & 0xFFu];
                cw |= (c0 | (c1 << 4)) << (8 * k);
                smp[k] = ((w[k] >> 8) & 0x00800080u) | (w[k] & 0x007F007Fu);
            }
            if (valid[g] < 8) cw &= (1u << (4 * valid[g])) - 1u;  // codes past n are 0
            const uint32_t sm_lo = __byte_perm(smp[0], smp[1], 0x6420);
            const uint32_t sm_hi = __byte_perm(smp[2], smp[3], 0x6420);
            codes[g][0] = cw;
            codes[g][1] = 0;
            uint32_t m = cw & (cw >> 1) & (cw >> 2) & (cw >> 3) & 0x11111111u;
            // compress nibble flags (bits 0,4,..,28) into bits 0..7
            uint32_t bits = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) bits |= ((m >> (4 * j)) & 1u) << j;
            emask[g] = bits;
            uint8_t *sm_dst = out + L.plane[0] + e0[g];
            uint8_t *cd_dst = out + L.code + e0[g] / 2;
            if (valid[g] == 8) {
                *reinterpret_cast<uint2 *>(sm_dst) = make_uint2(sm_lo, sm_hi);
                *reinterpret_cast<uint32_t *>(cd_dst) = cw;
            } else if (valid[g] > 0) {
                store_bytes(sm_dst, sm_lo, sm_hi, valid[g]);
                store_bytes(cd_dst, cw, 0, (valid[g] + 1) / 2);
            }
        } else {
            uint32_t cw[2] = {0, 0}, sign = 0, mant = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const uint32_t c = S.lut[(w[k] >> (8 * b + 2)) & 0x1Fu];
                    cw[k >> 1] |= c << (4 * (4 * (k & 1) + b));
                }
                sign |= ((((w[k] >> 7) & 0x01010101u) * 0x01020408u) >> 24) << (4 * k);
                const uint32_t x = w[k] & 0x03030303u;
                mant |= ((x | (x >> 6) | (x >> 12) | (x >> 18)) & 0xFFu) << (8 * k);
            }
            if (valid[g] < 16) {
                if (valid[g] < 8) {
                    cw[0] &= (1u << (4 * valid[g])) - 1u;
                    cw[1] = 0;
                } else {
                    cw[1] &= (valid[g] == 8) ? 0u : ((1u << (4 * (valid[g] - 8))) - 1u);
                }
            }
            codes[g][0] = cw[0];
            codes[g][1] = cw[1];
            uint32_t bits = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t m = cw[h] & (cw[h] >> 1) & (cw[h] >> 2) & (cw[h] >> 3) & 0x11111111u;
#pragma unroll
                for (int j = 0; j < 8; ++j) bits |= ((m >> (4 * j)) & 1u) << (8 * h + j);
            }
            emask[g] = bits;
            uint8_t *sg_dst = out + L.plane[0] + e0[g] / 8;
            uint8_t *mt_dst = out + L.plane[1] + e0[g] / 4;
            uint8_t *cd_dst = out + L.code + e0[g] / 2;
            if (valid[g] == 16) {
                *reinterpret_cast<uint16_t *>(sg_dst) = uint16_t(sign);
                *reinterpret_cast<uint32_t *>(mt_dst) = mant;
                *reinterpret_cast<uint2 *>(cd_dst) = make_uint2(cw[0], cw[1]);
            } else if (valid[g] > 0) {
                store_bytes(sg_dst, sign, 0, (valid[g] + 7) / 8);
                store_bytes(mt_dst, mant, 0, (valid[g] + 3) / 4);
                store_bytes(cd_dst, cw[0], cw[1], (valid[g] + 1) / 2);
            }
        }
    }

    // ---- 3. rank escapes within the tile; stage them in element order
    uint32_t packed = 0;
#pragma unroll
    for (int g = 0; g < G; ++g) packed |= uint32_t(__popc(emask[g])) << (16 * g);
    uint32_t total_packed;
    const uint32_t before = block_exclusive_scan<NT>(packed, S.warp, &total_packed);
    const uint32_t tile_escapes = (total_packed & 0xFFFFu) + (total_packed >> 16);
#pragma unroll
    for (int g = 0; g < G; ++g) {
        uint32_t r = (g == 0) ? (before & 0xFFFFu) : (total_packed & 0xFFFFu) + (before >> 16);
        uint32_t m = emask[g];
        while (m) {
            const uint32_t j = __ffs(m) - 1;
            m &= m - 1;
            uint32_t e;
            if constexpr (DT == SZ_BF16) {
                const uint32_t wj = pick4(v[g].x, v[g].y, v[g].z, v[g].w, j >> 1);
                e = (wj >> (16 * (j & 1) + 7)) & 0xFFu;
            } else {
                const uint32_t wj = pick4(v[g].x, v[g].y, v[g].z, v[g].w, j >> 2);
                e = (wj >> (8 * (j & 3) + 2)) & 0x1Fu;
            }
            S.esc[r++] = uint8_t(e);
        }
    }

    // ---- 4. escape offset of this tile within its tensor
    if (tid < 32) {
        bool timed_out;
        const uint32_t excl =
            lookback(p.status + p.tile_begin[t], tile, tile_escapes, epoch, &timed_out);
        if (tid == 0) {
            S.excl = excl;
            if (timed_out) set_error(p.ctl, SZ_ERR_TIMEOUT, job);
        }
    }
    __syncthreads();
    const uint32_t excl = S.excl;

    // ---- 5. escapes, offsets entry, and the stream frame (last tile)
    const uint64_t dst = L.esc + excl;
    for (uint32_t x = tid; x < tile_escapes; x += NT)
        if (dst + x < L.total) out[dst + x] = S.esc[x];
    if (tid == 0) {
        *reinterpret_cast<uint32_t *>(out + 64 + 4 * uint64_t(tile)) = excl;
        if (uint64_t(excl) + tile_escapes > H.E) set_error(p.ctl, SZ_ERR_PLAN_MISMATCH, job);
    }
    if (uint64_t(tile) + 1 == L.nb) {
        if (tid == 0 && uint64_t(excl) + tile_escapes != H.E)
            set_error(p.ctl, SZ_ERR_PLAN_MISMATCH, job);
        write_stream_frame<DT>(out, L, S.hdr, n, H.E);
    }
}

// Stream of an empty tensor: header, offsets[0] = 0, zero padding.
template <int DT, int MAXB>
__device__ void encode_empty(const EncodeParams<MAXB> &p, int t, TileShared &S) {
    const int tid = threadIdx.x;
    if (tid < 16) S.hdr[tid] = tid < 12 ? reinterpret_cast<const uint32_t *>(p.plans + 64 * size_t(t))[tid] : 0u;
    __syncthreads();
    const Header H = load_header(reinterpret_cast<const uint8_t *>(S.hdr));
    uint32_t why = 0;
    if (!header_ok<DT>(H, 0, p.cap[t], &why)) {
        if (tid == 0) set_error(p.ctl, why, uint32_t(t));
        return;
    }
    const Layout L = stream_layout(DT, 0, 0);
    write_stream_frame<DT>(p.out[t], L, S.hdr, 0, 0);
}

template <int DT, int MAXB>
__global__ void __launch_bounds__(NT) encode_kernel(const __grid_constant__ EncodeParams<MAXB> p) {
    __shared__ TileShared S;
    __shared__ uint32_t s_job, s_epoch;
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_job = atomicAdd(&p.ctl[kCtlTileCtr], 1u);
        s_epoch = ld_relaxed_u32(&p.ctl[kCtlEpoch]);
    }
    __syncthreads();
    const uint32_t job = s_job, epoch = s_epoch;
    if (job < p.total_tiles)
        encode_tile<DT, MAXB>(p, job, epoch, S);
    else if (job < p.total_jobs)
        encode_empty<DT, MAXB>(p, p.empty[job - p.total_tiles], S);
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

template <int DT, int MAXB>
sz_status launch_encode_t(const EncodeArgs &a, cudaStream_t stream) {
    EncodeParams<MAXB> p;
    p.ctl = a.ctl;
    p.status = a.status;
    p.plans = a.plans;
    p.T = a.T;
    p.n_empty = 0;
    p.tile_begin[0] = 0;
    for (int t = 0; t < a.T; ++t) {
        p.in[t] = static_cast<const uint8_t *>(a.in[t]);
        p.out[t] = static_cast<uint8_t *>(a.out[t]);
        p.n[t] = a.n[t];
        p.cap[t] = a.cap[t];
        p.tile_begin[t + 1] = p.tile_begin[t] + uint32_t(cdiv(a.n[t], kBlock));
        if (a.n[t] == 0) p.empty[p.n_empty++] = uint16_t(t);
    }
    p.total_tiles = p.tile_begin[a.T];
    p.total_jobs = p.total_tiles + uint32_t(p.n_empty);
    if (p.total_jobs == 0) return SZ_OK;
    encode_kernel<DT, MAXB><<<p.total_jobs, NT, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? SZ_OK : SZ_ERR_CUDA;
}

}  // namespace

sz_status launch_encode(const EncodeArgs &a, cudaStream_t stream) {
    if (a.dtype == SZ_BF16)
        return a.T <= kSmallBatch ? launch_encode_t<SZ_BF16, kSmallBatch>(a, stream)
                                  : launch_encode_t<SZ_BF16, kLargeBatch>(a, stream);
    return a.T <= kSmallBatch ? launch_encode_t<SZ_FP8_E5M2, kSmallBatch>(a, stream)
                              : launch_encode_t<SZ_FP8_E5M2, kLargeBatch>(a, stream);
}

}  // namespace sz
