// sz_decode.cu -- decode kernel: code -> exponent, escape gather, reassembly.
//
// SplitZip project page, FAQ "Is SplitZip lossy?": decoded tensors are
// bitwise identical to the originals; FAQ "How can I reduce KV cache transfer
// time ...": decompression runs on the decode GPU.  One CTA decodes one
// 4096-element tile, independently of every other tile (the stored per-block
// escape offsets make decode a pure gather):
//   1. plane and code loads (issued before the header check: the host has
//      already checked that the buffer holds the smallest stream for n);
//   2. header and offsets checks -- a stream that fails one sets
//      SZ_ERR_CORRUPT_STREAM and the tile writes nothing;
//   3. escape ranks by a CTA prefix sum; the count must match the tile's
//      offsets; the code -> exponent map is a 16-byte shared-memory table;
//   4. elements reassembled with byte permutes and written with 16-byte stores.
#include "sz_common.cuh"
#include "sz_internal.h"

namespace sz {

namespace {

constexpr int NT = kTileThreads;

// Load `nbytes` (<= 8) bytes at p into (lo, hi), byte by byte.
__device__ __forceinline__ void load_bytes(const uint8_t *p, int nbytes, uint32_t &lo, uint32_t &hi) {
    lo = hi = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (j < nbytes) {
            const uint32_t b = p[j];
            if (j < 4) lo |= b << (8 * j); else hi |= b << (8 * (j - 4));
        }
    }
}

template <int DT, int MAXB>
__global__ void __launch_bounds__(NT) decode_kernel(const __grid_constant__ DecodeParams<MAXB> p) {
    __shared__ uint32_t s_hdr[12];
    __shared__ uint32_t s_off[2];
    __shared__ uint32_t s_warp[NT / 32];
    __shared__ uint32_t s_bad;
    __shared__ uint8_t s_cb[16];
    const int tid = threadIdx.x;
    const uint32_t job = blockIdx.x;
    const int t = find_tensor<uint32_t, MAXB>(p.tile_begin, p.T, job);
    const uint32_t tile = job - p.tile_begin[t];
    const uint64_t n = p.n[t];
    const uint8_t *comp = p.comp[t];
    uint8_t *out = p.out[t];
    // the plane and code positions depend on n only (not on E)
    const Layout L0 = stream_layout(DT, n, 0);
    if (tid < 12) s_hdr[tid] = reinterpret_cast<const uint32_t *>(comp)[tid];
    if (tid < 2) s_off[tid] = reinterpret_cast<const uint32_t *>(comp + 64)[tile + tid];
    if (tid == 0) s_bad = 0;

    // ---- 1. loads
    constexpr int G = (DT == SZ_BF16) ? 2 : 1;
    constexpr int kGE = (DT == SZ_BF16) ? 8 : 16;
    const uint64_t e_tile = uint64_t(tile) * kBlock;
    uint64_t e0[G];
    int valid[G];
    uint32_t cw[G][2], pa[G], pb[G];  // codes; BF16: sm lo/hi ; E5M2: sign, mantissa
#pragma unroll
    for (int g = 0; g < G; ++g) {
        e0[g] = e_tile + uint64_t(g) * (kBlock / 2) + uint64_t(tid) * kGE;
        valid[g] = n > e0[g] ? int(min(uint64_t(kGE), n - e0[g])) : 0;
        cw[g][0] = cw[g][1] = pa[g] = pb[g] = 0;
        if constexpr (DT == SZ_BF16) {
            const uint8_t *cd = comp + L0.code + e0[g] / 2;
            const uint8_t *sm = comp + L0.plane[0] + e0[g];
            if (valid[g] == 8) {
                cw[g][0] = __ldcs(reinterpret_cast<const unsigned int *>(cd));
                const uint2 s = __ldcs(reinterpret_cast<const uint2 *>(sm));
                pa[g] = s.x;
                pb[g] = s.y;
            } else if (valid[g] > 0) {
                uint32_t unused;
                load_bytes(cd, (valid[g] + 1) / 2, cw[g][0], unused);
                load_bytes(sm, valid[g], pa[g], pb[g]);
            }
        } else {
            const uint8_t *sg = comp + L0.plane[0] + e0[g] / 8;
            const uint8_t *mt = comp + L0.plane[1] + e0[g] / 4;
            const uint8_t *cd = comp + L0.code + e0[g] / 2;
            if (valid[g] == 16) {
                pa[g] = __ldcs(reinterpret_cast<const unsigned short *>(sg));
                pb[g] = __ldcs(reinterpret_cast<const unsigned int *>(mt));
                const uint2 c = __ldcs(reinterpret_cast<const uint2 *>(cd));
                cw[g][0] = c.x;
                cw[g][1] = c.y;
            } else if (valid[g] > 0) {
                uint32_t unused;
                load_bytes(sg, (valid[g] + 7) / 8, pa[g], unused);
                load_bytes(mt, (valid[g] + 3) / 4, pb[g], unused);
                load_bytes(cd, (valid[g] + 1) / 2, cw[g][0], cw[g][1]);
            }
        }
        // codes of elements past n are ignored
        if (valid[g] < kGE) {
            if (valid[g] <= 8) {
                cw[g][0] &= (valid[g] == 8) ? 0xffffffffu : ((1u << (4 * valid[g])) - 1u);
                cw[g][1] = 0;
            } else {
                cw[g][1] &= (1u << (4 * (valid[g] - 8))) - 1u;
            }
        }
    }
    __syncthreads();

    // ---- 2. header and offsets checks
    const Header H = load_header(reinterpret_cast<const uint8_t *>(s_hdr));
    const uint64_t lo = s_off[0], hi = s_off[1];
    bool ok = H.magic == kMagic && (H.vtag & 0xFF00FFFFu) == (header_vtag(DT) & 0xFF00FFFFu) &&
              H.n == n && H.E <= n && (H.cbw[3] >> 24) == 0;
    const bool dtype_ok = ((H.vtag >> 16) & 0xFFu) == uint32_t(DT);
    ok = ok && dtype_ok;
    const Layout L = stream_layout(DT, n, ok ? H.E : 0);
    ok = ok && H.total == L.total && H.total <= p.comp_bytes[t];
    ok = ok && lo <= hi && hi <= H.E && hi - lo <= kBlock;
    ok = ok && (tile != 0 || lo == 0) && (uint64_t(tile) + 1 != L.nb || hi == H.E);
    if (tid < int(kCodes)) {
        const uint32_t c = cb_byte(H.cbw, tid);
        bool cb_ok = c < uint32_t(Dt<DT>::kBins);
        for (int d = 0; d < tid; ++d) cb_ok = cb_ok && cb_byte(H.cbw, d) != c;
        s_cb[tid] = uint8_t(c);
        if (!cb_ok) s_bad = 1;
    }
    if (tid == 15) s_cb[15] = 0;
    __syncthreads();
    if (!ok || s_bad) {
        if (tid == 0) set_error(p.ctl, dtype_ok || H.magic != kMagic ? SZ_ERR_CORRUPT_STREAM
                                                                     : SZ_ERR_UNSUPPORTED_DTYPE, job);
        return;
    }

    // ---- 3. escape ranks
    uint32_t emask[G];
    uint32_t packed = 0;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        uint32_t bits = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t c = cw[g][h];
            const uint32_t m = c & (c >> 1) & (c >> 2) & (c >> 3) & 0x11111111u;
#pragma unroll
            for (int j = 0; j < 8; ++j) bits |= ((m >> (4 * j)) & 1u) << (8 * h + j);
        }
        emask[g] = bits;
        packed |= uint32_t(__popc(bits)) << (16 * g);
    }
    uint32_t total_packed;
    const uint32_t before = block_exclusive_scan<NT>(packed, s_warp, &total_packed);
    const uint32_t tile_escapes = (total_packed & 0xFFFFu) + (total_packed >> 16);
    if (tile_escapes != hi - lo) {  // uniform across the CTA
        if (tid == 0) set_error(p.ctl, SZ_ERR_CORRUPT_STREAM, job);
        return;
    }
    const uint8_t *esc = comp + L.esc + lo;

    // ---- 4. reassemble and store
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (valid[g] <= 0) continue;
        uint32_t r = (g == 0) ? (before & 0xFFFFu) : (total_packed & 0xFFFFu) + (before >> 16);
        uint32_t ex[kGE];
#pragma unroll
        for (int j = 0; j < kGE; ++j) ex[j] = s_cb[(cw[g][j >> 3] >> (4 * (j & 7))) & 0xFu];
        uint32_t m = emask[g];
        bool bad_esc = false;
        while (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1;
            const uint32_t e = esc[r++];
            if (DT == SZ_FP8_E5M2 && e >= 32u) bad_esc = true;
#pragma unroll
            for (int q = 0; q < kGE; ++q)
                if (q == j) ex[q] = e & (Dt<DT>::kBins - 1);
        }
        if (bad_esc) set_error(p.ctl, SZ_ERR_CORRUPT_STREAM, job);
        uint32_t o[4];
        if constexpr (DT == SZ_BF16) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t src = (k < 2) ? pa[g] : pb[g];
                const uint32_t x = __byte_perm(src, 0, (k & 1) ? 0x4342 : 0x4140);
                const uint32_t e2 = ex[2 * k] | (ex[2 * k + 1] << 16);
                o[k] = (x & 0x007F007Fu) | ((x & 0x00800080u) << 8) | (e2 << 7);
            }
            uint8_t *dst = out + 2 * e0[g];
            if (valid[g] == 8) {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j < valid[g])
                        reinterpret_cast<uint16_t *>(dst)[j] = uint16_t(o[j >> 1] >> (16 * (j & 1)));
            }
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t s4 = (pa[g] >> (4 * k)) & 0xFu;
                const uint32_t sgn = ((s4 * 0x00204081u) & 0x01010101u) << 7;
                const uint32_t m8 = (pb[g] >> (8 * k)) & 0xFFu;
                const uint32_t mnt = (m8 | (m8 << 6) | (m8 << 12) | (m8 << 18)) & 0x03030303u;
                const uint32_t e4 = ex[4 * k] | (ex[4 * k + 1] << 8) | (ex[4 * k + 2] << 16) |
                                    (ex[4 * k + 3] << 24);
                o[k] = sgn | (e4 << 2) | mnt;
            }
            uint8_t *dst = out + e0[g];
            if (valid[g] == 16) {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (j < valid[g]) dst[j] = uint8_t(o[j >> 2] >> (8 * (j & 3)));
            }
        }
    }
}

template <int DT, int MAXB>
sz_status launch_decode_t(const DecodeArgs &a, cudaStream_t stream) {
    DecodeParams<MAXB> p;
    p.ctl = a.ctl;
    p.T = a.T;
    p.tile_begin[0] = 0;
    for (int t = 0; t < a.T; ++t) {
        p.comp[t] = static_cast<const uint8_t *>(a.comp[t]);
        p.comp_bytes[t] = a.comp_bytes[t];
        p.out[t] = static_cast<uint8_t *>(a.out[t]);
        p.n[t] = a.n[t];
        p.tile_begin[t + 1] = p.tile_begin[t] + uint32_t(cdiv(a.n[t], kBlock));
    }
    p.total_tiles = p.tile_begin[a.T];
    if (p.total_tiles == 0) return SZ_OK;
    decode_kernel<DT, MAXB><<<p.total_tiles, NT, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? SZ_OK : SZ_ERR_CUDA;
}

}  // namespace

sz_status launch_decode(const DecodeArgs &a, cudaStream_t stream) {
    if (a.dtype == SZ_BF16)
        return a.T <= kSmallBatch ? launch_decode_t<SZ_BF16, kSmallBatch>(a, stream)
                                  : launch_decode_t<SZ_BF16, kLargeBatch>(a, stream);
    return a.T <= kSmallBatch ? launch_decode_t<SZ_FP8_E5M2, kSmallBatch>(a, stream)
                              : launch_decode_t<SZ_FP8_E5M2, kLargeBatch>(a, stream);
}

}  // namespace sz
