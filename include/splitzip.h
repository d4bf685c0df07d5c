/*
 * splitzip.h -- C ABI of libsplitzip: lossless exponent-split coding of BF16
 * and FP8 E5M2 KV-cache tensors on a B200 (sm_100a) GPU.
 *
 * The method is the one on the SplitZip project page ("SplitZip: Ultra-Fast
 * Lossless KV Compression for Disaggregated LLM Serving"):
 *   - Abstract: exponents of BF16 KV activations are highly redundant; the
 *     most frequent exponent values get fixed 4-bit codes, sign and mantissa
 *     bits are kept exactly, and rare exponent values go through a sparse
 *     escape stream;
 *   - FAQ "Is SplitZip lossy?": decoded tensors are bitwise identical;
 *   - FAQ "How can I reduce KV cache transfer time ...": compress on the
 *     prefill GPU, decompress on the decode GPU;
 *   - FAQ "Does it work with an FP8 KV cache?": the same coding on E5M2.
 * The page prints no byte layout.  This library's stream format v1 is:
 *
 *   [0,64)  header: u32 magic 0x564B5A53 ("SZKV"), u16 version 1, u8 dtype,
 *           u8 block_log2 = 12, u64 n, u64 E (escapes), u8 cb[15] (codebook:
 *           exponent of code c), u8 flags, u64 total_bytes, 16 zero bytes
 *   [64, 64+4(nb+1))  u32 offsets[nb+1], nb = ceil(n/4096): escapes before
 *           each 4096-element block (exclusive prefix), offsets[nb] = E
 *   then, each section starting at the next multiple of 256 bytes:
 *     BF16: sm plane (n B: sign<<7 | mantissa7), code plane (ceil(n/2) B,
 *           element 2j in the low nibble of byte j), escapes (E B)
 *     E5M2: sign plane (ceil(n/8) B, element i at bit i%8 of byte i/8),
 *           mantissa plane (ceil(n/4) B, element i at bits 2(i%4)..+1 of
 *           byte i/4), code plane, escapes
 *   All multi-byte fields little-endian; every padding byte is zero.
 *   Codebook: the 15 exponent values ranked first by (count descending,
 *   value ascending); code c names cb[c]; code 15 = escape, whose exponent
 *   (zero-extended to a byte for E5M2) is the next byte of the escape stream,
 *   in element order.  The stream is a pure function of the input and the
 *   flags.
 *
 *   Header byte 39 holds the flags, 0 unless raw blocks are allowed.  With
 *   SZ_FLAG_RAW_BLOCKS, a block of m elements whose escapes would fill at
 *   least K = ceil(m/2) bytes (BF16) or ceil(m/8) bytes (E5M2) is stored raw
 *   instead: its code nibbles hold the low four bits of each exponent, and K
 *   escape-section bytes hold the rest (BF16: the high nibble of block
 *   element j's exponent in nibble j%2 of byte j/2; E5M2: bit 4 at bit j%8 of
 *   byte j/8).  The offsets table counts K for it; a coded block always has
 *   fewer escapes than K, so the count tells the two apart.  E is then the
 *   escape section's length.  A raw block costs exactly its raw bytes, so no
 *   block expands: a stream is at most the raw tensor plus header, table
 *   and section padding (uniform random bits would otherwise take some 19.5
 *   bits per BF16 element).  The project page describes no such fallback;
 *   it is this format's own extension for data the codebook does not fit.
 *
 * Conventions for every call:
 *   - Pointers named d_* are device pointers on the current device; the
 *     caller owns every buffer (inputs, outputs, workspace, plans).  The
 *     library allocates no device memory.
 *   - d_in, d_out and d_comp must be 16-byte aligned; d_ws and d_plan(s)
 *     8-byte aligned.  Inputs and outputs must not overlap.
 *   - Every call that takes a stream enqueues its work on that stream and
 *     returns without waiting, except sz_compressed_size(s) and
 *     sz_last_device_status, which synchronise the stream.
 *   - Host-detectable errors (null or misaligned pointer, n >= 2^32, too
 *     small a workspace or output, bad dtype, batch too large) are returned
 *     at once and nothing is enqueued.  Errors found on the device (corrupt
 *     stream, look-back timeout, plan/data mismatch, output capacity) are
 *     recorded in the workspace's device error word (the first error wins)
 *     and read, then cleared, by sz_last_device_status.  No call aborts,
 *     throws or traps the GPU.
 *   - CUDA graphs: the plan, encode and decode calls (contiguous, paged, reuse)
 *     only enqueue kernels on their stream -- no allocation, no synchronisation
 *     -- so a sequence of them can be captured into a CUDA graph and replayed,
 *     once each call has run on the device (its first call sets the kernel's
 *     shared-memory limit).  The buffers captured are the ones replayed.
 *   - Workspaces: size with sz_workspace_bytes*, zero once with
 *     sz_workspace_init before first use.  The kernels leave it ready for the
 *     next call.  A workspace serves one stream at a time; calls that use the
 *     same workspace concurrently on different streams race.  After a device
 *     error, call sz_workspace_init again.
 */
#ifndef SPLITZIP_H
#define SPLITZIP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef __CUDA_RUNTIME_API_H__
struct CUstream_st;
typedef struct CUstream_st *cudaStream_t;
#endif

typedef enum {
    SZ_OK = 0,
    SZ_ERR_INVALID_ARG = 1,       /* null/misaligned pointer, n >= 2^32, T out of range, n mismatch */
    SZ_ERR_UNSUPPORTED_DTYPE = 2, /* dtype not SZ_BF16 / SZ_FP8_E5M2, or stream of another dtype */
    SZ_ERR_BUFFER_TOO_SMALL = 3,  /* workspace or output capacity too small                       */
    SZ_ERR_CORRUPT_STREAM = 4,    /* stream fails a consistency check on decode                   */
    SZ_ERR_CUDA = 5,              /* a CUDA runtime call failed                                    */
    SZ_ERR_TIMEOUT = 6,           /* the escape-offset look-back waited longer than its limit      */
    SZ_ERR_PLAN_MISMATCH = 7,     /* encode data or sizes disagree with the plan                   */
    SZ_ERR_INTERNAL = 8           /* an internal consistency check failed                          */
} sz_status;

typedef enum { SZ_BF16 = 0, SZ_FP8_E5M2 = 1 } sz_dtype;

#define SZ_HEADER_BYTES 64
#define SZ_BLOCK_ELEMS 4096
#define SZ_MAX_BATCH 256
#define SZ_FORMAT_VERSION 1
#define SZ_FLAG_RAW_BLOCKS 1u /* header byte 39, bit 0: blocks that would expand are stored raw */

/* A plan is the 64-byte stream header of the tensor it was made for:
 * codebook, n, E and total_bytes.  It lives in device memory. */
typedef struct {
    unsigned char bytes[SZ_HEADER_BYTES];
} sz_plan_t;

/* A tensor held in pages of a page pool, as paged KV caches keep it: element
 * i lives at
 *     pool + pages[i / page_elems] * page_bytes + (i % page_elems) * elem_bytes
 * (elem_bytes = 2 for BF16, 1 for E5M2).  All fields are device-side data
 * described by the host; the descriptor itself is read on the host during the
 * call.
 *   pool        device base of the pool, 16-byte aligned
 *   pages       device array of ceil(n / page_elems) page ids, in element order
 *   pool_pages  number of pages in the pool; an id outside [0, pool_pages) is
 *               reported as SZ_ERR_INVALID_ARG on the device error word and
 *               that page is neither read nor written
 *   page_bytes  bytes from one page to the next, a multiple of 16 and at least
 *               page_elems * elem_bytes
 *   page_elems  elements of this tensor per page, a multiple of 1024, at most
 *               2^18 */
typedef struct {
    const void *pool;
    const int32_t *pages;
    uint64_t pool_pages;
    uint64_t page_bytes;
    uint32_t page_elems;
} sz_paged_t;

/* ------------------------------------------------------------ host-only */

/* Human-readable name of a status code (static string, never NULL). */
const char *sz_status_string(sz_status s);

/* Workspace bytes for one tensor of n elements (any of plan/encode/decode). */
size_t sz_workspace_bytes(sz_dtype dtype, uint64_t n);

/* Workspace bytes for a batch of T tensors with element counts n[0..T-1]
 * (host array).  Returns 0 if T is outside 1..SZ_MAX_BATCH. */
size_t sz_workspace_bytes_batched(sz_dtype dtype, int T, const uint64_t *n);

/* Stream length of n elements with E escapes (closed form of format v1);
 * 0 for a bad dtype. */
size_t sz_stream_bytes(sz_dtype dtype, uint64_t n, uint64_t E);

/* Largest possible stream for n elements (every element escaped, E = n). */
size_t sz_max_compressed_size(sz_dtype dtype, uint64_t n);

/* ------------------------------------------------------- stream-ordered */

/* Zero a workspace (cudaMemsetAsync).  Required once before first use and
 * after any device error. */
sz_status sz_workspace_init(void *d_ws, size_t ws_bytes, cudaStream_t stream);

/* Plan: exponent histogram and codebook (project page, Abstract: "the most
 * frequent exponent values").  Reads n elements at d_in (BF16: 2n bytes,
 * E5M2: n bytes), writes the 64-byte plan at d_plan.  n = 0 is valid. */
sz_status sz_plan(sz_dtype dtype, const void *d_in, uint64_t n, void *d_ws, size_t ws_bytes,
                  sz_plan_t *d_plan, cudaStream_t stream);

/* Plans for T tensors in one launch.  d_in and n are HOST arrays of T
 * entries (device pointers / element counts); d_plans points to T
 * consecutive plans in device memory.  Each tensor gets its own codebook. */
sz_status sz_plan_batched(sz_dtype dtype, int T, const void *const *d_in, const uint64_t *n,
                          void *d_ws, size_t ws_bytes, sz_plan_t *d_plans, cudaStream_t stream);

/* Stream length recorded in a plan.  Copies it to *h_bytes and synchronises
 * the stream. */
sz_status sz_compressed_size(const sz_plan_t *d_plan, uint64_t *h_bytes, cudaStream_t stream);

/* Stream lengths of T consecutive plans (one copy, one synchronise). */
sz_status sz_compressed_sizes(int T, const sz_plan_t *d_plans, uint64_t *h_bytes,
                              cudaStream_t stream);

/* Encode: split, code, pack, escape scatter and per-block escape offsets
 * (project page, Abstract).  d_plan must come from sz_plan on the same data.
 * Writes the whole stream (header included) to d_out, which must hold
 * out_cap >= the plan's total_bytes (sz_max_compressed_size always
 * suffices); a smaller capacity is reported as SZ_ERR_BUFFER_TOO_SMALL on
 * the device error word and nothing is written. */
sz_status sz_encode(sz_dtype dtype, const sz_plan_t *d_plan, const void *d_in, uint64_t n,
                    void *d_out, size_t out_cap, void *d_ws, size_t ws_bytes, cudaStream_t stream);

/* Encode T tensors in one launch.  d_in, n, d_out, out_cap are HOST arrays
 * of T entries; d_plans are the T consecutive plans from sz_plan_batched. */
sz_status sz_encode_batched(sz_dtype dtype, int T, const sz_plan_t *d_plans,
                            const void *const *d_in, const uint64_t *n, void *const *d_out,
                            const size_t *out_cap, void *d_ws, size_t ws_bytes,
                            cudaStream_t stream);

/* Set the header flags of T consecutive plans (byte 39; 0 or
 * SZ_FLAG_RAW_BLOCKS), stream-ordered after the sz_plan* call that wrote
 * them (a plan call writes flags 0).  Encoding with a plan, or with it as a
 * reused codebook, then allows raw blocks; the stream records the flag and
 * sz_decode reads it.  With raw blocks the plan's E and total_bytes are upper
 * bounds (a raw block stores fewer bytes than its escapes would): out_cap
 * checks use them, and the stream's own header (bytes 16..23 and 40..47) holds
 * the exact E and length.  SZ_ERR_INVALID_ARG for other flags, T out of
 * range or a null/misaligned pointer. */
sz_status sz_plan_set_flags(int T, sz_plan_t *d_plans, unsigned flags, cudaStream_t stream);

/* Codebook reuse: encode with the codebook of a plan made earlier -- for
 * another layer, or for the same tensor at an earlier step -- without a new
 * histogram pass.  Any codebook keeps the stream lossless: every exponent
 * outside it is escaped (project page, Abstract: rare exponent values go
 * through the sparse escape stream).  The stream is an ordinary format-v1
 * stream that sz_decode reads; its header records the given codebook and the
 * escape count E that codebook leaves for this data.
 *
 * Only the codebook bytes (plan bytes 24..38, 15 distinct values of the
 * dtype's exponent range) and the flags (byte 39, see sz_plan_set_flags) are
 * read from d_codebook; its n, E and total are ignored.  An invalid codebook is reported as
 * SZ_ERR_PLAN_MISMATCH on the device error word and nothing is written.
 *
 * out_cap must hold at least sz_stream_bytes(dtype, n, 0) (checked here).
 * The total is known only when the last block is coded: if the escapes do not
 * fit, SZ_ERR_BUFFER_TOO_SMALL is recorded and the stream is incomplete
 * (sz_max_compressed_size always suffices).  d_total (device, 8-byte aligned,
 * or NULL) receives the stream's length; the header holds it too (bytes
 * 40..47). */
sz_status sz_encode_reuse(sz_dtype dtype, const sz_plan_t *d_codebook, const void *d_in, uint64_t n,
                          void *d_out, size_t out_cap, uint64_t *d_total, void *d_ws, size_t ws_bytes,
                          cudaStream_t stream);

/* Codebook reuse for T tensors in one launch.  d_in, n, d_out, out_cap are
 * HOST arrays of T entries; d_codebooks are T consecutive plans in device
 * memory (tensor t uses the codebook of plan t); d_totals (device, or NULL)
 * receives T stream lengths. */
sz_status sz_encode_reuse_batched(sz_dtype dtype, int T, const sz_plan_t *d_codebooks,
                                  const void *const *d_in, const uint64_t *n, void *const *d_out,
                                  const size_t *out_cap, uint64_t *d_totals, void *d_ws, size_t ws_bytes,
                                  cudaStream_t stream);

/* Paged tensors (see sz_paged_t): the same three steps for tensors held in
 * the pages of a page pool -- the stream of a paged tensor is the stream of
 * its elements taken in order, as if gathered into one contiguous tensor.
 * src / dst are HOST arrays of T descriptors; everything else is as in the
 * contiguous calls.  Decode writes only the bytes of the tensor's elements
 * inside its pages. */
sz_status sz_plan_paged_batched(sz_dtype dtype, int T, const sz_paged_t *src, const uint64_t *n,
                                void *d_ws, size_t ws_bytes, sz_plan_t *d_plans, cudaStream_t stream);
sz_status sz_encode_paged_batched(sz_dtype dtype, int T, const sz_plan_t *d_plans, const sz_paged_t *src,
                                  const uint64_t *n, void *const *d_out, const size_t *out_cap, void *d_ws,
                                  size_t ws_bytes, cudaStream_t stream);
sz_status sz_decode_paged_batched(sz_dtype dtype, int T, const void *const *d_comp, const size_t *comp_bytes,
                                  const sz_paged_t *dst, const uint64_t *n, void *d_ws, size_t ws_bytes,
                                  cudaStream_t stream);

/* Codebook reuse (sz_encode_reuse_batched) for paged inputs. */
sz_status sz_encode_reuse_paged_batched(sz_dtype dtype, int T, const sz_plan_t *d_codebooks,
                                        const sz_paged_t *src, const uint64_t *n, void *const *d_out,
                                        const size_t *out_cap, uint64_t *d_totals, void *d_ws, size_t ws_bytes,
                                        cudaStream_t stream);

/* Let kernels on CUDA device `device` read the memory of device `peer`
 * directly (peer access over NVLink).  After it, sz_decode* on `device` may be
 * given streams that live on `peer`: the decode kernel then pulls each
 * stream's bytes across the link itself, with the same 1-D bulk copies it uses
 * for local streams (each CTA fetches its own tiles), so the transfer overlaps
 * the decoding tile by tile and the stream never lands in `device`'s memory.
 * SZ_OK if access is enabled (or already was; device == peer needs nothing),
 * SZ_ERR_CUDA if the two devices cannot reach each other. */
sz_status sz_enable_peer_access(int device, int peer);

/* Decode a stream of comp_bytes bytes holding n elements of dtype into d_out
 * (BF16: 2n bytes, E5M2: n bytes); the result is bitwise identical to the
 * encoded input (project page, FAQ "Is SplitZip lossy?").  A stream that fails
 * a check is reported as SZ_ERR_CORRUPT_STREAM on the device error word; the
 * affected output is then unspecified. */
sz_status sz_decode(sz_dtype dtype, const void *d_comp, size_t comp_bytes, void *d_out,
                    uint64_t n, void *d_ws, size_t ws_bytes, cudaStream_t stream);

/* Decode T streams in one launch (HOST arrays of T entries). */
sz_status sz_decode_batched(sz_dtype dtype, int T, const void *const *d_comp,
                            const size_t *comp_bytes, void *const *d_out, const uint64_t *n,
                            void *d_ws, size_t ws_bytes, cudaStream_t stream);

/* Synchronise the stream, return the device error word of d_ws and clear it. */
sz_status sz_last_device_status(void *d_ws, cudaStream_t stream);

/* Largest n accepted by sz_encode_noalloc (2^27 elements: 32768 tiles). */
#define SZ_NOALLOC_MAX_ELEMS (1ull << 27)

/* Encode without a caller-provided workspace.  The paper has no counterpart:
 * this is a convenience of this library.
 *
 * For callers that cannot allocate device memory where they encode -- for
 * example an engine that reserves all of the GPU's memory for its KV pool at
 * start-up and hands the codec only the tensor, the destination buffer and a
 * stream.  The call runs the same kernel as sz_encode on a scratch area held
 * by the library: a static device array of 271,888 bytes (the workspace of
 * one tensor of SZ_NOALLOC_MAX_ELEMS elements) that every GPU which loads the
 * library keeps until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine; it enqueues a memset of the scratch it uses, the encode
 * kernel and, if d_status is not NULL, a 4-byte device-to-device copy.
 *
 * Arguments are those of sz_encode; d_status (device, 4-byte aligned, may be
 * NULL) receives the call's device error word (SZ_OK or a device-found error)
 * once the stream reaches it.  n > SZ_NOALLOC_MAX_ELEMS returns
 * SZ_ERR_BUFFER_TOO_SMALL, and every other host check of sz_encode its
 * status, at once and with nothing enqueued.  The scratch used is the current
 * device's: a stream that belongs to another device is refused
 * (SZ_ERR_INVALID_ARG).
 *
 * The first call on each device looks up the scratch array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  Every call on a device shares the one scratch
 * array, which keeps the previous call's contents (the call clears what must
 * start at zero): calls whose work overlaps on the GPU -- on different
 * streams, or from different threads -- race and must not be issued. */
sz_status sz_encode_noalloc(sz_dtype dtype, const sz_plan_t *d_plan, const void *d_in, uint64_t n,
                            void *d_out, size_t out_cap, uint32_t *d_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SPLITZIP_H */
