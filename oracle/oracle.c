/*
 * oracle.c -- plain, slow, single-threaded CPU reference of the exponent-split
 * KV codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library and its Python binding) never calls it, links it or shares a
 * line of code with it.
 *
 * What is computed follows "SplitZip: Ultra-Fast Lossless KV Compression for
 * Disaggregated LLM Serving" (project page):
 *   - Abstract: BF16 KV exponents are highly redundant; the most frequent
 *     exponent values get fixed 4-bit codes, sign and mantissa bits are kept
 *     exactly, and rare exponent values go through a sparse escape stream.
 *   - FAQ "Is SplitZip lossy?": decoding is bitwise identical to the input.
 *   - FAQ "Does it work with an FP8 KV cache?": the same coding applies to
 *     FP8 E5M2 data.
 * The page prints no byte layout.  Everything about bytes below (header,
 * block size 4096, codebook of 15 with code 15 as escape, ties to the smaller
 * exponent, stored per-block escape offsets, 256-byte section alignment) is
 * this library's stream format v1, restated here independently of the CUDA
 * code:
 *
 *   [0,64)  header: u32 magic 0x564B5A53, u16 version 1, u8 dtype (0 BF16,
 *           1 E5M2), u8 block_log2 = 12, u64 n, u64 E, u8 cb[15], u8 0,
 *           u64 total_bytes, 16 zero bytes                 (little-endian)
 *   [64, 64+4(nb+1))  u32 offsets[nb+1], nb = ceil(n/4096):
 *           offsets[b] = escapes in blocks before b, offsets[nb] = E
 *   then sections, each starting at the next multiple of 256:
 *     BF16: sm plane (n bytes, sm = sign<<7 | mantissa7),
 *           code plane (ceil(n/2) bytes, even element in the low nibble),
 *           escapes (E bytes, the exponent of each escaped element, in
 *           element order)
 *     E5M2: sign plane (ceil(n/8) bytes, element i at bit i%8 of byte i/8),
 *           mantissa plane (ceil(n/4) bytes, element i at bits 2(i%4)..+1 of
 *           byte i/4), code plane, escapes
 *   All padding bytes and unused high bits are zero.
 *
 * Header byte 39 holds flags; bit 0 allows raw blocks.  Without it every
 * block is coded as above.  With it, a block of m elements whose escapes
 * would fill at least K = ceil(m/2) bytes (BF16) or ceil(m/8) bytes (E5M2) --
 * the size of its exponent bits above the low four -- is stored raw: its code
 * nibbles hold the low four bits of each exponent and its K escape-section
 * bytes the remaining bits (BF16: the high nibble of element j's exponent in
 * nibble j%2 of byte j/2; E5M2: bit 4 of element j's exponent at bit j%8 of
 * byte j/8; j counted within the block).  The offsets table counts K bytes
 * for such a block, and a coded block always has fewer than K escapes, so a
 * decoder tells the two apart by the count.  E in the header is the length
 * of the escape section.  A raw block costs exactly its raw bytes, so no
 * block expands.  The pages describe no such fallback; it is this format's
 * own extension for data whose exponents the codebook does not capture.
 *
 * Every loop below walks the elements one at a time, in order.  No blocking,
 * no vector tricks: a reader can check each step against the description.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define ORC_BF16 0
#define ORC_E5M2 1

enum {
    ORC_OK = 0,
    ORC_ERR_ARG = 1,      /* bad argument (null pointer, n too large)          */
    ORC_ERR_DTYPE = 2,    /* unknown element type                              */
    ORC_ERR_SMALL = 3,    /* output buffer smaller than the stream             */
    ORC_ERR_CORRUPT = 4   /* stream fails a consistency check                  */
};

#define ORC_MAGIC 0x564B5A53u
#define ORC_VERSION 1u
#define ORC_BLOCK_LOG2 12u
#define ORC_BLOCK 4096u
#define ORC_CODES 15u          /* codes 0..14 name codebook entries          */
#define ORC_ESCAPE 15u         /* code 15 marks an escaped exponent          */
#define ORC_FLAG_RAW_BLOCKS 1u /* header byte 39, bit 0: raw blocks allowed  */

/* ---------------------------------------------------------------- helpers */

static uint64_t align256(uint64_t x) { return (x + 255u) / 256u * 256u; }
static uint64_t ceil_div(uint64_t a, uint64_t b) { return (a + b - 1u) / b; }

/* Number of distinct exponent values: 8-bit exponent for BF16, 5-bit for E5M2. */
static unsigned exponent_values(int dtype) { return dtype == ORC_BF16 ? 256u : 32u; }

/* Raw bits of element i.  BF16 elements are little-endian 16-bit words. */
static unsigned element_bits(int dtype, const uint8_t *in, uint64_t i)
{
    if (dtype == ORC_BF16)
        return (unsigned)in[2 * i] | ((unsigned)in[2 * i + 1] << 8);
    return in[i];
}

/* Field split.  BF16 = s eeeeeeee mmmmmmm ; E5M2 = s eeeee mm. */
static unsigned sign_of(int dtype, unsigned bits)
{
    return dtype == ORC_BF16 ? (bits >> 15) & 1u : (bits >> 7) & 1u;
}
static unsigned exponent_of(int dtype, unsigned bits)
{
    return dtype == ORC_BF16 ? (bits >> 7) & 0xFFu : (bits >> 2) & 0x1Fu;
}
static unsigned mantissa_of(int dtype, unsigned bits)
{
    return dtype == ORC_BF16 ? bits & 0x7Fu : bits & 0x3u;
}
static unsigned assemble(int dtype, unsigned s, unsigned e, unsigned m)
{
    if (dtype == ORC_BF16)
        return (s << 15) | (e << 7) | m;
    return (s << 7) | (e << 2) | m;
}

static void put_u16(uint8_t *p, unsigned v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put_u32(uint8_t *p, uint32_t v)
{
    for (int k = 0; k < 4; k++) p[k] = (uint8_t)(v >> (8 * k));
}
static void put_u64(uint8_t *p, uint64_t v)
{
    for (int k = 0; k < 8; k++) p[k] = (uint8_t)(v >> (8 * k));
}
static unsigned get_u16(const uint8_t *p) { return (unsigned)p[0] | ((unsigned)p[1] << 8); }
static uint32_t get_u32(const uint8_t *p)
{
    uint32_t v = 0;
    for (int k = 0; k < 4; k++) v |= (uint32_t)p[k] << (8 * k);
    return v;
}
static uint64_t get_u64(const uint8_t *p)
{
    uint64_t v = 0;
    for (int k = 0; k < 8; k++) v |= (uint64_t)p[k] << (8 * k);
    return v;
}

/* Section start offsets of a stream with n elements and E escapes.
 * sec[0..nsec-1] are the planes in stream order, then the escape section. */
typedef struct {
    uint64_t nb;        /* number of 4096-element blocks                   */
    int nsec;           /* planes: 2 for BF16, 3 for E5M2                  */
    uint64_t sec[3];    /* plane start offsets                             */
    uint64_t len[3];    /* plane lengths in bytes                          */
    uint64_t esc;       /* escape section start                            */
    uint64_t total;     /* stream length in bytes                          */
} orc_layout;

static orc_layout layout_of(int dtype, uint64_t n, uint64_t E)
{
    orc_layout L;
    memset(&L, 0, sizeof L);
    L.nb = ceil_div(n, ORC_BLOCK);
    uint64_t pos = align256(64u + 4u * (L.nb + 1u));
    if (dtype == ORC_BF16) {
        L.nsec = 2;
        L.len[0] = n;                 /* sign|mantissa byte per element */
        L.len[1] = ceil_div(n, 2);    /* one nibble per element         */
    } else {
        L.nsec = 3;
        L.len[0] = ceil_div(n, 8);    /* one sign bit per element       */
        L.len[1] = ceil_div(n, 4);    /* two mantissa bits per element  */
        L.len[2] = ceil_div(n, 2);    /* one nibble per element         */
    }
    for (int s = 0; s < L.nsec; s++) {
        L.sec[s] = pos;
        pos = align256(pos + L.len[s]);
    }
    L.esc = pos;
    L.total = pos + E;
    return L;
}

/* ------------------------------------------------------------ public API */

/* Stream length for n elements with E escapes (format v1 closed form).
 * Returns 0 for an unknown dtype. */
uint64_t orc_compressed_size(int dtype, uint64_t n, uint64_t E)
{
    if (dtype != ORC_BF16 && dtype != ORC_E5M2) return 0;
    return layout_of(dtype, n, E).total;
}

/* Exponent histogram ("the most frequent exponent values", Abstract).
 * hist must hold 256 entries; entries beyond the dtype's range are zeroed. */
int orc_histogram(int dtype, const uint8_t *in, uint64_t n, uint64_t *hist)
{
    if (dtype != ORC_BF16 && dtype != ORC_E5M2) return ORC_ERR_DTYPE;
    if (!hist || (n && !in)) return ORC_ERR_ARG;
    for (unsigned v = 0; v < 256u; v++) hist[v] = 0;
    for (uint64_t i = 0; i < n; i++)
        hist[exponent_of(dtype, element_bits(dtype, in, i))] += 1;
    return ORC_OK;
}

/* Codebook: the 15 most frequent exponent values (Abstract).  Every value is
 * ranked by (count descending, value ascending); the value of rank c gets
 * code c.  Values that never occur still take part, so a tensor with fewer
 * than 15 distinct exponents fills the codebook with the smallest unused
 * values. */
int orc_codebook(int dtype, const uint64_t *hist, uint8_t *cb)
{
    if (dtype != ORC_BF16 && dtype != ORC_E5M2) return ORC_ERR_DTYPE;
    if (!hist || !cb) return ORC_ERR_ARG;
    unsigned nv = exponent_values(dtype);
    for (unsigned v = 0; v < nv; v++) {
        unsigned rank = 0;
        for (unsigned u = 0; u < nv; u++) {
            if (hist[u] > hist[v] || (hist[u] == hist[v] && u < v)) rank++;
        }
        if (rank < ORC_CODES) cb[rank] = (uint8_t)v;
    }
    return ORC_OK;
}

/* Code of exponent e under codebook cb: its codebook index, or the escape. */
static unsigned code_of(const uint8_t *cb, unsigned e)
{
    for (unsigned c = 0; c < ORC_CODES; c++)
        if (cb[c] == e) return c;
    return ORC_ESCAPE;
}

/* Elements of block b of a tensor of n elements. */
static uint64_t block_elems(uint64_t n, uint64_t b)
{
    uint64_t first = b * ORC_BLOCK;
    return n - first < ORC_BLOCK ? n - first : ORC_BLOCK;
}

/* Escape-section bytes of a raw block of m elements: its exponent bits above
 * the low four (four per BF16 element, one per E5M2 element). */
static uint64_t raw_block_bytes(int dtype, uint64_t m)
{
    return dtype == ORC_BF16 ? ceil_div(m, 2) : ceil_div(m, 8);
}

/* Whether block b is stored raw: raw blocks are allowed and the block's
 * escapes under cb would fill at least raw_block_bytes. */
static int block_is_raw(int dtype, const uint8_t *in, uint64_t n, const uint8_t *cb, unsigned flags,
                        uint64_t b)
{
    if (!(flags & ORC_FLAG_RAW_BLOCKS)) return 0;
    uint64_t m = block_elems(n, b), escapes = 0;
    for (uint64_t i = b * ORC_BLOCK; i < b * ORC_BLOCK + m; i++)
        if (code_of(cb, exponent_of(dtype, element_bits(dtype, in, i))) == ORC_ESCAPE) escapes++;
    return escapes >= raw_block_bytes(dtype, m);
}

/* Encode n elements into out (capacity cap bytes).  cb_given: a codebook of
 * 15 exponent values chosen by the caller, or NULL for the tensor's own (its
 * 15 most frequent exponent values, Abstract).  Any 15 distinct exponent
 * values of the dtype's range form a valid codebook, and the result is still
 * lossless: exponents outside it take the escape path (SplitZip project page,
 * Abstract: rare exponent values go through the sparse escape stream).  This
 * is what lets a codebook found once be reused for other layers or later
 * steps without a new histogram pass (the related-work list of the ZipServ
 * page names exponent reuse across iterations: "CIERA: Cross-Iteration
 * Exponent Reuse for Lossless Allgather in Sharded MoE Training").
 * flags: 0, or ORC_FLAG_RAW_BLOCKS to let blocks that would expand be stored
 * raw (see the format above).
 * Returns the stream length, or minus an ORC_ERR_* code. */
int64_t orc_encode_ex(int dtype, const uint8_t *in, uint64_t n, const uint8_t *cb_given, unsigned flags,
                      uint8_t *out, uint64_t cap)
{
    if (dtype != ORC_BF16 && dtype != ORC_E5M2) return -ORC_ERR_DTYPE;
    if ((n && !in) || !out || n >= (1ull << 32)) return -ORC_ERR_ARG;
    if (flags & ~ORC_FLAG_RAW_BLOCKS) return -ORC_ERR_ARG;
    uint8_t own[ORC_CODES];
    const uint8_t *cb = cb_given;
    if (cb) {
        for (unsigned c = 0; c < ORC_CODES; c++) {
            if (cb[c] >= exponent_values(dtype)) return -ORC_ERR_ARG;
            for (unsigned d = 0; d < c; d++)
                if (cb[d] == cb[c]) return -ORC_ERR_ARG;
        }
    } else {
        uint64_t hist[256];
        orc_histogram(dtype, in, n, hist);
        orc_codebook(dtype, hist, own);
        cb = own;
    }

    /* 1. escape count: every element whose exponent is not in the codebook
     *    (a raw block instead counts its raw_block_bytes) */
    uint64_t E = 0;
    uint64_t nb = ceil_div(n, ORC_BLOCK);
    for (uint64_t b = 0; b < nb; b++) {
        if (block_is_raw(dtype, in, n, cb, flags, b)) {
            E += raw_block_bytes(dtype, block_elems(n, b));
            continue;
        }
        for (uint64_t i = b * ORC_BLOCK; i < b * ORC_BLOCK + block_elems(n, b); i++)
            if (code_of(cb, exponent_of(dtype, element_bits(dtype, in, i))) == ORC_ESCAPE) E++;
    }

    orc_layout L = layout_of(dtype, n, E);
    if (cap < L.total) return -ORC_ERR_SMALL;
    memset(out, 0, L.total);

    /* 2. header */
    put_u32(out + 0, ORC_MAGIC);
    put_u16(out + 4, ORC_VERSION);
    out[6] = (uint8_t)dtype;
    out[7] = (uint8_t)ORC_BLOCK_LOG2;
    put_u64(out + 8, n);
    put_u64(out + 16, E);
    for (unsigned c = 0; c < ORC_CODES; c++) out[24 + c] = cb[c];
    out[39] = (uint8_t)flags;
    put_u64(out + 40, L.total);

    /* 3. one pass in element order: planes, codes, escapes, and the escape
     *    count before each block (the exclusive prefix over blocks). */
    uint64_t k = 0;      /* escape-section bytes emitted so far */
    int raw = 0;         /* the current block is stored raw      */
    uint64_t k_raw = 0;  /* where a raw block's high bits start  */
    for (uint64_t i = 0; i < n; i++) {
        if (i % ORC_BLOCK == 0) put_u32(out + 64 + 4 * (i / ORC_BLOCK), (uint32_t)k);
        if (i % ORC_BLOCK == 0) {
            raw = block_is_raw(dtype, in, n, cb, flags, i / ORC_BLOCK);
            k_raw = k;
            if (raw) k += raw_block_bytes(dtype, block_elems(n, i / ORC_BLOCK));
        }
        unsigned bits = element_bits(dtype, in, i);
        unsigned s = sign_of(dtype, bits), e = exponent_of(dtype, bits), m = mantissa_of(dtype, bits);
        unsigned c = raw ? (e & 0xFu) : code_of(cb, e);
        if (dtype == ORC_BF16) {
            out[L.sec[0] + i] = (uint8_t)((s << 7) | m);
        } else {
            out[L.sec[0] + i / 8] |= (uint8_t)(s << (i % 8));
            out[L.sec[1] + i / 4] |= (uint8_t)(m << (2 * (i % 4)));
        }
        uint64_t code_plane = L.sec[L.nsec - 1];
        out[code_plane + i / 2] |= (uint8_t)(c << (4 * (i % 2)));
        if (raw) {
            uint64_t j = i % ORC_BLOCK;  /* position within the block */
            if (dtype == ORC_BF16)
                out[L.esc + k_raw + j / 2] |= (uint8_t)((e >> 4) << (4 * (j % 2)));
            else
                out[L.esc + k_raw + j / 8] |= (uint8_t)((e >> 4) << (j % 8));
        } else if (c == ORC_ESCAPE) {
            out[L.esc + k] = (uint8_t)e;
            k++;
        }
    }
    put_u32(out + 64 + 4 * L.nb, (uint32_t)k);  /* offsets[nb] = E */
    return (int64_t)L.total;
}

/* Encode with a codebook given by the caller (codebook reuse), no raw blocks.
 * Returns the stream length, or minus an ORC_ERR_* code. */
int64_t orc_encode_codebook(int dtype, const uint8_t *in, uint64_t n, const uint8_t *cb,
                            uint8_t *out, uint64_t cap)
{
    if (!cb) return -ORC_ERR_ARG;
    return orc_encode_ex(dtype, in, n, cb, 0u, out, cap);
}

/* Encode n elements into out (capacity cap bytes) with the tensor's own
 * codebook: its 15 most frequent exponent values (Abstract), no raw blocks.
 * Returns the stream length, or minus an ORC_ERR_* code. */
int64_t orc_encode(int dtype, const uint8_t *in, uint64_t n, uint8_t *out, uint64_t cap)
{
    return orc_encode_ex(dtype, in, n, NULL, 0u, out, cap);
}

/* Read and check a stream header.  On success fills dtype, n, E, cb and the
 * layout.  Checks are the ones a decoder needs to stay inside the buffer and
 * to reject streams this format cannot produce. */
static int parse_header(const uint8_t *comp, uint64_t comp_bytes, int *dtype, uint64_t *n,
                        uint64_t *E, uint8_t *cb, unsigned *flags, orc_layout *L)
{
    if (!comp || comp_bytes < 64) return ORC_ERR_CORRUPT;
    if (get_u32(comp) != ORC_MAGIC) return ORC_ERR_CORRUPT;
    if (get_u16(comp + 4) != ORC_VERSION) return ORC_ERR_CORRUPT;
    if (comp[6] != ORC_BF16 && comp[6] != ORC_E5M2) return ORC_ERR_DTYPE;
    if (comp[7] != ORC_BLOCK_LOG2) return ORC_ERR_CORRUPT;
    *dtype = comp[6];
    *n = get_u64(comp + 8);
    *E = get_u64(comp + 16);
    if (*n >= (1ull << 32) || *E > *n) return ORC_ERR_CORRUPT;
    unsigned nv = exponent_values(*dtype);
    for (unsigned c = 0; c < ORC_CODES; c++) {
        cb[c] = comp[24 + c];
        if (cb[c] >= nv) return ORC_ERR_CORRUPT;
        for (unsigned d = 0; d < c; d++)
            if (cb[d] == cb[c]) return ORC_ERR_CORRUPT;
    }
    *flags = comp[39];
    if (*flags & ~ORC_FLAG_RAW_BLOCKS) return ORC_ERR_CORRUPT;
    *L = layout_of(*dtype, *n, *E);
    if (get_u64(comp + 40) != L->total) return ORC_ERR_CORRUPT;
    if (comp_bytes < L->total) return ORC_ERR_CORRUPT;
    return ORC_OK;
}

/* Decode a stream of n elements into out (n * element size bytes).
 * Returns ORC_OK or an ORC_ERR_* code; on error out may be partly written. */
int orc_decode(const uint8_t *comp, uint64_t comp_bytes, uint8_t *out, uint64_t n)
{
    int dtype;
    uint64_t sn, E;
    uint8_t cb[ORC_CODES];
    unsigned flags;
    orc_layout L;
    int rc = parse_header(comp, comp_bytes, &dtype, &sn, &E, cb, &flags, &L);
    if (rc) return rc;
    if (sn != n) return ORC_ERR_ARG;
    if (n && !out) return ORC_ERR_ARG;

    uint64_t k = 0;      /* escape-section bytes consumed so far */
    int raw = 0;         /* the current block is stored raw       */
    uint64_t k_raw = 0;  /* where a raw block's high bits start   */
    for (uint64_t i = 0; i < n; i++) {
        if (i % ORC_BLOCK == 0 && get_u32(comp + 64 + 4 * (i / ORC_BLOCK)) != k)
            return ORC_ERR_CORRUPT;  /* stored block offset disagrees */
        if (i % ORC_BLOCK == 0) {
            /* a block is raw exactly when its count is raw_block_bytes: a
             * coded block has fewer escapes than that */
            uint64_t next = get_u32(comp + 64 + 4 * (i / ORC_BLOCK + 1));
            uint64_t K = raw_block_bytes(dtype, block_elems(n, i / ORC_BLOCK));
            raw = (flags & ORC_FLAG_RAW_BLOCKS) && next >= k && next - k == K;
            k_raw = k;
            if (raw) {
                if (next > E) return ORC_ERR_CORRUPT;
                k = next;
            }
        }
        uint64_t code_plane = L.sec[L.nsec - 1];
        unsigned c = (comp[code_plane + i / 2] >> (4 * (i % 2))) & 0xFu;
        unsigned e;
        if (raw) {
            uint64_t j = i % ORC_BLOCK;  /* position within the block */
            unsigned high = dtype == ORC_BF16 ? (comp[L.esc + k_raw + j / 2] >> (4 * (j % 2))) & 0xFu
                                              : (comp[L.esc + k_raw + j / 8] >> (j % 8)) & 1u;
            e = (high << 4) | c;
        } else if (c < ORC_CODES) {
            e = cb[c];
        } else {
            if (k >= E) return ORC_ERR_CORRUPT;  /* more escapes than the header says */
            e = comp[L.esc + k];
            if (e >= exponent_values(dtype)) return ORC_ERR_CORRUPT;
            k++;
        }
        unsigned s, m;
        if (dtype == ORC_BF16) {
            unsigned sm = comp[L.sec[0] + i];
            s = sm >> 7;
            m = sm & 0x7Fu;
        } else {
            s = (comp[L.sec[0] + i / 8] >> (i % 8)) & 1u;
            m = (comp[L.sec[1] + i / 4] >> (2 * (i % 4))) & 3u;
        }
        unsigned bits = assemble(dtype, s, e, m);
        if (dtype == ORC_BF16) {
            out[2 * i] = (uint8_t)bits;
            out[2 * i + 1] = (uint8_t)(bits >> 8);
        } else {
            out[i] = (uint8_t)bits;
        }
    }
    if (k != E) return ORC_ERR_CORRUPT;
    if (get_u32(comp + 64 + 4 * L.nb) != E) return ORC_ERR_CORRUPT;
    return ORC_OK;
}
