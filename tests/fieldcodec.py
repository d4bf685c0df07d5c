"""Independent reader and checker of stream format v1, for pinning the oracle.

Written from the format's definition with `struct` and numpy bit operations;
it calls neither the oracle nor the CUDA library.  The codebook check uses a
library sort (numpy lexsort) instead of the oracle's rank counting.

Format v1 (little-endian):
  [0,64)  u32 magic 0x564B5A53, u16 version 1, u8 dtype (0 BF16, 1 E5M2),
          u8 block_log2 12, u64 n, u64 E, u8 cb[15], u8 flags, u64 total, 16 zero bytes
  [64, 64 + 4(nb+1))  u32 offsets[nb+1]: escapes before each 4096-element block
  sections at successive multiples of 256:
    BF16: sm plane (n B), code plane (ceil(n/2) B), escapes (E B)
    E5M2: sign plane (ceil(n/8) B), mantissa plane (ceil(n/4) B), code plane, escapes
Header byte 39 holds flags; bit 0 allows raw blocks: a block of m elements whose
escapes would fill at least K = ceil(m/2) (BF16) or ceil(m/8) (E5M2) bytes keeps
the low four exponent bits in its code nibbles and the rest in K escape-section
bytes (BF16: high nibbles, element j of the block in nibble j%2 of byte j/2;
E5M2: bit 4 at bit j%8 of byte j/8); the offsets table counts K for it.
"""
import struct

import numpy as np

MAGIC = 0x564B5A53
HEADER = struct.Struct("<IHBBQQ15sBQ16s")
assert HEADER.size == 64
BLOCK = 4096


def align256(x: int) -> int:
    return -(-x // 256) * 256


def layout(dtype: int, n: int, E: int):
    """(nb, plane starts, plane lengths, escape start, total)."""
    nb = -(-n // BLOCK)
    pos = align256(64 + 4 * (nb + 1))
    if dtype == 0:
        lens = [n, -(-n // 2)]
    else:
        lens = [-(-n // 8), -(-n // 4), -(-n // 2)]
    starts = []
    for ln in lens:
        starts.append(pos)
        pos = align256(pos + ln)
    return nb, starts, lens, pos, pos + E


def parse(stream) -> dict:
    s = np.asarray(stream, dtype=np.uint8)
    magic, ver, dtype, blog, n, E, cb, flags, total, tail = HEADER.unpack(s[:64].tobytes())
    nb, starts, lens, esc, tot = layout(dtype, n, E)
    offs = np.frombuffer(s[64:64 + 4 * (nb + 1)].tobytes(), dtype="<u4").astype(np.int64)
    return dict(magic=magic, version=ver, dtype=dtype, block_log2=blog, n=n, E=E,
                cb=np.frombuffer(cb, dtype=np.uint8).copy(), flags=flags, total=total, tail=tail,
                nb=nb, starts=starts, lens=lens, esc=esc, closed_total=tot, offsets=offs)


def _codes(s, f):
    n = f["n"]
    plane = s[f["starts"][-1]: f["starts"][-1] + f["lens"][-1]].astype(np.uint8)
    nib = np.empty(2 * plane.size, dtype=np.uint8)
    nib[0::2] = plane & 0xF
    nib[1::2] = plane >> 4
    return nib[:n]


def raw_block_bytes(dtype: int, m: int) -> int:
    """Escape-section bytes of a raw block of m elements."""
    return -(-m // 2) if dtype == 0 else -(-m // 8)


def block_sizes(n: int):
    return [min(BLOCK, n - b) for b in range(0, n, BLOCK)]


def _high_bits(packed: np.ndarray, dtype: int, m: int) -> np.ndarray:
    """The m high-exponent parts of a raw block from its escape-section bytes."""
    if dtype == 0:
        nib = np.empty(2 * packed.size, dtype=np.uint32)
        nib[0::2] = packed & 0xF
        nib[1::2] = packed >> 4
        return nib[:m]
    return np.unpackbits(packed, bitorder="little")[:m].astype(np.uint32)


def decode(stream) -> np.ndarray:
    """Decode to raw element bytes (little-endian) using only numpy."""
    s = np.asarray(stream, dtype=np.uint8)
    f = parse(s)
    n, dtype = f["n"], f["dtype"]
    codes = _codes(s, f)
    e = np.zeros(n, dtype=np.uint32)
    offs = f["offsets"]
    for b, m in enumerate(block_sizes(n)):
        lo, hi = b * BLOCK, b * BLOCK + m
        c = codes[lo:hi]
        cnt = int(offs[b + 1] - offs[b])
        seg = s[f["esc"] + int(offs[b]): f["esc"] + int(offs[b + 1])]
        if (f["flags"] & 1) and cnt == raw_block_bytes(dtype, m):
            e[lo:hi] = (_high_bits(seg, dtype, m) << 4) | c
        else:
            esc = c == 15
            e[lo:hi][~esc] = f["cb"][c[~esc]]
            e[lo:hi][esc] = seg
    if dtype == 0:
        sm = s[f["starts"][0]: f["starts"][0] + n].astype(np.uint32)
        bits = ((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)
        return bits.astype("<u2").view(np.uint8)
    sign = np.unpackbits(s[f["starts"][0]: f["starts"][0] + f["lens"][0]], bitorder="little")[:n]
    mplane = s[f["starts"][1]: f["starts"][1] + f["lens"][1]]
    idx = np.arange(n)
    mant = (mplane[idx // 4] >> (2 * (idx % 4))) & 3
    bits = (sign.astype(np.uint32) << 7) | (e << 2) | mant.astype(np.uint32)
    return bits.astype(np.uint8)


def exponents(raw: np.ndarray, dtype: int) -> np.ndarray:
    raw = np.asarray(raw, dtype=np.uint8).reshape(-1)
    if dtype == 0:
        w = raw.view("<u2").astype(np.uint32)
        return (w >> 7) & 0xFF
    return (raw.astype(np.uint32) >> 2) & 0x1F


def expected_codebook(raw: np.ndarray, dtype: int) -> np.ndarray:
    """Top 15 exponent values by (count desc, value asc), via np.bincount + np.lexsort."""
    nv = 256 if dtype == 0 else 32
    cnt = np.bincount(exponents(raw, dtype), minlength=nv)
    vals = np.arange(nv)
    order = np.lexsort((vals, -cnt.astype(np.int64)))  # primary: -count, secondary: value
    return order[:15].astype(np.uint8)


def check(stream, raw, dtype: int, codebook=None, raw_blocks=False) -> None:
    """Assert that `stream` is exactly the v1 encoding of `raw` (raises AssertionError):
    with the tensor's own top-15 codebook, or with `codebook` when one is given;
    with raw blocks allowed when `raw_blocks`."""
    s = np.asarray(stream, dtype=np.uint8)
    raw = np.asarray(raw, dtype=np.uint8).reshape(-1)
    n = raw.size // (2 if dtype == 0 else 1)
    f = parse(s)
    assert f["magic"] == MAGIC, hex(f["magic"])
    assert f["version"] == 1 and f["dtype"] == dtype and f["block_log2"] == 12
    assert f["n"] == n
    assert f["flags"] == (1 if raw_blocks else 0) and f["tail"] == bytes(16)
    cb = expected_codebook(raw, dtype) if codebook is None else np.asarray(codebook, dtype=np.uint8)
    assert np.array_equal(f["cb"], cb), (f["cb"], cb)
    e = exponents(raw, dtype)
    lut = np.full(256, 15, dtype=np.uint8)
    lut[cb] = np.arange(15, dtype=np.uint8)
    codes = lut[e]
    # per block: coded (its escapes' exponents, in element order) or raw (the
    # low exponent nibbles as codes, the high bits packed in the escape section)
    segs, counts = [], []
    for b, m in enumerate(block_sizes(n)):
        lo, hi = b * BLOCK, b * BLOCK + m
        esc = codes[lo:hi] == 15
        K = raw_block_bytes(dtype, m)
        if raw_blocks and int(esc.sum()) >= K:
            codes[lo:hi] = e[lo:hi] & 0xF
            high = (e[lo:hi] >> 4).astype(np.uint8)
            if dtype == 0:
                h2 = np.concatenate([high, np.zeros(m % 2, np.uint8)]).reshape(-1, 2)
                seg = (h2[:, 0] | (h2[:, 1] << 4)).astype(np.uint8)
            else:
                seg = np.packbits(high, bitorder="little")
            assert seg.size == K
        else:
            seg = e[lo:hi][esc].astype(np.uint8)
        segs.append(seg)
        counts.append(seg.size)
    E = int(sum(counts))
    assert f["E"] == E
    assert f["total"] == f["closed_total"] == s.size
    # code plane
    assert np.array_equal(_codes(s, f), codes)
    # escape section: the blocks' segments in block order
    expect_esc = np.concatenate(segs) if segs else np.zeros(0, np.uint8)
    assert np.array_equal(s[f["esc"]: f["esc"] + E], expect_esc)
    # offsets: exclusive prefix of the per-block counts; offsets[nb] = E
    nb = f["nb"]
    expect_offs = np.concatenate([[0], np.cumsum(np.array(counts, dtype=np.int64))])
    assert np.array_equal(f["offsets"], expect_offs), (f["offsets"][:8], expect_offs[:8])
    # exact planes
    if dtype == 0:
        w = raw.view("<u2").astype(np.uint32)
        sm = (((w >> 15) & 1) << 7) | (w & 0x7F)
        assert np.array_equal(s[f["starts"][0]: f["starts"][0] + n], sm.astype(np.uint8))
    else:
        b = raw.astype(np.uint32)
        sign = (b >> 7) & 1
        packed = np.packbits(sign.astype(np.uint8), bitorder="little")
        assert np.array_equal(s[f["starts"][0]: f["starts"][0] + f["lens"][0]], packed)
        mant = b & 3
        pad = (-n) % 4
        m4 = np.concatenate([mant, np.zeros(pad, np.uint32)]).reshape(-1, 4)
        mp = (m4[:, 0] | (m4[:, 1] << 2) | (m4[:, 2] << 4) | (m4[:, 3] << 6)).astype(np.uint8)
        assert np.array_equal(s[f["starts"][1]: f["starts"][1] + f["lens"][1]], mp)
    # every byte outside header, table, planes and escapes is zero
    used = np.zeros(s.size, dtype=bool)
    used[:64 + 4 * (nb + 1)] = True
    for st, ln in zip(f["starts"], f["lens"]):
        used[st: st + ln] = True
    used[f["esc"]: f["esc"] + E] = True
    assert not s[~used].any(), "non-zero padding"
    # round trip through this reader
    assert np.array_equal(decode(s), raw)
