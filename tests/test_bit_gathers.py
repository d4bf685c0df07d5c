"""The multiply gathers and spreads of the E5M2 kernels, checked exhaustively on the host.

The E5M2 encode moves sign and mantissa bits between an element's byte and the
packed sign (1 bit per element) and mantissa (2 bits per element) planes with
integer multiplies, and the decode moves them back the same way.  Each trick
relies on no two partial products of the multiply sharing a bit that is kept
(no carries into the kept bits).  These tests restate the constants and masks
the kernels use and compare each trick with the plain bit-by-bit definition
over every input that reaches the multiply (the masks clear all other bits).
"""
import numpy as np


def _mul32(a, b):
    return (np.asarray(a, dtype=np.uint64) * np.uint64(b)) & np.uint64(0xFFFFFFFF)


def _byte_perm(a, b, sel):
    """__byte_perm(a, b, sel) for selectors whose nibbles are all below 8."""
    pair = [(int(a) >> (8 * i)) & 0xFF for i in range(4)] + [(int(b) >> (8 * i)) & 0xFF for i in range(4)]
    return sum(pair[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def _word(bits_per_byte, shift):
    """32-bit words whose byte i holds field value v_i at `shift`, for every
    combination of the four fields (bits_per_byte wide each)."""
    n = 1 << bits_per_byte
    vals = np.arange(n ** 4, dtype=np.uint64)
    fields = [(vals >> np.uint64(bits_per_byte * i)) & np.uint64(n - 1) for i in range(4)]
    w = sum(f << np.uint64(8 * i + shift) for i, f in enumerate(fields))
    return w, fields


def test_encode_sign_pair_gather():
    # signs of elements 0-3 (word w0) and 4-7 (word w1): bit 7 of each byte
    signs = np.arange(256, dtype=np.uint64)
    w0 = sum(((signs >> np.uint64(b)) & np.uint64(1)) << np.uint64(8 * b + 7) for b in range(4))
    w1 = sum(((signs >> np.uint64(4 + b)) & np.uint64(1)) << np.uint64(8 * b + 7) for b in range(4))
    m = np.uint64(0x80808080)
    x = ((w0 & m) >> np.uint64(4)) | (w1 & m)
    top = (_mul32(x, 0x00204081) >> np.uint64(24)) & np.uint64(0xFF)
    assert np.array_equal(top, signs)


def test_encode_mantissa_gather():
    w, fields = _word(2, 0)
    top = (_mul32(w & np.uint64(0x03030303), 0x01041040) >> np.uint64(24)) & np.uint64(0xFF)
    expect = sum(f << np.uint64(2 * i) for i, f in enumerate(fields))
    assert np.array_equal(top, expect)


def test_encode_plane_byte_permutes():
    rng = np.random.default_rng(7)
    for _ in range(200):
        p = [int(v) for v in rng.integers(0, 2 ** 32, size=4, dtype=np.uint64)]
        sign = _byte_perm(p[0], p[1], 0x0073) & 0xFFFF
        assert sign == (p[0] >> 24) | ((p[1] >> 24) << 8)
        mant = _byte_perm(_byte_perm(p[0], p[1], 0x0073), _byte_perm(p[2], p[3], 0x0073), 0x5410)
        assert mant == sum((p[k] >> 24) << (8 * k) for k in range(4))


def test_decode_sign_spread():
    nib = np.arange(16, dtype=np.uint64)
    expect = sum(((nib >> np.uint64(b)) & np.uint64(1)) << np.uint64(8 * b + 7) for b in range(4))
    even = _mul32(nib, 0x10204080) & np.uint64(0x80808080)             # signs at bits 0-3
    odd = _mul32(nib << np.uint64(4), 0x01020408) & np.uint64(0x80808080)  # signs at bits 4-7
    assert np.array_equal(even, expect)
    assert np.array_equal(odd, expect)


def test_decode_mantissa_spread():
    byte = np.arange(256, dtype=np.uint64)
    ev = byte & np.uint64(0x33)   # mantissas of elements 0 and 2 of the byte
    od = byte & np.uint64(0xCC)   # of elements 1 and 3
    got = (_mul32(ev, 0x1001) + _mul32(od, 0x40040)) & np.uint64(0xFFFFFFFF) & np.uint64(0x03030303)
    expect = sum(((byte >> np.uint64(2 * b)) & np.uint64(3)) << np.uint64(8 * b) for b in range(4))
    assert np.array_equal(got, expect)


def test_escape_flag_word():
    """fl = n0 | n1 << 1 from the escape-nibble flags of two code words has one
    bit per code 15, and fl & (fl - 1) is nonzero exactly when two or more."""
    rng = np.random.default_rng(3)
    for _ in range(2000):
        codes = rng.integers(0, 16, size=16)
        codes[rng.random(16) < 0.2] = 15
        c0 = sum(int(c) << (4 * j) for j, c in enumerate(codes[:8]))
        c1 = sum(int(c) << (4 * j) for j, c in enumerate(codes[8:]))

        def nibbles(cw):
            t = cw & (cw >> 1)
            return t & (t >> 2) & 0x11111111

        fl = nibbles(c0) | (nibbles(c1) << 1)
        esc = [j for j in range(16) if codes[j] == 15]
        assert bin(fl).count("1") == len(esc)
        assert ((fl & (fl - 1)) != 0) == (len(esc) >= 2)
        if len(esc) == 1:
            p = (fl & -fl).bit_length() - 1
            j = (p >> 2) | ((p & 1) << 3)
            assert j == esc[0]
