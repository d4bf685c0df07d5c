"""Pins for the CPU oracle: checks against facts that do not come from the oracle itself.

Each pin takes an `oracle.Oracle` instance (the committed build, or a mutated
build in the mutation test) and raises AssertionError on failure.  What pins
what:

  golden          hand-worked streams (tests/golden/*.txt) -> header, table,
                  planes, codes, escapes, padding, byte for byte
  exhaustive      every BF16 and every E5M2 bit pattern round-trips bitwise
                  (lossless: SplitZip project page, FAQ "Is SplitZip lossy?")
                  and matches the independent numpy reader (fieldcodec.check)
  ragged sizes    closed-form size and layout for n around block and
                  alignment boundaries, via the independent reader
  brute force     the codebook maximises coverage and is the lexicographically
                  smallest such set, by enumerating every candidate subset
  special cases   all-zero, <= 15 distinct exponents, 16 equally frequent
                  exponents, uniform random bits (np.bincount + sort)
  ratio           ratio <= 16/12 (BF16) and <= 8/7 (E5M2): 12 and 7 coded bits
                  per element plus escapes (project page: "up to 1.14x" on FP8)
  codebook reuse  encoding with a given codebook: the ordinary encoding when it
                  is the tensor's own (found by numpy), the reader-checked v1
                  encoding under any other, a hand-worked golden stream
                  (bf16_n17_reuse.txt), and refusal of invalid codebooks
  raw blocks      with header flag bit 0: hand-worked golden streams
                  (bf16_n17_raw.txt, e5m2_n17_raw.txt), the exact threshold
                  (K - 1 escapes coded, K raw), the ordinary stream when no
                  block reaches it, no block above its raw bytes (closed form
                  for uniform random bits), mixed streams checked by the
                  independent reader, every bit pattern round-trips
"""
import itertools
import os

import numpy as np

import fieldcodec
import oracle

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ------------------------------------------------------------------ golden

def load_golden(path):
    """Parse a golden fixture: returns (dtype, raw input bytes, expected stream).
    A fixture with a `codebook` line was encoded with that given codebook; see
    golden_codebook().  A `flags 1` line means raw blocks were allowed."""
    dtype = n = total = None
    raw = None
    at = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, _, rest = line.partition(" ")
            if key == "dtype":
                dtype = int(rest)
            elif key == "n":
                n = int(rest)
            elif key == "total":
                total = int(rest)
            elif key == "input_hex":
                words = [int(w, 16) for w in rest.split()]
                raw = np.array(words, dtype="<u2" if dtype == 0 else np.uint8).view(np.uint8)
            elif key in ("codebook", "flags"):
                pass
            elif key == "at":
                off, _, hexes = rest.partition(":")
                at.append((int(off), bytes(int(h, 16) for h in hexes.split())))
    assert raw is not None and raw.size == n * (2 if dtype == 0 else 1)
    expect = np.zeros(total, dtype=np.uint8)
    for off, b in at:
        expect[off: off + len(b)] = np.frombuffer(b, dtype=np.uint8)
    return dtype, raw, expect


def golden_codebook(path):
    """The given codebook of a codebook-reuse fixture (15 uint8), or None."""
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line.startswith("codebook "):
                cb = np.array([int(h, 16) for h in line.split()[1:]], dtype=np.uint8)
                assert cb.size == 15
                return cb
    return None


def golden_flags(path):
    """The header flags a fixture was encoded with (0 unless a `flags` line says)."""
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line.startswith("flags "):
                return int(line.split()[1])
    return 0


def golden_files():
    return sorted(os.path.join(GOLDEN_DIR, f) for f in os.listdir(GOLDEN_DIR) if f.endswith(".txt")
                  and f != "README.txt")


def pin_golden(orc):
    for path in golden_files():
        dtype, raw, expect = load_golden(path)
        cb = golden_codebook(path)
        rb = golden_flags(path) == 1
        got = orc.encode(dtype, raw, raw_blocks=rb) if cb is None else orc.encode_codebook(dtype, raw, cb, raw_blocks=rb)
        assert got.size == expect.size, (path, got.size, expect.size)
        diff = np.nonzero(got != expect)[0]
        assert diff.size == 0, (path, "first differing byte", int(diff[0]))
        n = raw.size // (2 if dtype == 0 else 1)
        assert np.array_equal(orc.decode(expect, n, dtype), raw), path
        assert np.array_equal(fieldcodec.decode(expect), raw), path


# -------------------------------------------------------------- exhaustive

def _roundtrip_and_check(orc, raw, dtype):
    n = raw.size // (2 if dtype == 0 else 1)
    s = orc.encode(dtype, raw)
    back = orc.decode(s, n, dtype)
    assert np.array_equal(back, raw), "round trip differs"
    fieldcodec.check(s, raw, dtype)


def pin_exhaustive_bf16(orc, repeats=(1, 3)):
    allp = np.arange(65536, dtype=np.uint32).astype("<u2")
    rng = np.random.default_rng(0)
    shuffled = allp[rng.permutation(allp.size)]
    for x in (allp, shuffled):
        for k in repeats:
            _roundtrip_and_check(orc, np.repeat(x, k).view(np.uint8), 0)


def pin_exhaustive_e5m2(orc, repeats=(1, 3, 5, 17)):
    allp = np.arange(256, dtype=np.uint32).astype(np.uint8)
    rng = np.random.default_rng(0)
    shuffled = allp[rng.permutation(allp.size)]
    for x in (allp, shuffled):
        for k in repeats:
            _roundtrip_and_check(orc, np.repeat(x, k), 1)


# ------------------------------------------------------------ ragged sizes

RAGGED_N = (0, 1, 2, 3, 7, 8, 9, 255, 256, 257, 511, 4095, 4096, 4097, 8191, 8192, 8193, 12289,
            3 * 4096 + 1001)


def _kvlike(rng, n, dtype):
    """Small KV-like input: normal values with per-position scale, some zeros."""
    v = rng.standard_normal(n).astype(np.float32) * np.exp(rng.standard_normal(n)).astype(np.float32)
    bits = v.view(np.uint32) >> 16  # truncation to bf16 bits is enough for a test input
    bits[rng.random(n) < 0.01] = 0
    if dtype == 0:
        return bits.astype("<u2").view(np.uint8)
    # an E5M2-like byte: sign, exponent from the bf16 exponent clamped into 5 bits, 2 mantissa bits
    e8 = (bits >> 7) & 0xFF
    e5 = np.clip(e8.astype(np.int64) - 112, 0, 31).astype(np.uint32)
    return (((bits >> 15) & 1) << 7 | (e5 << 2) | ((bits >> 5) & 3)).astype(np.uint8)


def pin_ragged_sizes(orc):
    rng = np.random.default_rng(1234)
    for dtype in (0, 1):
        for n in RAGGED_N:
            for kind in ("kv", "uniform"):
                if kind == "kv":
                    raw = _kvlike(rng, n, dtype)
                else:
                    raw = rng.integers(0, 256, n * (2 if dtype == 0 else 1)).astype(np.uint8)
                s = orc.encode(dtype, raw)
                f = fieldcodec.parse(s)
                assert s.size == fieldcodec.layout(dtype, n, f["E"])[4]
                assert s.size == orc.compressed_size(dtype, n, f["E"])
                # E equals n minus the top-15 coverage of the exponent histogram
                e = fieldcodec.exponents(raw, dtype)
                cnt = np.bincount(e, minlength=256 if dtype == 0 else 32)
                assert f["E"] == n - int(np.sort(cnt)[::-1][:15].sum())
                _roundtrip_and_check(orc, raw, dtype)


# ------------------------------------------------------------- brute force

def _bruteforce_best(cnt, present):
    """Every 15-subset of the present values: (max coverage, lexicographically smallest best set).

    With at least 15 present values, any set holding an absent value (count 0)
    covers less than some set of present values, so the enumeration over present
    values alone covers every candidate that can reach the maximum."""
    best, best_sets = -1, []
    for S in itertools.combinations(sorted(present), 15):
        cov = int(sum(cnt[v] for v in S))
        if cov > best:
            best, best_sets = cov, [S]
        elif cov == best:
            best_sets.append(S)
    return best, min(best_sets)


def pin_bruteforce_codebook(orc, cases=40):
    rng = np.random.default_rng(7)
    for case in range(cases):
        dtype = case % 2
        nv = 256 if dtype == 0 else 32
        k = int(rng.integers(15, 21))              # alphabet of 15..20 values
        alphabet = rng.choice(nv, size=k, replace=False)
        n = int(rng.integers(k, 65))               # n <= 64, every value at least once
        e = np.concatenate([alphabet, rng.choice(alphabet, size=n - k)])
        rng.shuffle(e)
        if dtype == 0:
            raw = ((rng.integers(0, 2, n) << 15) | (e << 7) | rng.integers(0, 128, n)).astype("<u2").view(np.uint8)
        else:
            raw = ((rng.integers(0, 2, n) << 7) | (e << 2) | rng.integers(0, 4, n)).astype(np.uint8)
        cnt = np.bincount(e, minlength=nv)
        cb = orc.codebook(dtype, orc.histogram(dtype, raw))
        best, best_set = _bruteforce_best(cnt, alphabet.tolist())
        assert int(cnt[cb].sum()) == best, "codebook does not maximise coverage"
        assert tuple(sorted(cb.tolist())) == best_set, "not the smallest-valued best set"
        # codes in rank order: counts non-increasing, ties by increasing value
        for c in range(14):
            a, b = int(cb[c]), int(cb[c + 1])
            assert cnt[a] > cnt[b] or (cnt[a] == cnt[b] and a < b), (c, a, b)
        s = orc.encode(dtype, raw)
        assert fieldcodec.parse(s)["E"] == n - best


# ----------------------------------------------------------- special cases

def pin_special_cases(orc):
    # all zero (+0.0): E = 0, codebook 0..14, sm plane all 0x00; -0.0 gives 0x80
    for val, smb in ((0x0000, 0x00), (0x8000, 0x80)):
        raw = np.full(5000, val, dtype="<u2").view(np.uint8)
        s = orc.encode(0, raw)
        f = fieldcodec.parse(s)
        assert f["E"] == 0 and f["cb"].tolist() == list(range(15))
        assert (s[f["starts"][0]: f["starts"][0] + 5000] == smb).all()
        assert np.array_equal(orc.decode(s, 5000, 0), raw)
    # <= 15 distinct exponents: no escapes; unused codes go to the smallest absent values
    rng = np.random.default_rng(3)
    for k in (1, 2, 5, 14, 15):
        vals = rng.choice(256, size=k, replace=False)
        e = rng.choice(vals, size=3000)
        raw = ((e << 7) | rng.integers(0, 128, 3000)).astype("<u2").view(np.uint8)
        s = orc.encode(0, raw)
        f = fieldcodec.parse(s)
        assert f["E"] == 0
        present = set(np.unique(e).tolist())
        assert present <= set(f["cb"].tolist())
        absent = [v for v in f["cb"].tolist() if v not in present]
        assert absent == sorted(v for v in range(256) if v not in present)[: len(absent)]
    # 16 equally frequent exponents: the largest is escaped, E = n/16
    e = np.tile(np.arange(100, 116), 256)
    rng.shuffle(e)
    raw = (e << 7).astype("<u2").view(np.uint8)
    s = orc.encode(0, raw)
    f = fieldcodec.parse(s)
    assert f["E"] == e.size // 16
    assert sorted(f["cb"].tolist()) == list(range(100, 115))
    assert (s[f["esc"]: f["esc"] + f["E"]] == 115).all()
    # uniform random bits: E = n - (sum of the 15 largest exponent counts)
    raw = rng.integers(0, 256, 2 * 40000).astype(np.uint8)
    s = orc.encode(0, raw)
    cnt = np.bincount(fieldcodec.exponents(raw, 0), minlength=256)
    assert fieldcodec.parse(s)["E"] == 40000 - int(np.sort(cnt)[::-1][:15].sum())


def pin_ratio_ceiling(orc):
    rng = np.random.default_rng(11)
    for dtype, ceiling in ((0, 16 / 12), (1, 8 / 7)):
        for n in (1, 4096, 100000, 1 << 20):
            raw = _kvlike(rng, n, dtype)
            s = orc.encode(dtype, raw)
            assert raw.size / s.size <= ceiling
        # no escapes and large n: the ratio approaches the ceiling
        n = 1 << 20
        raw = np.zeros(n * (2 if dtype == 0 else 1), dtype=np.uint8)
        assert raw.size / orc.encode(dtype, raw).size > ceiling * 0.995


# ---------------------------------------------------------- codebook reuse

def pin_codebook_reuse(orc):
    """Encoding with a given codebook: with the tensor's own codebook (found here
    by numpy, not by the oracle) it is the ordinary encoding; with any other it is
    still the v1 encoding of the data under that codebook, checked field by field
    by the independent reader, and lossless; bad codebooks are refused."""
    rng = np.random.default_rng(77)
    for dtype in (0, 1):
        nbins = 256 if dtype == 0 else 32
        for n in (0, 1, 4095, 4096, 4097, 9000, 20000):
            raw = _kvlike(rng, n, dtype)
            own = fieldcodec.expected_codebook(raw, dtype)
            assert np.array_equal(orc.encode_codebook(dtype, raw, own), orc.encode(dtype, raw))
            other = _kvlike(rng, 5000, dtype)
            foreign = [fieldcodec.expected_codebook(other, dtype),           # another tensor's
                       rng.choice(nbins, 15, replace=False).astype(np.uint8),  # arbitrary
                       np.arange(nbins - 15, nbins, dtype=np.uint8)]          # misses most values
            for cb in foreign:
                st = orc.encode_codebook(dtype, raw, cb)
                fieldcodec.check(st, raw, dtype, codebook=cb)
                assert np.array_equal(orc.decode(st, n, dtype), raw)
        # nothing in the codebook occurs: every element escapes, E = n
        raw = np.full(3000, 0x3F80 if dtype == 0 else 0x3C, dtype="<u2" if dtype == 0 else np.uint8).view(np.uint8)
        e0 = int(fieldcodec.exponents(raw, dtype)[0])
        cb = np.array([v for v in range(nbins) if v != e0][:15], dtype=np.uint8)
        st = orc.encode_codebook(dtype, raw, cb)
        assert fieldcodec.parse(st)["E"] == 3000
        fieldcodec.check(st, raw, dtype, codebook=cb)
        # refused: a repeated value, a value outside the exponent range
        dup = cb.copy()
        dup[3] = dup[2]
        assert orc.encode_codebook_status(dtype, raw, dup)[0] == -oracle.ERR_ARG
        if dtype == 1:  # every byte value is a BF16 exponent; 32 is out of E5M2's range
            big = cb.copy()
            big[0] = 32
            assert orc.encode_codebook_status(dtype, raw, big)[0] == -oracle.ERR_ARG


# -------------------------------------------------------------- raw blocks

def _threshold_block(rng, dtype, escapes):
    """One full 4096-element block whose own codebook leaves exactly `escapes`
    escapes: 15 frequent exponents share the rest, and the escaped elements are
    spread over rare exponents that each occur less often than any frequent one."""
    common = np.arange(100, 115) if dtype == 0 else np.arange(8, 23)
    rare = (np.arange(20, 84) if dtype == 0 else np.concatenate([np.arange(0, 8), np.arange(23, 32)]))
    n_common = BLOCK_ELEMS - escapes
    e = np.concatenate([np.resize(common, n_common), np.resize(rare, escapes)])
    rng.shuffle(e)
    if dtype == 0:
        return ((rng.integers(0, 2, e.size) << 15) | (e << 7) | rng.integers(0, 128, e.size)).astype("<u2").view(np.uint8)
    return ((rng.integers(0, 2, e.size) << 7) | (e << 2) | rng.integers(0, 4, e.size)).astype(np.uint8)


BLOCK_ELEMS = 4096


def pin_raw_blocks(orc):
    """Raw blocks (header flag bit 0): checked field by field by the independent
    reader; the threshold is exact (K - 1 escapes stay coded, K go raw); data
    whose blocks never reach it gives the ordinary stream with only the flag
    byte changed; no block ever expands, so a stream is at most the raw bytes
    plus header, table and section padding; lossless on every bit pattern."""
    rng = np.random.default_rng(99)
    for dtype in (0, 1):
        es = 2 if dtype == 0 else 1
        K = 2048 if dtype == 0 else 512
        # the threshold, in a block of its own and next to other blocks
        for escapes, is_raw in ((K - 1, False), (K, True), (K + 1, True)):
            blk = _threshold_block(rng, dtype, escapes)
            st = orc.encode(dtype, blk, raw_blocks=True)
            fieldcodec.check(st, blk, dtype, raw_blocks=True)
            f = fieldcodec.parse(st)
            assert f["E"] == (K if is_raw else escapes), (dtype, escapes, f["E"])
            plain = orc.encode(dtype, blk)
            if not is_raw:
                same = plain.copy()
                same[39] = 1
                assert np.array_equal(st, same)
            else:
                assert st.size == plain.size - (escapes - K)
            assert np.array_equal(orc.decode(st, BLOCK_ELEMS, dtype), blk)
        # KV-like data: no block reaches the threshold; only the flag differs
        for n in (1, 4095, 4097, 20000):
            raw = _kvlike(rng, n, dtype)
            st = orc.encode(dtype, raw, raw_blocks=True)
            same = orc.encode(dtype, raw)
            same[39] = 1
            assert np.array_equal(st, same)
        # uniform random bits: every block raw; closed-form size; never above raw
        for n in RAGGED_N:
            raw = rng.integers(0, 256, n * es).astype(np.uint8)
            st = orc.encode(dtype, raw, raw_blocks=True)
            fieldcodec.check(st, raw, dtype, raw_blocks=True)
            sizes = fieldcodec.block_sizes(n)
            escaped = fieldcodec.parse(orc.encode(dtype, raw))["offsets"]
            all_raw = all(int(escaped[b + 1] - escaped[b]) >= fieldcodec.raw_block_bytes(dtype, m)
                          for b, m in enumerate(sizes))
            E_raw = sum(fieldcodec.raw_block_bytes(dtype, m) for m in sizes)
            if all_raw:
                assert fieldcodec.parse(st)["E"] == E_raw
            layout = fieldcodec.layout(dtype, n, fieldcodec.parse(st)["E"])
            assert st.size == layout[4]
            table = fieldcodec.align256(64 + 4 * (layout[0] + 1))
            assert st.size <= table + raw.size + 256 * len(layout[2]), (dtype, n, st.size)
            assert np.array_equal(orc.decode(st, n, dtype), raw)
        # blocks of both kinds in one stream, partial last block included
        parts = [_kvlike(rng, 4096, dtype), rng.integers(0, 256, 4096 * es).astype(np.uint8),
                 _kvlike(rng, 4096, dtype), rng.integers(0, 256, 1500 * es).astype(np.uint8)]
        raw = np.concatenate(parts)
        n = raw.size // es
        st = orc.encode(dtype, raw, raw_blocks=True)
        fieldcodec.check(st, raw, dtype, raw_blocks=True)
        counts = np.diff(fieldcodec.parse(st)["offsets"])
        assert counts[1] == K and counts[3] == fieldcodec.raw_block_bytes(dtype, 1500)
        assert counts[0] < K and counts[2] < K
        assert np.array_equal(orc.decode(st, n, dtype), raw)
        # a codebook that holds nothing of the data: every block raw, still lossless
        raw = _kvlike(rng, 9000, dtype)
        e = set(fieldcodec.exponents(raw, dtype).tolist())
        nbins = 256 if dtype == 0 else 32
        absent = [v for v in range(nbins) if v not in e]
        if len(absent) >= 15:
            cb = np.array(absent[:15], dtype=np.uint8)
            st = orc.encode_codebook(dtype, raw, cb, raw_blocks=True)
            fieldcodec.check(st, raw, dtype, codebook=cb, raw_blocks=True)
            assert fieldcodec.parse(st)["E"] == sum(fieldcodec.raw_block_bytes(dtype, m)
                                                   for m in fieldcodec.block_sizes(9000))
            assert np.array_equal(orc.decode(st, 9000, dtype), raw)
    # every bit pattern, with raw blocks allowed
    allp = np.arange(65536, dtype=np.uint32).astype("<u2")
    shuffled = allp[np.random.default_rng(0).permutation(allp.size)]
    for x in (allp, shuffled):
        st = orc.encode(0, x.view(np.uint8), raw_blocks=True)
        fieldcodec.check(st, x.view(np.uint8), 0, raw_blocks=True)
        assert np.array_equal(orc.decode(st, 65536, 0), x.view(np.uint8))
    e5 = np.repeat(np.arange(256, dtype=np.uint8), 33)
    st = orc.encode(1, e5, raw_blocks=True)
    fieldcodec.check(st, e5, 1, raw_blocks=True)
    assert np.array_equal(orc.decode(st, e5.size, 1), e5)


ALL_PINS = (pin_golden, pin_exhaustive_bf16, pin_exhaustive_e5m2, pin_ragged_sizes,
            pin_bruteforce_codebook, pin_special_cases, pin_ratio_ceiling, pin_codebook_reuse,
            pin_raw_blocks)
