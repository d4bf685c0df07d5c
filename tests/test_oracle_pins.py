"""The CPU oracle against its pins (no GPU).  See oracle_pins for what pins what."""
import numpy as np
import pytest

import fieldcodec
import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_exhaustive_bf16_odd_repeats(orc):
    oracle_pins.pin_exhaustive_bf16(orc, repeats=(5, 7))


def test_golden_fixtures_present():
    names = [f.rsplit("/", 1)[-1] for f in oracle_pins.golden_files()]
    assert "bf16_n17.txt" in names and "e5m2_n17.txt" in names
    assert "bf16_n17_raw.txt" in names and "e5m2_n17_raw.txt" in names


def test_encode_reports_small_buffer(orc):
    raw = np.zeros(2 * 1000, dtype=np.uint8)
    need = orc.compressed_size(0, 1000, 0)
    r, _ = orc.encode_status(0, raw, cap=need - 1)
    assert r == -oracle.ERR_SMALL
    r, s = orc.encode_status(0, raw, cap=need)
    assert r == need


def test_encode_rejects_bad_dtype(orc):
    r, _ = orc.encode_status(7, np.zeros(10, np.uint8), cap=4096)
    assert r == -oracle.ERR_DTYPE


def _stream(orc, n=10000, seed=5):
    rng = np.random.default_rng(seed)
    raw = oracle_pins._kvlike(rng, n, 0)
    # force some escapes: 20 distinct rare exponents
    w = raw.view("<u2").copy()
    w[::97] = (np.arange(w[::97].size) % 20 + 20) << 7
    raw = w.view(np.uint8)
    s = orc.encode(0, raw)
    assert fieldcodec.parse(s)["E"] > 0
    return raw, s


CORRUPTIONS = {
    "magic": lambda s, f: s.__setitem__(0, s[0] ^ 1),
    "version": lambda s, f: s.__setitem__(4, 2),
    "dtype": lambda s, f: s.__setitem__(6, 9),
    "block_log2": lambda s, f: s.__setitem__(7, 11),
    "n_mismatch": lambda s, f: s.__setitem__(8, s[8] ^ 1),
    "E_too_large": lambda s, f: s.__setitem__(slice(16, 24), np.frombuffer(np.uint64(f["n"] + 1).tobytes(), np.uint8)),
    "total_wrong": lambda s, f: s.__setitem__(40, s[40] ^ 1),
    "cb_duplicate": lambda s, f: s.__setitem__(25, s[24]),
    "unknown_flag": lambda s, f: s.__setitem__(39, 2),
    "offset_tampered": lambda s, f: s.__setitem__(64 + 4, s[64 + 4] ^ 1),
    "last_offset": lambda s, f: s.__setitem__(64 + 4 * f["nb"], s[64 + 4 * f["nb"]] ^ 1),
}


@pytest.mark.parametrize("what", sorted(CORRUPTIONS))
def test_decode_rejects_corruption(orc, what):
    raw, s = _stream(orc)
    f = fieldcodec.parse(s)
    bad = s.copy()
    CORRUPTIONS[what](bad, f)
    rc, _ = orc.decode_status(bad, 10000, 0)
    assert rc != oracle.OK


def test_decode_rejects_truncation(orc):
    raw, s = _stream(orc)
    for cut in (0, 10, 63, 64, s.size // 2, s.size - 1):
        rc, _ = orc.decode_status(s[:cut], 10000, 0)
        assert rc == oracle.ERR_CORRUPT


def test_decode_rejects_wrong_n(orc):
    raw, s = _stream(orc)
    rc, _ = orc.decode_status(s, 9999, 0)
    assert rc == oracle.ERR_ARG


@pytest.mark.parametrize("dtype", [0, 1])
def test_decode_rejects_broken_raw_marker(orc, dtype):
    """A flagged stream whose offsets table no longer marks its raw blocks, or that lost
    its flag, is rejected (the same cases the GPU decoder reports)."""
    rng = np.random.default_rng(9 + dtype)
    n = 3 * 4096 + 100
    raw = rng.integers(0, 256, n * (2 if dtype == 0 else 1)).astype(np.uint8)
    s = orc.encode(dtype, raw, raw_blocks=True)
    assert np.array_equal(orc.decode(s, n, dtype), raw)
    for what in ("count_plus_one", "flag_cleared"):
        bad = s.copy()
        if what == "count_plus_one":
            bad[68] ^= 1
        else:
            bad[39] = 0
        rc, _ = orc.decode_status(bad, n, dtype)
        assert rc == oracle.ERR_CORRUPT, what
