"""The C-ABI library loads and exports every function include/splitzip.h declares;
host-only size functions agree with the oracle's closed form (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "splitzip.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sz_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    path = __graft_entry__._build_module().build()
    return ctypes.CDLL(path)


def test_header_declares_the_calls():
    names = _declared()
    for must in ("sz_plan", "sz_encode", "sz_decode", "sz_compressed_size", "sz_plan_batched",
                 "sz_encode_batched", "sz_decode_batched", "sz_last_device_status",
                 "sz_workspace_bytes", "sz_max_compressed_size", "sz_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_header():
    import fp8_kv_cache_exp_b200 as sz
    for n in _declared():
        assert hasattr(sz, n), n


@pytest.mark.parametrize("dtype", [0, 1])
def test_host_sizes_match_oracle(lib, dtype):
    lib.sz_stream_bytes.restype = ctypes.c_size_t
    lib.sz_stream_bytes.argtypes = [ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64]
    lib.sz_max_compressed_size.restype = ctypes.c_size_t
    lib.sz_max_compressed_size.argtypes = [ctypes.c_int, ctypes.c_uint64]
    rng = np.random.default_rng(0)
    for n in [0, 1, 2, 4095, 4096, 4097, 8388608, (1 << 31), (1 << 32) - 1] + list(rng.integers(0, 1 << 30, 20)):
        n = int(n)
        for E in (0, n // 7, n):
            assert lib.sz_stream_bytes(dtype, n, E) == oracle.compressed_size(dtype, n, E)
        assert lib.sz_max_compressed_size(dtype, n) == oracle.compressed_size(dtype, n, n)
    assert lib.sz_stream_bytes(9, 10, 0) == 0


def test_workspace_sizes(lib):
    import fp8_kv_cache_exp_b200 as sz
    # control block, histograms, tickets, one look-back word per 4096-element
    # block, then one per 32 blocks plus one per tensor and one more
    one = sz.sz_workspace_bytes(0, 8388608)
    assert one == 256 + 1024 + 256 + 8 * 2048 + 8 * (2048 // 32 + 1 + 1)
    assert sz.sz_workspace_bytes_batched(0, [8388608] * 64) == \
        256 + 64 * 1024 + 256 + 8 * 2048 * 64 + 8 * (2048 * 64 // 32 + 64 + 1)
    assert sz.sz_workspace_bytes_batched(0, [1] * 257) == 0


def test_status_strings():
    import fp8_kv_cache_exp_b200 as sz
    assert sz.sz_status_string(0) == "ok"
    assert "corrupt" in sz.sz_status_string(4)
    assert sz.sz_status_string(99) == "unknown status"


def test_plan_set_flags_host_checks(lib):
    """Rejected on the host, before any CUDA call: no plans, too many, a null or
    misaligned pointer, unknown flag bits."""
    f = lib.sz_plan_set_flags
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_uint, ctypes.c_void_p]
    fake = 1 << 20  # never dereferenced: every call below fails its checks first
    assert f(0, fake, 1, None) == 1
    assert f(257, fake, 1, None) == 1
    assert f(1, None, 1, None) == 1
    assert f(1, fake + 4, 1, None) == 1
    assert f(1, fake, 2, None) == 1


def test_binding_host_checks():
    """The binding's own argument checks on a batch (no GPU call is reached)."""
    import torch
    import fp8_kv_cache_exp_b200 as sz
    plans = torch.zeros((2, 64), dtype=torch.uint8)
    xs = [torch.zeros(16, dtype=torch.bfloat16)]
    with pytest.raises(ValueError):
        sz.Batch(sz.SZ_BF16, xs, [], torch.zeros(1024, dtype=torch.uint8), plans)
    with pytest.raises(ValueError):
        sz.Batch(sz.SZ_BF16, None, [torch.zeros(256, dtype=torch.uint8)], torch.zeros(1024, dtype=torch.uint8),
                 plans, src_pages=[sz.sz_paged_t()])  # paged without element counts
