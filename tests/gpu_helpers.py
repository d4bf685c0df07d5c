"""Helpers for the GPU parity tests: run the CUDA library through its C ABI and
compare with the CPU oracle byte for byte."""
import numpy as np
import pytest
import torch

import oracle


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA GPU (run the gpu-marked tests on a B200)")


def sz():
    require_gpu()
    import fp8_kv_cache_exp_b200 as m  # loads libsplitzip.so or raises
    return m


def raw_of(x: torch.Tensor) -> np.ndarray:
    """Little-endian bytes of a tensor, on the host."""
    return x.detach().contiguous().view(torch.uint8).reshape(-1).cpu().numpy()


def from_raw(raw: np.ndarray, dtype: int, device="cuda") -> torch.Tensor:
    tdt = torch.bfloat16 if dtype == 0 else torch.float8_e5m2
    if raw.size == 0:
        return torch.empty(0, dtype=tdt, device=device)
    t = torch.from_numpy(np.ascontiguousarray(raw).copy()).to(device)
    return t.view(tdt)


POISON = 0xA5


def gpu_encode(dtype: int, x: torch.Tensor, ws=None):
    """Plan + encode one tensor on the GPU; returns (plan bytes, stream bytes) on the host."""
    m = sz()
    n = m.numel_of(x, dtype)
    if ws is None:
        ws = m.new_workspace(dtype, [n])
    plan = m.new_plans(1)
    m.sz_plan(dtype, x, ws, plan)
    size = m.sz_compressed_size(plan)
    cap = m.sz_max_compressed_size(dtype, n)
    out = torch.full((cap,), POISON, dtype=torch.uint8, device=x.device)
    m.sz_encode(dtype, plan, x, out, ws)
    st = m.sz_last_device_status(ws)
    assert st == 0, m.sz_status_string(st)
    return plan.cpu().numpy().reshape(-1), out[:size].cpu().numpy()


def gpu_decode(dtype: int, stream: np.ndarray, n: int, ws=None, expect_status=0):
    m = sz()
    comp = torch.from_numpy(np.ascontiguousarray(stream).copy()).cuda()
    out = torch.full((max(n, 1) * (2 if dtype == 0 else 1),), POISON, dtype=torch.uint8, device="cuda")
    out = out[: n * (2 if dtype == 0 else 1)]
    if ws is None:
        ws = m.new_workspace(dtype, [n])
    m.sz_decode(dtype, comp, out, ws)
    st = m.sz_last_device_status(ws)
    assert st == expect_status, (m.sz_status_string(st), st)
    return out.cpu().numpy()


def check_parity(dtype: int, raw: np.ndarray):
    """GPU plan, stream and decode equal the oracle's, bit for bit; cross-decode both ways."""
    n = raw.size // (2 if dtype == 0 else 1)
    ref = oracle.encode(dtype, raw)
    x = from_raw(raw, dtype)
    plan, stream = gpu_encode(dtype, x)
    assert np.array_equal(plan, ref[:64]), ("plan differs", plan[:48], ref[:48])
    assert stream.size == ref.size, (stream.size, ref.size)
    diff = np.nonzero(stream != ref)[0]
    assert diff.size == 0, ("stream differs", int(diff[0]), int(stream[diff[0]]), int(ref[diff[0]]))
    dec = gpu_decode(dtype, stream, n)
    assert np.array_equal(dec, raw), "GPU decode of the GPU stream differs"
    dec2 = gpu_decode(dtype, ref, n)
    assert np.array_equal(dec2, raw), "GPU decode of the oracle stream differs"
    assert np.array_equal(oracle.decode(stream, n, dtype), raw)
    return ref
