"""sz_encode_noalloc: encoding for callers that cannot allocate device memory.

Some callers -- an engine whose GPU memory is all reserved for its KV pool, or
a transfer hook that gets only the tensor, the destination and a stream -- have
no workspace to pass.  sz_encode_noalloc runs the ordinary encode kernel on a
scratch array the library holds itself.  This test calls it through the C ABI
and checks that its stream equals the one sz_encode writes with a workspace,
byte for byte, on two calls in a row (the second call finds the first call's
leftovers in the shared scratch).  It lives in a file of its own, collected
last, and passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import pytest
import torch

import kvgen
from gpu_helpers import sz

pytestmark = pytest.mark.gpu


def _reference_stream(m, dtype, x):
    n = m.numel_of(x, dtype)
    ws = m.new_workspace(dtype, [n])
    plan = m.new_plans(1)
    m.sz_plan(dtype, x, ws, plan)
    out = torch.full((m.sz_max_compressed_size(dtype, n),), 0xA5, dtype=torch.uint8, device="cuda")
    m.sz_encode(dtype, plan, x, out, ws)
    assert m.sz_last_device_status(ws) == 0
    return plan, out[: m.sz_compressed_size(plan)]


def _noalloc_call(m, dtype, plan, x, out):
    """One sz_encode_noalloc call through the C ABI; returns (host status, device status)."""
    n = m.numel_of(x, dtype)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = m.lib.sz_encode_noalloc(dtype, ctypes.c_void_p(plan.data_ptr()), ctypes.c_void_p(x.data_ptr()), n,
                                 ctypes.c_void_p(out.data_ptr()), out.nbytes,
                                 ctypes.c_void_p(status.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, int(status.item())


def _stream_len(out):
    """Stream length recorded in a stream's own header (bytes 40..47)."""
    return int(out[40:48].cpu().view(torch.int64).item())


def _noalloc_stream(m, dtype, plan, x):
    n = m.numel_of(x, dtype)
    out = torch.full((m.sz_max_compressed_size(dtype, n),), 0x5A, dtype=torch.uint8, device="cuda")
    st, dev = _noalloc_call(m, dtype, plan, x, out)
    assert st == m.SZ_OK, m.sz_status_string(st)
    assert dev == m.SZ_OK, m.sz_status_string(dev)
    return out[: _stream_len(out)]


def test_noalloc_matches_workspace_encode_twice():
    m = sz()
    cfg = kvgen.CONFIGS["llama3-8b"]
    inputs = [(0, kvgen.kv_tensor(cfg, 0, 0, device="cuda")),        # 8.4M elements, 2048 tiles
              (0, kvgen.stress_tensor(4096 * 37 + 11, 10, 123, device="cuda")),
              (1, kvgen.kv_tensor(kvgen.CONFIGS["qwen3-30b-a3b-e5m2"], 0, 1, device="cuda"))]
    for dtype, x in inputs:
        plan, ref = _reference_stream(m, dtype, x)
        first = _noalloc_stream(m, dtype, plan, x)
        second = _noalloc_stream(m, dtype, plan, x)
        assert torch.equal(first, ref)
        assert torch.equal(second, ref)


def test_noalloc_rejects_tensors_beyond_its_scratch():
    m = sz()
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(256, dtype=torch.uint8, device="cuda")
    plan = m.new_plans(1)
    st = m.lib.sz_encode_noalloc(0, ctypes.c_void_p(plan.data_ptr()), ctypes.c_void_p(x.data_ptr()),
                                 m.SZ_NOALLOC_MAX_ELEMS + 1, ctypes.c_void_p(out.data_ptr()), out.nbytes,
                                 None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == m.SZ_ERR_BUFFER_TOO_SMALL


def test_noalloc_reports_device_errors_and_next_call_clears_them():
    """A device-side error of one call reaches d_status; the next clean call,
    which finds that error word in the shared scratch, reports SZ_OK again."""
    m = sz()
    n = 4096 * 21 + 5
    x = kvgen.stress_tensor(n, 10, 77, device="cuda")       # 10% rare exponents: many escapes
    y = kvgen.stress_tensor(n, 0, 78, device="cuda")        # no rare exponent: a different E
    plan_x, ref = _reference_stream(m, 0, x)
    plan_y, _ = _reference_stream(m, 0, y)
    # output capacity: room for the escape-free stream only, the plan needs more
    small = torch.zeros(m.sz_stream_bytes(0, n, 0), dtype=torch.uint8, device="cuda")
    st, dev = _noalloc_call(m, 0, plan_x, x, small)
    assert st == m.SZ_OK
    assert dev == m.SZ_ERR_BUFFER_TOO_SMALL
    assert torch.equal(_noalloc_stream(m, 0, plan_x, x), ref)
    # a plan made for other data of the same size
    out = torch.zeros(m.sz_max_compressed_size(0, n), dtype=torch.uint8, device="cuda")
    st, dev = _noalloc_call(m, 0, plan_y, x, out)
    assert st == m.SZ_OK
    assert dev == m.SZ_ERR_PLAN_MISMATCH
    assert torch.equal(_noalloc_stream(m, 0, plan_x, x), ref)


def test_noalloc_raw_block_plan_matches_workspace_encode():
    """A plan flagged for raw blocks, on uniformly random bits (every block raw)."""
    m = sz()
    n = 4096 * 9 + 100
    x = kvgen.stress_tensor(n, None, 4321, device="cuda")
    ws = m.new_workspace(0, [n])
    plan = m.new_plans(1)
    m.sz_plan(0, x, ws, plan)
    assert m.lib.sz_plan_set_flags(1, ctypes.c_void_p(plan.data_ptr()), m.SZ_FLAG_RAW_BLOCKS,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == m.SZ_OK
    ref = torch.full((m.sz_max_compressed_size(0, n),), 0xA5, dtype=torch.uint8, device="cuda")
    m.sz_encode(0, plan, x, ref, ws)
    assert m.sz_last_device_status(ws) == 0
    ref = ref[: _stream_len(ref)]
    assert ref[39].item() == m.SZ_FLAG_RAW_BLOCKS
    for _ in range(2):
        assert torch.equal(_noalloc_stream(m, 0, plan, x), ref)


def test_noalloc_host_refusal_enqueues_nothing():
    """A call refused on the host (misaligned output) returns at once; its
    d_status copy was never enqueued, so the sentinel stays."""
    m = sz()
    x = kvgen.stress_tensor(4096, 0, 5, device="cuda")
    plan, _ = _reference_stream(m, 0, x)
    buf = torch.zeros(m.sz_max_compressed_size(0, 4096) + 16, dtype=torch.uint8, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = m.lib.sz_encode_noalloc(0, ctypes.c_void_p(plan.data_ptr()), ctypes.c_void_p(x.data_ptr()), 4096,
                                 ctypes.c_void_p(buf.data_ptr() + 1), buf.nbytes - 16,
                                 ctypes.c_void_p(status.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert st == m.SZ_ERR_INVALID_ARG
    assert int(status.item()) == -1
