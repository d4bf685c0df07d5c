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


def _noalloc_stream(m, dtype, plan, x):
    n = m.numel_of(x, dtype)
    out = torch.full((m.sz_max_compressed_size(dtype, n),), 0x5A, dtype=torch.uint8, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = m.lib.sz_encode_noalloc(dtype, ctypes.c_void_p(plan.data_ptr()), ctypes.c_void_p(x.data_ptr()), n,
                                 ctypes.c_void_p(out.data_ptr()), out.nbytes,
                                 ctypes.c_void_p(status.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == m.SZ_OK, m.sz_status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == m.SZ_OK
    return out[: m.sz_compressed_size(plan)]


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
