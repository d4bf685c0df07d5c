"""Error paths of the CUDA library: every failure is a status, never a fault or a hang.

Faults are made on the host (corrupted bytes, bad arguments, a job counter
moved so that a predecessor tile never publishes); no test faults, traps or
hangs the GPU: the look-back wait gives up after its limit and reports.
"""
import ctypes

import numpy as np
import pytest
import torch

import fieldcodec
import kvgen
import oracle_pins
from gpu_helpers import from_raw, gpu_decode, gpu_encode, raw_of, sz

pytestmark = pytest.mark.gpu


def _stream():
    rng = np.random.default_rng(5)
    raw = oracle_pins._kvlike(rng, 10000, 0)
    w = raw.view("<u2").copy()
    w[::97] = (np.arange(w[::97].size) % 20 + 20) << 7     # 20 rare exponents -> escapes
    raw = w.view(np.uint8)
    plan, s = gpu_encode(0, from_raw(raw, 0))
    assert fieldcodec.parse(s)["E"] > 0
    return raw, s


CORRUPTIONS = {
    "magic": lambda s, f: s.__setitem__(0, s[0] ^ 1),
    "version": lambda s, f: s.__setitem__(4, 2),
    "block_log2": lambda s, f: s.__setitem__(7, 11),
    "n_mismatch": lambda s, f: s.__setitem__(8, s[8] ^ 1),
    "E_too_large": lambda s, f: s.__setitem__(slice(16, 24), np.frombuffer(np.uint64(f["n"] + 1).tobytes(), np.uint8)),
    "total_wrong": lambda s, f: s.__setitem__(40, s[40] ^ 1),
    "cb_duplicate": lambda s, f: s.__setitem__(25, s[24]),
    "unknown_flag": lambda s, f: s.__setitem__(39, 2),
    "offset_tampered": lambda s, f: s.__setitem__(64 + 4, s[64 + 4] ^ 1),
    "first_offset": lambda s, f: s.__setitem__(64, 1),
    "last_offset": lambda s, f: s.__setitem__(64 + 4 * f["nb"], s[64 + 4 * f["nb"]] ^ 1),
    "code_flipped_to_escape": lambda s, f: s.__setitem__(f["starts"][-1] + 3, 0xFF),
}


@pytest.mark.parametrize("what", sorted(CORRUPTIONS))
def test_corrupt_stream_is_reported(what):
    m = sz()
    raw, s = _stream()
    f = fieldcodec.parse(s)
    bad = s.copy()
    CORRUPTIONS[what](bad, f)
    gpu_decode(0, bad, 10000, expect_status=m.SZ_ERR_CORRUPT_STREAM)


def test_wrong_dtype_stream():
    m = sz()
    raw, s = _stream()
    bad = s.copy()
    bad[6] = 1  # claims E5M2; decoding it as BF16 is refused
    gpu_decode(0, bad, 10000, expect_status=m.SZ_ERR_UNSUPPORTED_DTYPE)


def test_truncated_stream_rejected_on_host_or_device():
    m = sz()
    raw, s = _stream()
    comp = torch.from_numpy(s.copy()).cuda()
    out = torch.empty(20000, dtype=torch.uint8, device="cuda")
    ws = m.new_workspace(0, [10000])
    min_total = m.sz_stream_bytes(0, 10000, 0)
    with pytest.raises(m.SplitZipError) as e:          # shorter than any stream for n: host check
        m.sz_decode(0, comp, out.view(torch.bfloat16), ws, comp_bytes=min_total - 1)
    assert e.value.status == m.SZ_ERR_CORRUPT_STREAM
    m.sz_decode(0, comp, out.view(torch.bfloat16), ws, comp_bytes=s.size - 1)  # escapes cut: device check
    assert m.sz_last_device_status(ws) == m.SZ_ERR_CORRUPT_STREAM
    m.sz_decode(0, comp, out.view(torch.bfloat16), ws)
    assert m.sz_last_device_status(ws) == 0
    assert np.array_equal(out.cpu().numpy(), raw)


def test_host_argument_checks():
    m = sz()
    x = torch.zeros(4096 * 2 + 8, dtype=torch.bfloat16, device="cuda")
    ws = m.new_workspace(0, [x.numel()])
    plan = m.new_plans(1)
    mis = x.view(torch.uint8)[2:2 + 2 * 4096].view(torch.bfloat16)  # 2-byte offset: misaligned
    with pytest.raises(m.SplitZipError) as e:
        m.sz_plan(0, mis, ws, plan)
    assert e.value.status == m.SZ_ERR_INVALID_ARG
    with pytest.raises(m.SplitZipError) as e:
        m.sz_plan(0, x, ws[:100], plan)
    assert e.value.status == m.SZ_ERR_BUFFER_TOO_SMALL
    with pytest.raises(m.SplitZipError) as e:
        m.sz_plan(7, x, ws, plan)
    assert e.value.status == m.SZ_ERR_UNSUPPORTED_DTYPE
    # n >= 2^32 is refused before anything touches the (small) buffer
    st = m.lib.sz_plan(0, ctypes.c_void_p(x.data_ptr()), 1 << 32, ctypes.c_void_p(ws.data_ptr()),
                       ws.nbytes, ctypes.c_void_p(plan.data_ptr()),
                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == m.SZ_ERR_INVALID_ARG
    # batch size limits
    st = m.lib.sz_plan_batched(0, 0, None, None, ctypes.c_void_p(ws.data_ptr()), ws.nbytes,
                               ctypes.c_void_p(plan.data_ptr()), None)
    assert st == m.SZ_ERR_INVALID_ARG
    assert m.sz_last_device_status(ws) == 0


def test_output_capacity():
    m = sz()
    raw, s = _stream()
    x = from_raw(raw, 0)
    ws = m.new_workspace(0, [10000])
    plan = m.new_plans(1)
    m.sz_plan(0, x, ws, plan)
    total = m.sz_compressed_size(plan)
    small = torch.zeros(m.sz_stream_bytes(0, 10000, 0) - 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.SplitZipError) as e:          # below the smallest stream: host check
        m.sz_encode(0, plan, x, small, ws)
    assert e.value.status == m.SZ_ERR_BUFFER_TOO_SMALL
    out = torch.full((total - 1,), 0xA5, dtype=torch.uint8, device="cuda")
    m.sz_encode(0, plan, x, out, ws)                    # escapes do not fit: device check
    assert m.sz_last_device_status(ws) == m.SZ_ERR_BUFFER_TOO_SMALL
    assert (out.cpu().numpy() == 0xA5).all(), "nothing may be written"
    out = torch.zeros(total, dtype=torch.uint8, device="cuda")
    m.sz_encode(0, plan, x, out, ws)
    assert m.sz_last_device_status(ws) == 0
    assert np.array_equal(out.cpu().numpy(), s)


def test_plan_mismatch():
    m = sz()
    raw, s = _stream()
    x = from_raw(raw, 0)
    other = from_raw(np.random.default_rng(3).integers(0, 256, raw.size).astype(np.uint8), 0)
    ws = m.new_workspace(0, [10000])
    plan = m.new_plans(1)
    m.sz_plan(0, x, ws, plan)
    out = torch.zeros(m.sz_max_compressed_size(0, 10000), dtype=torch.uint8, device="cuda")
    m.sz_encode(0, plan, other, out, ws)               # same n, other data: E differs
    assert m.sz_last_device_status(ws) == m.SZ_ERR_PLAN_MISMATCH
    y = x[:9000]
    m.sz_encode(0, plan, y, out, ws)                   # other n
    assert m.sz_last_device_status(ws) == m.SZ_ERR_PLAN_MISMATCH
    m.sz_workspace_init(ws)
    m.sz_encode(0, plan, x, out, ws)
    assert m.sz_last_device_status(ws) == 0
    assert np.array_equal(out[: s.size].cpu().numpy(), s)


def test_lookback_wait_times_out_and_reports():
    """A predecessor tile that never publishes: the wait ends after its limit with
    SZ_ERR_TIMEOUT, the kernel returns, and the context stays usable.

    The workspace's job counter (control word 3) is moved to 1 on the host, so job 0
    -- the tensor's first chunk of blocks -- is never run and its status word is
    never set; every later chunk's look-back waits on it."""
    m = sz()
    n = 4096 * 64
    x = kvgen.stress_tensor(n, 10, 77).cuda()
    ws = m.new_workspace(0, [n])
    plan = m.new_plans(1)
    m.sz_plan(0, x, ws, plan)
    out = torch.zeros(m.sz_max_compressed_size(0, n), dtype=torch.uint8, device="cuda")
    ws.view(torch.int32)[3] = 1
    m.sz_encode(0, plan, x, out, ws)
    assert m.sz_last_device_status(ws) == m.SZ_ERR_TIMEOUT
    # the kernel left its counters ready; a fresh run is correct again
    m.sz_workspace_init(ws)
    ref_plan, ref = gpu_encode(0, x)
    m.sz_encode(0, plan, x, out, ws)
    assert m.sz_last_device_status(ws) == 0
    assert np.array_equal(out[: ref.size].cpu().numpy(), ref)
