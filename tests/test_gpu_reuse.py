"""Codebook reuse on the GPU: encode with a codebook made earlier, compared byte for
byte with the oracle's orc_encode_codebook on the same input and the same codebook.

The codebooks are made on the host (the oracle's histogram + codebook, or a
hand-picked set) and written into plan buffers, so nothing the oracle sees comes
from the CUDA path.
"""
import numpy as np
import pytest
import torch

import fieldcodec
import kvgen
import oracle
import oracle_pins
from gpu_helpers import from_raw, raw_of, sz

pytestmark = pytest.mark.gpu

POISON = 0xA5


def plan_with_codebook(cbs):
    """Device plans (T x 64 bytes) holding only the given codebooks (bytes 24..38)."""
    cbs = [np.asarray(c, dtype=np.uint8).reshape(15) for c in cbs]
    h = np.zeros((len(cbs), 64), dtype=np.uint8)
    for i, c in enumerate(cbs):
        h[i, 24:39] = c
    return torch.from_numpy(h).cuda()


def own_codebook(raw, dtype):
    return oracle.codebook(dtype, oracle.histogram(dtype, raw))


def reuse_encode(dtype, raw, cb, cap=None):
    m = sz()
    x = from_raw(raw, dtype)
    n = m.numel_of(x, dtype)
    ws = m.new_workspace(dtype, [n])
    plan = plan_with_codebook([cb])
    cap = m.sz_max_compressed_size(dtype, n) if cap is None else cap
    out = torch.full((cap,), POISON, dtype=torch.uint8, device="cuda")
    total = torch.zeros(1, dtype=torch.int64, device="cuda")
    m.sz_encode_reuse(dtype, plan, x, out, ws, total=total)
    st = m.sz_last_device_status(ws)
    return st, int(total.item()), out.cpu().numpy()


@pytest.mark.parametrize("dtype", [0, 1])
@pytest.mark.parametrize("n", [0, 1, 4095, 4096, 4097, 8 * 4096 + 77, 40 * 4096 + 5])
def test_reuse_matches_oracle(dtype, n):
    rng = np.random.default_rng(n + 17 * dtype)
    raw = oracle_pins._kvlike(rng, n, dtype)
    other = oracle_pins._kvlike(rng, 30000, dtype)
    nbins = 256 if dtype == 0 else 32
    for cb in (own_codebook(raw, dtype), own_codebook(other, dtype),
               rng.choice(nbins, 15, replace=False).astype(np.uint8)):
        ref = oracle.encode_codebook(dtype, raw, cb)
        st, total, out = reuse_encode(dtype, raw, cb)
        assert st == 0
        assert total == ref.size
        assert np.array_equal(out[:total], ref)
        assert np.array_equal(oracle.decode(out[:total], n, dtype), raw)


def test_reuse_with_own_codebook_is_the_ordinary_stream():
    rng = np.random.default_rng(3)
    for dtype in (0, 1):
        raw = oracle_pins._kvlike(rng, 50000, dtype)
        st, total, out = reuse_encode(dtype, raw, own_codebook(raw, dtype))
        assert st == 0 and np.array_equal(out[:total], oracle.encode(dtype, raw))


def test_reuse_across_layers_batched():
    """The Llama-3-8B use: layer 0's codebooks serve every layer of a batch."""
    m = sz()
    cfg = kvgen.CONFIGS["llama3-8b"]
    xs = [kvgen.kv_tensor(cfg, layer, kv) for layer in (0, 5, 31) for kv in (0, 1)]
    raws = [raw_of(x) for x in xs]
    cbs = [own_codebook(raws[kv], 0) for kv in (0, 1)] * 3      # K's and V's of layer 0
    dxs = [x.cuda() for x in xs]
    ns = [x.numel() for x in xs]
    ws = m.new_workspace(0, ns)
    plans = plan_with_codebook(cbs)
    outs = [torch.full((m.sz_max_compressed_size(0, n),), POISON, dtype=torch.uint8, device="cuda") for n in ns]
    totals = torch.zeros(len(xs), dtype=torch.int64, device="cuda")
    m.sz_encode_reuse_batched(0, plans, dxs, outs, ws, totals=totals)
    assert m.sz_last_device_status(ws) == 0
    decs = [torch.empty_like(x) for x in dxs]
    tot = totals.cpu().tolist()
    m.sz_decode_batched(0, [o[:t] for o, t in zip(outs, tot)], decs, ws)
    assert m.sz_last_device_status(ws) == 0
    for raw, cb, out, t, dec in zip(raws, cbs, outs, tot, decs):
        ref = oracle.encode_codebook(0, raw, cb)
        assert t == ref.size
        assert np.array_equal(out[:t].cpu().numpy(), ref)
        assert np.array_equal(raw_of(dec), raw)


def test_reuse_escapes_beyond_capacity_are_reported():
    """A codebook that misses every exponent: all n elements escape.  With only
    the smallest stream's room the call records SZ_ERR_BUFFER_TOO_SMALL."""
    m = sz()
    n = 3 * 4096 + 10
    raw = np.full(n, 0x3F80, dtype="<u2").view(np.uint8)
    cb = np.arange(15, dtype=np.uint8)                      # exponent 127 is not in it
    cap = m.sz_stream_bytes(0, n, 0)
    st, total, out = reuse_encode(0, raw, cb, cap=cap)
    assert st == m.SZ_ERR_BUFFER_TOO_SMALL
    assert total == m.sz_stream_bytes(0, n, n)
    st, total, out = reuse_encode(0, raw, cb)
    assert st == 0
    ref = oracle.encode_codebook(0, raw, cb)
    assert np.array_equal(out[:total], ref) and fieldcodec.parse(ref)["E"] == n


def test_reuse_refuses_invalid_codebooks():
    m = sz()
    raw = oracle_pins._kvlike(np.random.default_rng(1), 10000, 1)
    good = own_codebook(raw, 1)
    dup = good.copy()
    dup[4] = dup[3]
    big = good.copy()
    big[0] = 32                                             # outside E5M2's exponent range
    for cb in (dup, big):
        st, total, out = reuse_encode(1, raw, cb)
        assert st == m.SZ_ERR_PLAN_MISMATCH
        assert (out == POISON).all(), "nothing may be written"
    # the workspace is usable again after a reported error
    st, total, out = reuse_encode(1, raw, good)
    assert st == 0 and np.array_equal(out[:total], oracle.encode_codebook(1, raw, good))


def test_reuse_then_ordinary_encode_on_one_workspace():
    m = sz()
    rng = np.random.default_rng(8)
    raw = oracle_pins._kvlike(rng, 70000, 0)
    x = from_raw(raw, 0)
    ws = m.new_workspace(0, [70000])
    out = torch.zeros(m.sz_max_compressed_size(0, 70000), dtype=torch.uint8, device="cuda")
    cb = own_codebook(oracle_pins._kvlike(rng, 9000, 0), 0)
    for _ in range(2):
        m.sz_encode_reuse(0, plan_with_codebook([cb]), x, out, ws)
        assert m.sz_last_device_status(ws) == 0
        plan = m.new_plans(1)
        m.sz_plan(0, x, ws, plan)
        m.sz_encode(0, plan, x, out, ws)
        assert m.sz_last_device_status(ws) == 0
        ref = oracle.encode(0, raw)
        assert np.array_equal(out[: ref.size].cpu().numpy(), ref)


def test_batch_encode_reuse():
    """Batch.encode_reuse with the batch's own earlier plans and with given codebooks."""
    m = sz()
    rng = np.random.default_rng(12)
    sizes = [4096 * 9 + 1, 0, 5000]
    raws = [oracle_pins._kvlike(rng, n, 1) for n in sizes]
    xs = [from_raw(r, 1) for r in raws]
    ws = m.new_workspace(1, sizes)
    plans = m.new_plans(len(xs))
    outs = [torch.zeros(m.sz_max_compressed_size(1, n), dtype=torch.uint8, device="cuda") for n in sizes]
    decs = [torch.empty_like(x) for x in xs]
    b = m.Batch(1, xs, outs, ws, plans, decs=decs)
    b.plan()
    b.encode_reuse()
    b.decode()
    assert m.sz_last_device_status(ws) == 0
    for raw, out, dec in zip(raws, outs, decs):
        ref = oracle.encode(1, raw)
        assert np.array_equal(out[: ref.size].cpu().numpy(), ref)
        assert np.array_equal(raw_of(dec), raw)
    cb = own_codebook(raws[2], 1)
    totals = torch.zeros(3, dtype=torch.int64, device="cuda")
    b.encode_reuse(plan_with_codebook([cb] * 3), totals=totals)
    assert m.sz_last_device_status(ws) == 0
    for raw, out, t in zip(raws, outs, totals.cpu().tolist()):
        assert np.array_equal(out[:t].cpu().numpy(), oracle.encode_codebook(1, raw, cb))


@pytest.mark.slow
def test_reuse_full_size_qwen3_32b_layer():
    """One Qwen3-32B layer (2 x 134M elements) encoded with layer 0's codebooks."""
    m = sz()
    cfg = kvgen.CONFIGS["qwen3-32b"]
    cbs = [own_codebook(raw_of(kvgen.kv_tensor(cfg, 0, kv)), 0) for kv in (0, 1)]
    xs = [kvgen.kv_tensor(cfg, 31, kv) for kv in (0, 1)]
    raws = [raw_of(x) for x in xs]
    dxs = [x.cuda() for x in xs]
    ns = [x.numel() for x in xs]
    ws = m.new_workspace(0, ns)
    outs = [torch.zeros(m.sz_max_compressed_size(0, n), dtype=torch.uint8, device="cuda") for n in ns]
    totals = torch.zeros(2, dtype=torch.int64, device="cuda")
    m.sz_encode_reuse_batched(0, plan_with_codebook(cbs), dxs, outs, ws, totals=totals)
    assert m.sz_last_device_status(ws) == 0
    for raw, cb, out, t in zip(raws, cbs, outs, totals.cpu().tolist()):
        ref = oracle.encode_codebook(0, raw, cb)
        assert t == ref.size and np.array_equal(out[:t].cpu().numpy(), ref)
