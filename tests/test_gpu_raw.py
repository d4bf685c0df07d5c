"""Raw blocks on the GPU (header flag SZ_FLAG_RAW_BLOCKS): streams byte for byte
equal to the oracle's with raw blocks allowed, decoded bitwise, for blocks at,
below and above the threshold, uniform random bits (every block raw), mixed
streams, partial last blocks, batches mixing flagged and plain plans, reused
codebooks and paged tensors.

Inputs are made on the host; expected streams come from the oracle only.
"""
import numpy as np
import pytest
import torch

import fieldcodec
import oracle
import oracle_pins
from gpu_helpers import POISON, from_raw, raw_of, sz

pytestmark = pytest.mark.gpu


def es(dtype):
    return 2 if dtype == 0 else 1


def gpu_encode_raw(dtype, raw, cap=None):
    """Plan, set the raw-blocks flag, encode one tensor; returns (status, plan, stream)."""
    m = sz()
    x = from_raw(raw, dtype)
    n = m.numel_of(x, dtype)
    ws = m.new_workspace(dtype, [n])
    plan = m.new_plans(1)
    m.sz_plan(dtype, x, ws, plan)
    m.sz_plan_set_flags(plan, m.SZ_FLAG_RAW_BLOCKS)
    upper = m.sz_compressed_size(plan)
    cap = upper if cap is None else cap
    out = torch.full((max(cap, 1),), POISON, dtype=torch.uint8, device="cuda")[:cap]
    m.sz_encode(dtype, plan, x, out, ws)
    st = m.sz_last_device_status(ws)
    h = out.cpu().numpy()
    total = int(h[40:48].view(np.uint64)[0]) if h.size >= 48 else 0
    return st, plan.cpu().numpy().reshape(-1), h[:total]


def decode_on_gpu(dtype, stream, n):
    m = sz()
    comp = torch.from_numpy(np.ascontiguousarray(stream).copy()).cuda()
    out = torch.full((max(n, 1) * es(dtype),), POISON, dtype=torch.uint8, device="cuda")[: n * es(dtype)]
    ws = m.new_workspace(dtype, [n])
    m.sz_decode(dtype, comp, out, ws)
    assert m.sz_last_device_status(ws) == 0
    return out.cpu().numpy()


def check(dtype, raw):
    n = raw.size // es(dtype)
    ref = oracle.encode(dtype, raw, raw_blocks=True)
    st, plan, stream = gpu_encode_raw(dtype, raw)
    assert st == 0, sz().sz_status_string(st)
    # the plan is the ordinary plan with the flag set; its E and total are upper bounds
    plain = oracle.encode(dtype, raw)
    expect_plan = plain[:64].copy()
    expect_plan[39] = 1
    assert np.array_equal(plan, expect_plan)
    assert stream.size == ref.size, (stream.size, ref.size)
    diff = np.nonzero(stream != ref)[0]
    assert diff.size == 0, ("stream differs", int(diff[0]), int(stream[diff[0]]), int(ref[diff[0]]))
    assert np.array_equal(decode_on_gpu(dtype, stream, n), raw)
    return ref


def uniform(rng, n, dtype):
    return rng.integers(0, 256, n * es(dtype)).astype(np.uint8)


@pytest.mark.parametrize("dtype", [0, 1])
@pytest.mark.parametrize("n", [1, 2, 17, 4095, 4096, 4097, 3 * 4096 + 1001, 37 * 4096 + 5, 1 << 20])
def test_uniform_bits_every_block_raw(dtype, n):
    rng = np.random.default_rng(n * 3 + dtype)
    raw = uniform(rng, n, dtype)
    ref = check(dtype, raw)
    f = fieldcodec.parse(ref)
    if n >= 64:
        assert f["E"] == sum(fieldcodec.raw_block_bytes(dtype, m) for m in fieldcodec.block_sizes(n))


@pytest.mark.parametrize("dtype", [0, 1])
def test_threshold(dtype):
    rng = np.random.default_rng(5 + dtype)
    K = 2048 if dtype == 0 else 512
    for escapes in (K - 1, K, K + 1):
        blk = oracle_pins._threshold_block(rng, dtype, escapes)
        # the block alone, and between coded blocks
        check(dtype, blk)
        check(dtype, np.concatenate([oracle_pins._kvlike(rng, 4096, dtype), blk,
                                     oracle_pins._kvlike(rng, 5000, dtype)]))


@pytest.mark.parametrize("dtype", [0, 1])
def test_mixed_blocks(dtype):
    rng = np.random.default_rng(11 + dtype)
    for pattern in ("kv,rand,kv,rand", "rand,kv,kv,kv,kv,kv,kv,kv,kv,rand", "kv,kv,kv,kv,kv,kv,kv,kv,kv,kv,kv,rand"):
        parts = [oracle_pins._kvlike(rng, 4096, dtype) if p == "kv" else uniform(rng, 4096, dtype)
                 for p in pattern.split(",")]
        parts.append(uniform(rng, 777, dtype))  # a partial last block, raw
        check(dtype, np.concatenate(parts))


@pytest.mark.parametrize("dtype", [0, 1])
def test_no_raw_block_is_the_plain_stream(dtype):
    rng = np.random.default_rng(21 + dtype)
    raw = oracle_pins._kvlike(rng, 200000, dtype)
    ref = check(dtype, raw)
    plain = oracle.encode(dtype, raw)
    plain[39] = 1
    assert np.array_equal(ref, plain)


def test_batch_mixes_flagged_and_plain_plans():
    m = sz()
    rng = np.random.default_rng(31)
    for dtype in (0, 1):
        raws = [uniform(rng, 50000, dtype), oracle_pins._kvlike(rng, 60000, dtype),
                uniform(rng, 4097, dtype), oracle_pins._kvlike(rng, 1, dtype)]
        flags = [1, 1, 0, 1]
        xs = [from_raw(r, dtype) for r in raws]
        ns = [m.numel_of(x, dtype) for x in xs]
        ws = m.new_workspace(dtype, ns)
        plans = m.new_plans(len(xs))
        m.sz_plan_batched(dtype, xs, ws, plans)
        for t, fl in enumerate(flags):
            if fl:
                m.sz_plan_set_flags(plans[t:t + 1], m.SZ_FLAG_RAW_BLOCKS)
        outs = [torch.full((m.sz_max_compressed_size(dtype, n),), POISON, dtype=torch.uint8, device="cuda")
                for n in ns]
        m.sz_encode_batched(dtype, plans, xs, outs, ws)
        assert m.sz_last_device_status(ws) == 0
        decs = [torch.empty_like(x) for x in xs]
        m.sz_decode_batched(dtype, outs, decs, ws)
        assert m.sz_last_device_status(ws) == 0
        for raw, fl, o, d in zip(raws, flags, outs, decs):
            ref = oracle.encode(dtype, raw, raw_blocks=bool(fl))
            assert np.array_equal(o.cpu().numpy()[:ref.size], ref)
            assert np.array_equal(raw_of(d), raw)


def test_reused_codebook_with_raw_blocks():
    """A codebook that holds none of the data's exponents: every block raw."""
    m = sz()
    rng = np.random.default_rng(41)
    for dtype in (0, 1):
        for n in (5000, 3 * 4096, 70001):
            raw = oracle_pins._kvlike(rng, n, dtype)
            present = set(fieldcodec.exponents(raw, dtype).tolist())
            nbins = 256 if dtype == 0 else 32
            absent = [v for v in range(nbins) if v not in present]
            if len(absent) < 15:
                continue
            cb = np.array(absent[:15], dtype=np.uint8)
            for rb in (False, True):
                h = np.zeros((1, 64), dtype=np.uint8)
                h[0, 24:39] = cb
                h[0, 39] = 1 if rb else 0
                plan = torch.from_numpy(h).cuda()
                x = from_raw(raw, dtype)
                ws = m.new_workspace(dtype, [n])
                out = torch.full((m.sz_max_compressed_size(dtype, n),), POISON, dtype=torch.uint8, device="cuda")
                total = torch.zeros(1, dtype=torch.int64, device="cuda")
                m.sz_encode_reuse(dtype, plan, x, out, ws, total=total)
                assert m.sz_last_device_status(ws) == 0
                ref = oracle.encode_codebook(dtype, raw, cb, raw_blocks=rb)
                assert int(total.item()) == ref.size
                assert np.array_equal(out.cpu().numpy()[:ref.size], ref)
                assert np.array_equal(decode_on_gpu(dtype, ref, n), raw)


def test_paged_with_raw_blocks():
    m = sz()
    rng = np.random.default_rng(51)
    for dtype in (0, 1):
        page_elems, npages = 1024, 40
        eb = es(dtype)
        n = 37 * 1024 + 300
        parts = [oracle_pins._kvlike(rng, 8192, dtype), uniform(rng, 8192, dtype),
                 oracle_pins._kvlike(rng, 12288, dtype), uniform(rng, n - 28672, dtype)]
        raw = np.concatenate(parts)
        need = -(-n // page_elems)
        ids = rng.permutation(npages)[:need].astype(np.int32)
        pool = torch.zeros(npages * page_elems * eb, dtype=torch.uint8, device="cuda")
        host_pool = np.zeros(npages * page_elems * eb, dtype=np.uint8)
        for i, pid in enumerate(ids):
            chunk = raw[i * page_elems * eb:(i + 1) * page_elems * eb]
            host_pool[pid * page_elems * eb: pid * page_elems * eb + chunk.size] = chunk
        pool.copy_(torch.from_numpy(host_pool))
        pages = torch.from_numpy(ids).cuda()
        src = m.paged(dtype, pool, pages, page_elems)
        ws = m.new_workspace(dtype, [n])
        plans = m.new_plans(1)
        m.sz_plan_paged_batched(dtype, [src], [n], ws, plans)
        m.sz_plan_set_flags(plans, m.SZ_FLAG_RAW_BLOCKS)
        out = torch.full((m.sz_max_compressed_size(dtype, n),), POISON, dtype=torch.uint8, device="cuda")
        m.sz_encode_paged_batched(dtype, plans, [src], [n], [out], ws)
        assert m.sz_last_device_status(ws) == 0
        ref = oracle.encode(dtype, raw, raw_blocks=True)
        assert np.array_equal(out.cpu().numpy()[:ref.size], ref)
        # decode into a second pool with the same page table
        pool2 = torch.full_like(pool, POISON)
        dst = m.paged(dtype, pool2, pages, page_elems)
        m.sz_decode_paged_batched(dtype, [out], [dst], [n], ws)
        assert m.sz_last_device_status(ws) == 0
        back = pool2.cpu().numpy()
        got = np.concatenate([back[pid * page_elems * eb: pid * page_elems * eb + page_elems * eb]
                              for pid in ids])[: n * eb]
        assert np.array_equal(got, raw)


def test_set_flags_rejects_unknown_flags():
    m = sz()
    plans = m.new_plans(2)
    with pytest.raises(m.SplitZipError):
        m.sz_plan_set_flags(plans, 2)


@pytest.mark.slow
def test_uniform_bits_full_size():
    """2^27 uniform random BF16 elements (256 MiB): every block raw; the stream is
    at most the raw bytes plus header, table and padding."""
    rng = np.random.default_rng(61)
    n = 1 << 27
    raw = uniform(rng, n, 0)
    ref = check(0, raw)
    assert ref.size <= raw.size + fieldcodec.align256(64 + 4 * (n // 4096 + 1)) + 512


@pytest.mark.parametrize("dtype", [0, 1])
def test_corrupt_raw_stream_is_reported(dtype):
    """A flagged stream whose offsets table no longer marks its raw blocks is
    reported as corrupt (the decode stays inside the stream and the output)."""
    m = sz()
    rng = np.random.default_rng(71 + dtype)
    n = 3 * 4096 + 100
    raw = uniform(rng, n, dtype)
    st, _, stream = gpu_encode_raw(dtype, raw)
    assert st == 0
    for what in ("count_plus_one", "flag_cleared"):
        bad = stream.copy()
        if what == "count_plus_one":
            bad[68] ^= 1  # offsets[1]: block 0's count is no longer its raw size
        else:
            bad[39] = 0   # without the flag the raw blocks read as coded ones
        comp = torch.from_numpy(bad).cuda()
        out = torch.empty(n * es(dtype), dtype=torch.uint8, device="cuda")
        ws = m.new_workspace(dtype, [n])
        m.sz_decode(dtype, comp, out, ws)
        assert m.sz_last_device_status(ws) == m.SZ_ERR_CORRUPT_STREAM, what
