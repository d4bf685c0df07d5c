"""Paged tensors on the GPU: plan, encode and decode of tensors held in the pages of a
page pool (a page table of int32 ids, as paged KV caches keep them).

The stream of a paged tensor is the stream of its elements in order, so the
oracle encodes the tensor gathered on the host (a numpy gather, a library
primitive) and the GPU's paged calls must produce the same bytes; decode must
write exactly the tensor's bytes into its pages and nothing else.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle_pins
from gpu_helpers import sz

pytestmark = pytest.mark.gpu

POISON = 0xA5


def build_pool(rng, dtype, raws, page_elems, gap_bytes, spare_pages=3):
    """Scatter the raw tensors into one pool in a random page order.  Returns
    (pool tensor, [page-id tensors], page_bytes, pool_pages)."""
    eb = 2 if dtype == 0 else 1
    page_bytes = page_elems * eb + gap_bytes
    counts = [-(-(r.size // eb) // page_elems) for r in raws]
    pool_pages = sum(counts) + spare_pages
    order = rng.permutation(pool_pages)
    pool = np.full(pool_pages * page_bytes, POISON, dtype=np.uint8)
    tables, k = [], 0
    for r, c in zip(raws, counts):
        ids = order[k: k + c].astype(np.int32)
        k += c
        for j, pid in enumerate(ids):
            piece = r[j * page_elems * eb: (j + 1) * page_elems * eb]
            pool[pid * page_bytes: pid * page_bytes + piece.size] = piece
        tables.append(ids)
    return pool, tables, page_bytes, pool_pages


def gather(pool, ids, n, dtype, page_elems, page_bytes):
    eb = 2 if dtype == 0 else 1
    out = np.concatenate([pool[pid * page_bytes: pid * page_bytes + page_elems * eb] for pid in ids]) \
        if len(ids) else np.zeros(0, np.uint8)
    return out[: n * eb]


@pytest.mark.parametrize("dtype", [0, 1])
@pytest.mark.parametrize("page_elems,gap", [(1024, 0), (16384, 0), (5 * 1024, 512)])
def test_paged_round_trip_matches_oracle(dtype, page_elems, gap):
    m = sz()
    rng = np.random.default_rng(page_elems + gap + dtype)
    sizes = [page_elems * 7 + 1000, 3 * 4096 + 5, 1, 0, 40000]
    raws = [oracle_pins._kvlike(rng, n, dtype) for n in sizes]
    pool_h, tables_h, page_bytes, pool_pages = build_pool(rng, dtype, raws, page_elems, gap)
    pool = torch.from_numpy(pool_h).cuda()
    tables = [torch.from_numpy(t).cuda() if t.size else torch.zeros(1, dtype=torch.int32, device="cuda")
              for t in tables_h]
    srcs = [m.paged(dtype, pool, t, page_elems, page_bytes, pool_pages) for t in tables]
    ws = m.new_workspace(dtype, sizes)
    plans = m.new_plans(len(sizes))
    m.sz_plan_paged_batched(dtype, srcs, sizes, ws, plans)
    outs = [torch.full((m.sz_max_compressed_size(dtype, n),), POISON, dtype=torch.uint8, device="cuda")
            for n in sizes]
    m.sz_encode_paged_batched(dtype, plans, srcs, sizes, outs, ws)
    assert m.sz_last_device_status(ws) == 0
    totals = m.sz_compressed_sizes(plans)
    for raw, out, tot in zip(raws, outs, totals):
        ref = oracle.encode(dtype, raw)
        assert tot == ref.size
        assert np.array_equal(out[:tot].cpu().numpy(), ref)
    # decode into another pool, in another page order; bytes outside the tensors stay poisoned
    pool2_h, tables2_h, _, _ = build_pool(rng, dtype, [np.zeros_like(r) for r in raws], page_elems, gap)
    pool2_h[:] = POISON
    pool2 = torch.from_numpy(pool2_h).cuda()
    tables2 = [torch.from_numpy(t).cuda() if t.size else torch.zeros(1, dtype=torch.int32, device="cuda")
               for t in tables2_h]
    dsts = [m.paged(dtype, pool2, t, page_elems, page_bytes, pool_pages) for t in tables2]
    m.sz_decode_paged_batched(dtype, [o[:t] for o, t in zip(outs, totals)], dsts, sizes, ws)
    assert m.sz_last_device_status(ws) == 0
    got = pool2.cpu().numpy()
    written = np.zeros(got.size, dtype=bool)
    eb = 2 if dtype == 0 else 1
    for raw, ids, n in zip(raws, tables2_h, sizes):
        assert np.array_equal(gather(got, ids, n, dtype, page_elems, page_bytes), raw)
        for j, pid in enumerate(ids):
            k = min(page_elems, n - j * page_elems) * eb
            written[pid * page_bytes: pid * page_bytes + k] = True
    assert (got[~written] == POISON).all(), "decode wrote outside the tensors' elements"


def test_paged_matches_contiguous_on_a_kv_layer():
    """A Llama-3-8B-shaped K tensor in vLLM-style pages (16 tokens x 8 heads x 128)."""
    import kvgen
    from gpu_helpers import gpu_encode, raw_of
    m = sz()
    x = kvgen.kv_tensor(kvgen.CONFIGS["llama3-8b"], 3, 0)
    raw = raw_of(x)
    n = x.numel()
    page_elems = 16 * 8 * 128
    rng = np.random.default_rng(4)
    pool_h, tables_h, page_bytes, pool_pages = build_pool(rng, 0, [raw], page_elems, 0)
    pool = torch.from_numpy(pool_h).cuda()
    src = m.paged(0, pool, torch.from_numpy(tables_h[0]).cuda(), page_elems)
    ws = m.new_workspace(0, [n])
    plans = m.new_plans(1)
    m.sz_plan_paged_batched(0, [src], [n], ws, plans)
    out = torch.zeros(m.sz_max_compressed_size(0, n), dtype=torch.uint8, device="cuda")
    m.sz_encode_paged_batched(0, plans, [src], [n], [out], ws)
    assert m.sz_last_device_status(ws) == 0
    _, ref = gpu_encode(0, x.cuda())
    assert np.array_equal(out[: ref.size].cpu().numpy(), ref)


def test_page_ids_outside_the_pool_are_reported():
    m = sz()
    rng = np.random.default_rng(9)
    n = 4096 * 6
    raw = oracle_pins._kvlike(rng, n, 0)
    pool_h, tables_h, page_bytes, pool_pages = build_pool(rng, 0, [raw], 4096, 0)
    pool = torch.from_numpy(pool_h).cuda()
    ws = m.new_workspace(0, [n])
    plans = m.new_plans(1)
    for bad_id in (pool_pages, -1):
        ids = tables_h[0].copy()
        ids[2] = bad_id
        src = m.paged(0, pool, torch.from_numpy(ids).cuda(), 4096, page_bytes, pool_pages)
        m.sz_plan_paged_batched(0, [src], [n], ws, plans)
        assert m.sz_last_device_status(ws) == m.SZ_ERR_INVALID_ARG
        m.sz_workspace_init(ws)
        good = m.paged(0, pool, torch.from_numpy(tables_h[0]).cuda(), 4096, page_bytes, pool_pages)
        m.sz_plan_paged_batched(0, [good], [n], ws, plans)
        out = torch.zeros(m.sz_max_compressed_size(0, n), dtype=torch.uint8, device="cuda")
        m.sz_encode_paged_batched(0, plans, [src], [n], [out], ws)
        assert m.sz_last_device_status(ws) == m.SZ_ERR_INVALID_ARG
        m.sz_workspace_init(ws)
        # decode into pages through the bad table: the bad page is not written
        m.sz_encode_paged_batched(0, plans, [good], [n], [out], ws)
        assert m.sz_last_device_status(ws) == 0
        tot = m.sz_compressed_size(plans)
        before = pool.clone()
        m.sz_decode_paged_batched(0, [out[:tot]], [src], [n], ws)
        assert m.sz_last_device_status(ws) == m.SZ_ERR_INVALID_ARG
        m.sz_workspace_init(ws)
        after = pool.cpu().numpy()
        assert np.array_equal(after, before.cpu().numpy()), "decode rewrote the same bytes elsewhere"


def test_paged_host_checks():
    m = sz()
    pool = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    ids = torch.zeros(4, dtype=torch.int32, device="cuda")
    ws = m.new_workspace(0, [4096])
    plans = m.new_plans(1)
    for kw in (dict(page_elems=1000), dict(page_elems=1024, page_bytes=2 * 1024 + 8),
               dict(page_elems=1024, page_bytes=1024), dict(page_elems=(1 << 18) + 1024)):
        d = m.paged(0, pool, ids, **kw)
        with pytest.raises(m.SplitZipError) as e:
            m.sz_plan_paged_batched(0, [d], [4096], ws, plans)
        assert e.value.status == m.SZ_ERR_INVALID_ARG


def test_paged_batch_and_reuse():
    """Batch over paged inputs and outputs, with codebook reuse from paged inputs."""
    m = sz()
    rng = np.random.default_rng(21)
    sizes = [16384 * 3 + 77, 9000]
    raws = [oracle_pins._kvlike(rng, n, 1) for n in sizes]
    pool_h, tables_h, page_bytes, pool_pages = build_pool(rng, 1, raws, 16384, 0)
    pool = torch.from_numpy(pool_h).cuda()
    srcs = [m.paged(1, pool, torch.from_numpy(t).cuda(), 16384, page_bytes, pool_pages) for t in tables_h]
    dpool = torch.full_like(pool, POISON)
    dsts = [m.paged(1, dpool, torch.from_numpy(t).cuda(), 16384, page_bytes, pool_pages) for t in tables_h]
    ws = m.new_workspace(1, sizes)
    plans = m.new_plans(2)
    outs = [torch.zeros(m.sz_max_compressed_size(1, n), dtype=torch.uint8, device="cuda") for n in sizes]
    b = m.Batch(1, None, outs, ws, plans, src_pages=srcs, dst_pages=dsts, n=sizes)
    b.plan()
    b.encode()
    b.decode()
    assert m.sz_last_device_status(ws) == 0
    got = dpool.cpu().numpy()
    for raw, ids, n, out in zip(raws, tables_h, sizes, outs):
        assert np.array_equal(gather(got, ids, n, 1, 16384, page_bytes), raw)
        ref = oracle.encode(1, raw)
        assert np.array_equal(out[: ref.size].cpu().numpy(), ref)
    cb = oracle.codebook(1, oracle.histogram(1, raws[1]))
    h = np.zeros((2, 64), dtype=np.uint8)
    h[:, 24:39] = cb
    totals = torch.zeros(2, dtype=torch.int64, device="cuda")
    b.encode_reuse(torch.from_numpy(h).cuda(), totals=totals)
    assert m.sz_last_device_status(ws) == 0
    for raw, out, t in zip(raws, outs, totals.cpu().tolist()):
        assert np.array_equal(out[:t].cpu().numpy(), oracle.encode_codebook(1, raw, cb))


def test_largest_pages():
    """Pages of 2^18 elements (the limit): the histogram's per-lane counts stay in range."""
    m = sz()
    rng = np.random.default_rng(31)
    pe = 1 << 18
    sizes = [3 * pe + 4100, 70000]
    raws = [oracle_pins._kvlike(rng, n, 0) for n in sizes]
    # one exponent dominates, so single counters grow as fast as possible
    for r in raws:
        w = r.view("<u2")
        w[rng.random(w.size) < 0.9] = 0x3F80
    pool_h, tables_h, page_bytes, pool_pages = build_pool(rng, 0, raws, pe, 0)
    pool = torch.from_numpy(pool_h).cuda()
    tables = [torch.from_numpy(t).cuda() for t in tables_h]
    srcs = [m.paged(0, pool, t, pe, page_bytes, pool_pages) for t in tables]
    ws = m.new_workspace(0, sizes)
    plans = m.new_plans(2)
    m.sz_plan_paged_batched(0, srcs, sizes, ws, plans)
    outs = [torch.zeros(m.sz_max_compressed_size(0, n), dtype=torch.uint8, device="cuda") for n in sizes]
    m.sz_encode_paged_batched(0, plans, srcs, sizes, outs, ws)
    assert m.sz_last_device_status(ws) == 0
    for raw, out in zip(raws, outs):
        ref = oracle.encode(0, raw)
        assert np.array_equal(out[: ref.size].cpu().numpy(), ref)
