"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle, bit for bit.

Small and ragged sizes span several 4096-element tiles and a partial last tile;
the plan (= stream header), the whole compressed stream and the decoded tensor
must equal the oracle's exactly (no tolerance: every step is integer work).
"""
import numpy as np
import pytest
import torch

import kvgen
import oracle
import oracle_pins
from gpu_helpers import check_parity, from_raw, gpu_decode, gpu_encode, raw_of, sz

pytestmark = pytest.mark.gpu

RAGGED = (1, 2, 3, 7, 8, 9, 15, 16, 17, 255, 256, 257, 4095, 4096, 4097, 8191, 8193, 12289,
          65536 + 5, (1 << 20) + 3)


@pytest.mark.parametrize("kv", [0, 1], ids=["K", "V"])
def test_phi2_layer(kv):
    x = kvgen.kv_tensor(kvgen.CONFIGS["phi2"], 0, kv)
    check_parity(0, raw_of(x))


@pytest.mark.parametrize("dtype", [0, 1], ids=["bf16", "e5m2"])
@pytest.mark.parametrize("n", RAGGED)
def test_ragged_kvlike(dtype, n):
    rng = np.random.default_rng(n)
    check_parity(dtype, oracle_pins._kvlike(rng, n, dtype))


@pytest.mark.parametrize("dtype", [0, 1], ids=["bf16", "e5m2"])
@pytest.mark.parametrize("n", (1, 17, 4097, 50001))
def test_ragged_uniform_bits(dtype, n):
    rng = np.random.default_rng(100 + n)
    check_parity(dtype, rng.integers(0, 256, n * (2 if dtype == 0 else 1)).astype(np.uint8))


def test_exhaustive_bf16_patterns():
    allp = np.arange(65536, dtype=np.uint32).astype("<u2")
    rng = np.random.default_rng(0)
    for x in (allp, allp[rng.permutation(allp.size)], np.repeat(allp, 3)):
        check_parity(0, x.view(np.uint8))


def test_exhaustive_e5m2_patterns():
    allp = np.arange(256, dtype=np.uint32).astype(np.uint8)
    rng = np.random.default_rng(0)
    for x in (allp, allp[rng.permutation(allp.size)], np.repeat(allp, 17), np.tile(allp, 4099)):
        check_parity(1, x)


def test_special_cases():
    check_parity(0, np.zeros(2 * 10000, np.uint8))                              # all +0.0
    check_parity(0, np.full(9999, 0x8000, "<u2").view(np.uint8))                # all -0.0
    check_parity(1, np.zeros(10001, np.uint8))
    e = np.tile(np.arange(100, 116), 1024)                                      # 16 equal exponents
    np.random.default_rng(1).shuffle(e)
    check_parity(0, (e << 7).astype("<u2").view(np.uint8))
    rng = np.random.default_rng(2)                                              # <= 15 distinct
    vals = rng.choice(256, size=9, replace=False)
    check_parity(0, ((rng.choice(vals, 20000) << 7) | rng.integers(0, 128, 20000)).astype("<u2").view(np.uint8))


def test_golden_streams_on_gpu():
    m = sz()
    for path in oracle_pins.golden_files():
        dtype, raw, expect = oracle_pins.load_golden(path)
        cb = oracle_pins.golden_codebook(path)
        flags = oracle_pins.golden_flags(path)
        if cb is None:
            assert flags == 0
            plan, stream = gpu_encode(dtype, from_raw(raw, dtype))
        else:  # a codebook-reuse fixture: encode with the given codebook (and flags)
            x = from_raw(raw, dtype)
            n = m.numel_of(x, dtype)
            ws = m.new_workspace(dtype, [n])
            h = np.zeros((1, 64), dtype=np.uint8)
            h[0, 24:39] = cb
            h[0, 39] = flags
            out = torch.full((m.sz_max_compressed_size(dtype, n),), 0xA5, dtype=torch.uint8, device="cuda")
            m.sz_encode_reuse(dtype, torch.from_numpy(h).cuda(), x, out, ws)
            assert m.sz_last_device_status(ws) == 0
            stream = out[: expect.size].cpu().numpy()
        assert np.array_equal(stream, expect), path
        n = raw.size // (2 if dtype == 0 else 1)
        assert np.array_equal(gpu_decode(dtype, expect, n), raw), path


def test_empty_tensor():
    m = sz()
    for dtype in (0, 1):
        ref = oracle.encode(dtype, np.zeros(0, np.uint8))
        x = torch.empty(0, dtype=torch.bfloat16 if dtype == 0 else torch.float8_e5m2, device="cuda")
        plan, stream = gpu_encode(dtype, x)
        assert np.array_equal(stream, ref) and stream.size == 256


def test_batched_matches_single():
    """One launch per kernel over tensors of mixed sizes (empty ones included)."""
    m = sz()
    rng = np.random.default_rng(9)
    for dtype in (0, 1):
        sizes = [4096 * 3 + 17, 0, 1, 65536, 100003, 0, 4096, 777]
        raws = [oracle_pins._kvlike(rng, n, dtype) for n in sizes]
        xs = [from_raw(r, dtype) for r in raws]
        ws = m.new_workspace(dtype, sizes)
        plans = m.new_plans(len(xs))
        m.sz_plan_batched(dtype, xs, ws, plans)
        totals = m.sz_compressed_sizes(plans)
        outs = [torch.full((m.sz_max_compressed_size(dtype, n),), 0xA5, dtype=torch.uint8, device="cuda")
                for n in sizes]
        m.sz_encode_batched(dtype, plans, xs, outs, ws)
        decs = [torch.full_like(x.view(torch.uint8), 0xA5) for x in xs]
        m.sz_decode_batched(dtype, [o[:t] for o, t in zip(outs, totals)],
                            [d.view(x.dtype) for d, x in zip(decs, xs)], ws)
        assert m.sz_last_device_status(ws) == 0
        for raw, out, tot, dec in zip(raws, outs, totals, decs):
            ref = oracle.encode(dtype, raw)
            assert tot == ref.size
            assert np.array_equal(out[:tot].cpu().numpy(), ref)
            assert np.array_equal(dec.cpu().numpy(), raw)


def test_workspace_reuse_is_deterministic():
    m = sz()
    x = kvgen.kv_tensor(kvgen.CONFIGS["phi2"], 0, 1).cuda()
    ws = m.new_workspace(0, [x.numel()])
    first = gpu_encode(0, x, ws)[1]
    for _ in range(3):
        assert np.array_equal(gpu_encode(0, x, ws)[1], first)
    # a different batch through the same workspace, then the single tensor again
    y = x.view(-1)[: 4096 * 5]
    gpu_encode(0, y, ws)
    assert np.array_equal(gpu_encode(0, x, ws)[1], first)


def test_batched_decode_claims_every_block_and_resets():
    """Decode hands blocks out from per-tensor counters in the workspace: with
    more tensors than one warp scans at a time (empty and one-element tensors
    among them), every block is decoded exactly right, the counters are zero
    again after each call, and plan can reuse the workspace straight away."""
    m = sz()
    rng = np.random.default_rng(21)
    for dtype in (0, 1):
        sizes = [int(s) for s in rng.choice([0, 1, 4095, 4096, 4097, 3 * 4096 + 5, 9 * 4096, 40000], 70)]
        raws = [oracle_pins._kvlike(rng, n, dtype) for n in sizes]
        xs = [from_raw(r, dtype) for r in raws]
        ws = m.new_workspace(dtype, sizes)
        plans = m.new_plans(len(xs))
        m.sz_plan_batched(dtype, xs, ws, plans)
        totals = m.sz_compressed_sizes(plans)
        outs = [torch.zeros(m.sz_max_compressed_size(dtype, n), dtype=torch.uint8, device="cuda") for n in sizes]
        m.sz_encode_batched(dtype, plans, xs, outs, ws)
        assert m.sz_last_device_status(ws) == 0
        for rep in range(3):
            decs = [torch.full_like(x.view(torch.uint8), 0xA5) for x in xs]
            m.sz_decode_batched(dtype, [o[:t] for o, t in zip(outs, totals)],
                                [d.view(x.dtype) for d, x in zip(decs, xs)], ws)
            assert m.sz_last_device_status(ws) == 0
            words = ws.view(torch.int32)
            assert words[5].item() == 0
            assert not words[64: 64 + 256 * len(sizes)].any().item(), "claim counters left set"
            for raw, dec in zip(raws, decs):
                assert np.array_equal(dec.cpu().numpy(), raw)
        plans2 = m.new_plans(len(xs))
        m.sz_plan_batched(dtype, xs, ws, plans2)
        assert torch.equal(plans2, plans)


def test_prepared_batch_matches_functional_calls():
    """Batch marshals the pointer arrays once; its calls give the same streams and
    round trip as the per-call functions."""
    m = sz()
    rng = np.random.default_rng(33)
    for dtype in (0, 1):
        sizes = [4096 * 5 + 3, 0, 70000, 4096]
        raws = [oracle_pins._kvlike(rng, n, dtype) for n in sizes]
        xs = [from_raw(r, dtype) for r in raws]
        ws = m.new_workspace(dtype, sizes)
        plans = m.new_plans(len(xs))
        outs = [torch.zeros(m.sz_max_compressed_size(dtype, n), dtype=torch.uint8, device="cuda") for n in sizes]
        decs = [torch.full_like(x.view(torch.uint8), 0xA5).view(x.dtype) for x in xs]
        b = m.Batch(dtype, xs, outs, ws, plans, decs=decs)
        for _ in range(2):
            b.plan()
            b.encode()
            b.decode()
            assert m.sz_last_device_status(ws) == 0
        totals = m.sz_compressed_sizes(plans)
        for raw, out, tot, dec in zip(raws, outs, totals, decs):
            assert np.array_equal(out[:tot].cpu().numpy(), oracle.encode(dtype, raw))
            assert np.array_equal(dec.view(torch.uint8).cpu().numpy(), raw)
    with pytest.raises(ValueError):
        m.Batch(0, [torch.zeros(8, 8, dtype=torch.bfloat16, device="cuda").t()], [outs[0]], ws, plans)


def test_calls_capture_into_a_cuda_graph():
    """plan, encode and decode enqueue kernels only (no allocation, no
    synchronisation), so a step captures into a CUDA graph; replays on new data in
    the same buffers give the oracle's streams and exact round trips."""
    m = sz()
    rng = np.random.default_rng(41)
    for dtype in (0, 1):
        sizes = [4096 * 9 + 7, 70000, 0]
        raws = [oracle_pins._kvlike(rng, n, dtype) for n in sizes]
        xs = [from_raw(r, dtype) for r in raws]
        ws = m.new_workspace(dtype, sizes)
        plans = m.new_plans(len(xs))
        outs = [torch.zeros(m.sz_max_compressed_size(dtype, n), dtype=torch.uint8, device="cuda") for n in sizes]
        decs = [torch.empty_like(x) for x in xs]
        b = m.Batch(dtype, xs, outs, ws, plans, decs=decs)
        b.plan(); b.encode(); b.decode()            # first calls set each kernel up on the device
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s), torch.cuda.graph(graph, stream=s):
            b.plan(); b.encode(); b.decode()
        torch.cuda.current_stream().wait_stream(s)
        for rep in range(2):
            new = [oracle_pins._kvlike(rng, n, dtype) for n in sizes]
            for x, r in zip(xs, new):
                if r.size:
                    x.view(torch.uint8).copy_(torch.from_numpy(r).cuda())
            graph.replay()
            torch.cuda.synchronize()
            assert m.sz_last_device_status(ws) == 0
            totals = m.sz_compressed_sizes(plans)
            for r, out, tot, dec in zip(new, outs, totals, decs):
                ref = oracle.encode(dtype, r)
                assert tot == ref.size and np.array_equal(out[:tot].cpu().numpy(), ref)
                assert np.array_equal(dec.view(torch.uint8).cpu().numpy(), r)
        del graph


@pytest.mark.parametrize("per_lane", [1, 2, 3], ids=["one", "two", "three"])
@pytest.mark.parametrize("dtype", [0, 1], ids=["bf16", "e5m2"])
def test_escapes_per_lane_step(dtype, per_lane):
    """Every lane's share of every decode step (8 BF16 or 16 E5M2 consecutive
    elements) holds exactly `per_lane` escapes, at random places, so that each
    block has hundreds of escapes (ranks far past the 32 a warp holds in
    registers) and every step takes the one-, two- or three-or-more-escape path.
    Fifteen common exponents fill the rest; the escapes take rare ones."""
    rng = np.random.default_rng(31 * per_lane + dtype)
    le = 8 if dtype == 0 else 16
    n = 4096 * 5 + 3 * le + 5  # whole blocks, then a ragged tail
    common = np.arange(100, 115) if dtype == 0 else np.arange(5, 20)
    # many rare values, each less frequent than any common one, so that all escape
    rare = np.arange(40, 72) if dtype == 0 else np.setdiff1d(np.arange(32), common)
    e = rng.choice(common, n)
    for g in range(0, n - le + 1, le):
        pos = rng.choice(le, per_lane, replace=False)
        e[g + pos] = rng.choice(rare, per_lane)
    if dtype == 0:
        w = (rng.integers(0, 2, n) << 15) | (e << 7) | rng.integers(0, 128, n)
        raw = w.astype(np.uint16).view(np.uint8)
    else:
        w = (rng.integers(0, 2, n) << 7) | (e << 2) | rng.integers(0, 4, n)
        raw = w.astype(np.uint8)
    check_parity(dtype, raw)
