"""Benchmark of the exponent-split KV codec on B200.

One step = the whole hot path over one batch: plan (histogram + codebook),
encode and decode of every K and V tensor of the workload, one batched launch
per kernel (default workload: Llama-3-8B KV after an 8192-token prefill, 32
layers x {K, V} x [8192, 8, 128] bf16 = 1.07 GB).  Inputs are seeded synthetic
tensors resident in HBM; the batch (1.07 GB) is larger than L2 (126 MB), so no
flush is needed between steps.

Prints one JSON line.  `value` is raw input bytes per second through a full
round trip (plan + encode + decode); encode (plan + encode) and decode rates,
per-kernel roofline fractions and the compression ratio ride along.  With the
default workload the line also carries `configs`: the other KV workloads,
measured in the same run --

  qwen3-32b            64 layers x {K,V} x [131072, 8, 128] bf16 (34.4 GB),
                       generated on the device one layer at a time and coded
                       layer by layer (537 MB per call), L2 flushed before
                       each layer;
  qwen3-30b-a3b-e5m2   48 layers x {K,V} x [32768, 4, 128] FP8 E5M2, one batch;
  llama3-8b-per-layer  the Llama-3-8B KV coded layer by layer (33.5 MB per
                       call), 32 calls per step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload llama3-8b|qwen3-32b-layer|qwen3-30b-a3b-e5m2|stress-uniform-bf16]
                  [--mode batch|per_layer] [--reuse] [--paged TOKENS] [--raw-blocks]
                  [--transfer] [--no-graph] [--no-e2e] [--no-records] [--layers N]
                  [--kernel-reps R]

Timing: every figure comes from CUDA events on the launching stream.  The K
timed steps are the step captured once as a CUDA graph and replayed
(`ms_per_step`, `value`); `step_stats` adds the median over max(K, 50)
further replays.  Per-kernel figures come from each kernel's own graph (its
launches of one step), replayed max(K, R) times in step order: `ms` is the
mean, `ms_median` the median.  `e2e` repeats the step through the public API
from pinned host memory and back, pipelining the copies of consecutive steps
with the kernels.

`--impl reference` times the CPU oracle (plain single-threaded C, pinned to one
core) on a bounded sample of the same workload: the only reference
implementation there is.  For N > 1 (torchrun), every rank codes its own batch
of the same size (weak scaling: the tensors are independent, no data-path
collective); timing is the max over ranks.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import kvgen  # noqa: E402

METRIC = "encode/decode GB/s (raw bytes) on 1 B200, % of HBM roofline, compression ratio"
UNIT = "GB/s"


# ------------------------------------------------------------ host logic

def rank_layers(cfg_layers: int, rank: int, world: int):
    """Layers coded by one rank: every rank gets a full batch of its own layers
    (weak scaling).  Rank r uses layer indices r*L .. r*L + L - 1 of the seeded
    generator, so ranks never code the same tensor."""
    return list(range(rank * cfg_layers, (rank + 1) * cfg_layers))


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


WORKLOADS = {
    # name: (config, layers per step, description)
    "llama3-8b": ("llama3-8b", None, "Llama-3-8B KV, 8192-token prefill: 32 layers x {K,V} x [8192,8,128] bf16"),
    "qwen3-32b-layer": ("qwen3-32b", 1, "Qwen3-32B KV at 131072 tokens, one layer: {K,V} x [131072,8,128] bf16"),
    "qwen3-30b-a3b-e5m2": ("qwen3-30b-a3b-e5m2", None, "Qwen3-30B-A3B KV, FP8 E5M2: 48 layers x {K,V} x [32768,4,128]"),
    "stress-uniform-bf16": ("stress-uniform", 1, "escape stress, worst case: one flat bf16 tensor of 2^29 uniformly "
                                                "random 16-bit patterns (1 GiB)"),
}
STRESS_N = 1 << 29        # elements of the stress tensor (1 GiB of bf16)
STRESS_SAMPLE_N = 1 << 23  # elements of the CPU oracle's sample of it


def stress_seed(rank: int = 0) -> int:
    # the 1 GB uniform-bits case of the escape-stress family (seed 4_000_000 + case); ranks offset
    return 4_000_000 + kvgen.stress_case(2, len(kvgen.STRESS_RARE_PERCENT) - 1) + 1000 * rank


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


KERNEL_SOURCES = ("sz_common.cuh", "sz_plan.cu", "sz_encode.cu", "sz_decode.cu")


def _code_only(src: str) -> str:
    """C/CUDA source without comments and blank lines (comments do not change a kernel)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    lines = [re.sub(r"//.*", "", ln).rstrip() for ln in src.splitlines()]
    return "\n".join(ln for ln in lines if ln.strip())


# the sources each kernel's code comes from
KERNEL_FILES = {"plan_kernel": ("sz_common.cuh", "sz_plan.cu"),
                "encode_kernel": ("sz_common.cuh", "sz_encode.cu"),
                "decode_kernel": ("sz_common.cuh", "sz_decode.cu")}


def kernel_source_hash(kernel: str = None) -> str:
    """Hash of the device-code sources, comments left out: of all of them (which build
    a profile describes), or of one kernel's (whether its recorded traffic still
    applies).  Host-only files (the C-ABI layer, the header) do not change it."""
    import hashlib
    names = KERNEL_SOURCES if kernel is None else KERNEL_FILES[kernel]
    files = [os.path.join(ROOT, "fp8_kv_cache_exp_b200", "csrc", f) for f in names]
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded by ncu for this kernel source, or None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    src = kernel_source_hash(kernel)
    for line in lines:
        parts = line.split()
        if len(parts) == 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload \
                and parts[3] == src:
            return int(parts[2])
    return None


def gpu_uuid(device) -> str:
    """nvidia-smi id of a torch device (its UUID, whatever CUDA_VISIBLE_DEVICES says)."""
    u = str(torch.cuda.get_device_properties(device).uuid)
    return u if u.startswith("GPU-") else "GPU-" + u


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def head_start(ms: float = 2.0):
    """Keep the GPU busy for about `ms` so that the host enqueues the work that
    follows before the GPU reaches it (no host gap inside a measurement)."""
    torch.cuda._sleep(int(ms * 2e6))


def capture_graph(fn, stream, device):
    """fn() (calls that only enqueue kernels) captured once as a CUDA graph."""
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device=device)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap), torch.cuda.graph(g, stream=cap):
        fn()
    stream.wait_stream(cap)
    return g


def graph_part_times(parts: dict, reps: int, stream, device, warmup: int = 3) -> dict:
    """Each of `parts` (name -> fn enqueuing kernels) captured as its own CUDA
    graph; all of them replayed in order `reps` times with a CUDA event between
    consecutive graphs.  Returns name -> list of ms per replay."""
    graphs = {k: capture_graph(fn, stream, device) for k, fn in parts.items()}
    for _ in range(warmup):
        for g in graphs.values():
            g.replay()
    torch.cuda.synchronize()
    names = list(graphs)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(reps)]
    head_start()
    for r in range(reps):
        ev[r][0].record(stream)
        for i, k in enumerate(names):
            graphs[k].replay()
            ev[r][i + 1].record(stream)
    torch.cuda.synchronize()
    out = {k: [ev[r][i].elapsed_time(ev[r][i + 1]) for r in range(reps)] for i, k in enumerate(names)}
    del graphs
    return out


def kernel_figures(times_ms, nbytes: int, peak: float) -> dict:
    """Mean and median of a kernel's times and its algorithmic GB/s and fraction
    of peak (from the mean)."""
    ms = sum(times_ms) / len(times_ms)
    med = statistics.median(times_ms)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": ms, "ms_median": med, "gbs": gbs, "frac": gbs / peak,
            "frac_median": nbytes / (med * 1e-3) / 1e9 / peak}


def check_status(sz, workspaces, where: str):
    for w in workspaces:
        st = sz.sz_last_device_status(w)
        if st != 0:
            raise RuntimeError("device status (%s): %s" % (where, sz.sz_status_string(st)))


# ------------------------------------------------------------- our arm

class Workload:
    def __init__(self, name: str, rank: int, world: int, device, layers=None):
        cfg_name, layers_per_step, desc = WORKLOADS[name]
        self.name, self.desc = name, desc
        if cfg_name == "stress-uniform":
            self.cfg, self.dtype, self.esize, self.layers = None, 0, 2, [0]
            self.xs = [kvgen.stress_tensor(STRESS_N, None, stress_seed(rank), device=device)]
            self.n = [STRESS_N]
            self.raw_bytes = STRESS_N * 2
            return
        self.cfg = kvgen.CONFIGS[cfg_name]
        self.dtype = 1 if self.cfg.fp8 else 0
        nl = self.cfg.layers if layers_per_step is None else layers_per_step
        if layers is not None:  # a smaller batch of the same tensors (profiler captures)
            nl = layers
        self.layers = rank_layers(nl, rank, world)
        self.xs = [kvgen.kv_tensor(self.cfg, l % self.cfg.layers if world == 1 else l, kv, device=device)
                   for l in self.layers for kv in (0, 1)]
        self.n = [x.numel() for x in self.xs]
        self.esize = 1 if self.cfg.fp8 else 2
        self.raw_bytes = sum(self.n) * self.esize


def paged_pools(wl, page_tokens: int, device):
    """Two page pools holding the workload's tensors in pages of page_tokens
    tokens, each in its own random page order (seeded).  Returns (source pool,
    destination pool, source page tables, destination page tables, elements per page)."""
    shape = wl.xs[0].shape  # [tokens, heads, head_dim]
    page_elems = page_tokens * shape[1] * shape[2]
    if page_elems % 1024:
        raise SystemExit("--paged: a page must hold a multiple of 1024 elements")
    counts = [-(-n // page_elems) for n in wl.n]
    total = sum(counts)
    pb = page_elems * wl.esize
    src_pool = torch.empty(total * pb, dtype=torch.uint8, device=device)
    dst_pool = torch.zeros(total * pb, dtype=torch.uint8, device=device)
    g = torch.Generator(device="cpu")
    g.manual_seed(7_000_000 + page_tokens)
    src_order = torch.randperm(total, generator=g).to(torch.int32)
    dst_order = torch.randperm(total, generator=g).to(torch.int32)
    src_tabs, dst_tabs, k = [], [], 0
    for x, c in zip(wl.xs, counts):
        sid, did = src_order[k: k + c].to(device), dst_order[k: k + c].to(device)
        k += c
        flat = x.view(torch.uint8).reshape(-1)
        padded = torch.zeros(c * pb, dtype=torch.uint8, device=device)
        padded[: flat.numel()] = flat
        src_pool.view(total, pb)[sid.long()] = padded.view(c, pb)
        src_tabs.append(sid)
        dst_tabs.append(did)
    return src_pool, dst_pool, src_tabs, dst_tabs, page_elems


def run_ours(args, rank, world, device, wl=None):
    import fp8_kv_cache_exp_b200 as sz
    if wl is None:
        wl = Workload(args.workload, rank, world, device, args.layers)
    if wl.cfg is None and (args.mode != "batch" or args.paged or args.transfer or args.layers):
        raise SystemExit("the stress workload is one flat tensor: batch mode only")
    dt = wl.dtype
    T = len(wl.xs)
    stream = torch.cuda.current_stream()
    ws = sz.new_workspace(dt, wl.n)
    plans = sz.new_plans(T)
    caps = [sz.sz_max_compressed_size(dt, n) for n in wl.n]
    outs = [torch.empty(c, dtype=torch.uint8, device=device) for c in caps]
    decs = [torch.empty_like(x) for x in wl.xs]

    if args.mode == "batch":
        groups = [list(range(T))]
    else:  # per layer: K and V of one layer per call
        groups = [[2 * i, 2 * i + 1] for i in range(T // 2)]
    ws_g = [sz.new_workspace(dt, [wl.n[i] for i in g]) for g in groups] if args.mode != "batch" else [ws]
    plans_g = [plans[g[0]: g[-1] + 1] for g in groups]

    # the buffers stay in place across steps: marshal each call's arrays once
    if args.paged:
        # paged KV: every tensor's pages sit in one pool in a random order (the
        # prefill side), and decode writes into a second pool with its own random
        # page order (the decode side)
        src_pool, dst_pool, src_tabs, dst_tabs, page_elems = paged_pools(wl, args.paged, device)
        srcs = [sz.paged(dt, src_pool, tb, page_elems) for tb in src_tabs]
        dsts = [sz.paged(dt, dst_pool, tb, page_elems) for tb in dst_tabs]
        batches = [sz.Batch(dt, None, [outs[i] for i in g], w, p, src_pages=[srcs[i] for i in g],
                            dst_pages=[dsts[i] for i in g], n=[wl.n[i] for i in g], raw_blocks=args.raw_blocks)
                   for g, w, p in zip(groups, ws_g, plans_g)]
    else:
        batches = [sz.Batch(dt, [wl.xs[i] for i in g], [outs[i] for i in g], w, p, decs=[decs[i] for i in g],
                            raw_blocks=args.raw_blocks)
                   for g, w, p in zip(groups, ws_g, plans_g)]

    def plan_all():
        for b in batches:
            b.plan()

    def encode_all():
        for b in batches:
            if args.reuse:
                b.encode_reuse()  # codebooks of the calibration plan, no histogram pass
            else:
                b.encode()

    def decode_all():
        for b in batches:
            b.decode()

    # correctness of this very configuration before timing (with --reuse, this
    # plan is the calibration whose codebooks every timed step reuses)
    plan_all(); encode_all(); decode_all()
    for w in ws_g:
        st = sz.sz_last_device_status(w)
        if st != 0:
            raise RuntimeError("device status %s" % sz.sz_status_string(st))
    if args.paged:
        decs = [dst_pool.view(-1, page_elems * wl.esize)[tb.long()].reshape(-1)[: n * wl.esize]
                for tb, n in zip(dst_tabs, wl.n)]
    for x, d in zip(wl.xs, decs):
        if not torch.equal(x.view(torch.uint8).reshape(-1), d.view(torch.uint8).reshape(-1)):
            raise RuntimeError("round trip mismatch")
    # stream lengths and escape-section bytes from the streams' own headers
    # (with raw blocks the plans hold upper bounds)
    heads = torch.stack([o[:64] for o in outs]).cpu()
    stream_bytes = int(heads[:, 40:48].contiguous().view(torch.int64).sum().item())
    E_total = int(heads[:, 16:24].contiguous().view(torch.int64).sum().item())

    if args.reuse:
        def plan_all():  # noqa: F811 -- the timed step reuses the calibration codebooks
            pass

    for _ in range(args.warmup):
        plan_all(); encode_all(); decode_all()
    torch.cuda.synchronize()

    K = args.steps
    R = max(K, args.kernel_reps)
    # Per-kernel figures: each kernel's launches of one step captured as a graph
    # of its own (no host gap inside a measurement), replayed in step order.
    parts = {"encode": encode_all, "decode": decode_all}
    if not args.reuse:
        parts = {"plan": plan_all, **parts}
    kt = graph_part_times(parts, R, stream, device, args.warmup)
    check_status(sz, ws_g, "kernel timing")

    # The timed region: K steps, the whole step captured once as a CUDA graph
    # (--no-graph: direct launches), bracketed by a barrier and a synchronize.
    graph = None
    if args.graph:
        graph = capture_graph(lambda: (plan_all(), encode_all(), decode_all()), stream, device)
        for _ in range(args.warmup):
            graph.replay()
    step = graph.replay if graph is not None else (lambda: (plan_all(), encode_all(), decode_all()))
    clocks = ClockSampler(gpu_uuid(device))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    head_start()
    ev[0].record(stream)
    for k in range(K):
        step()
        ev[k + 1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    total_ms = ev[0].elapsed_time(ev[K])
    step_ms = [ev[k].elapsed_time(ev[k + 1]) for k in range(K)]
    check_status(sz, ws_g, "timed steps")
    # the median step over more replays (outside the timed region)
    reps = max(K, 50)
    ev2 = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    head_start()
    ev2[0].record(stream)
    for k in range(reps):
        step()
        ev2[k + 1].record(stream)
    torch.cuda.synchronize()
    more = sorted(ev2[k].elapsed_time(ev2[k + 1]) for k in range(reps))
    check_status(sz, ws_g, "step replays")
    if not args.paged:
        for x, d in zip(wl.xs, decs):
            if not torch.equal(x.view(torch.uint8), d.view(torch.uint8)):
                raise RuntimeError("round trip mismatch after timing")
    del graph

    ms_step = max_over_ranks(total_ms / K, world, device)
    raw_all = sum_over_ranks(float(wl.raw_bytes), world, device)
    value = raw_all / (ms_step * 1e-3) / 1e9

    peak, peak_kind = load_peaks()
    # plan, encode, decode per call (no plan with --reuse); paged and E5M2 decode add their
    # raw-block pass
    launches_per_step = ((2 if args.reuse else 3) + (1 if args.paged or dt == 1 else 0)) * len(groups)
    kbytes = {"plan": wl.raw_bytes + 64 * T, "encode": wl.raw_bytes + stream_bytes,
              "decode": stream_bytes + wl.raw_bytes}
    kern = {k: kernel_figures(kt[k], kbytes[k], peak) for k in kt}
    dom = max(kern, key=lambda k: kern[k]["ms"])
    key = wl.name + ("+paged%d" % args.paged if args.paged else "")
    traffic = profiled_traffic(dom + "_kernel", key) if world == 1 and not args.layers and \
        args.mode == "batch" else None
    roof = {"kernel": dom, "bound": "hbm", "achieved": round(kern[dom]["gbs"], 1), "peak": peak,
            "unit": "GB/s", "frac": round(kern[dom]["frac"], 4),
            "traffic": traffic, "algorithmic_bytes": kbytes[dom],
            "peak_source": peak_kind, "launches_timed": R,
            "timing": "mean of %d replays of the kernel's own graph (one step's launches)" % R}
    t_plan = kern["plan"]["ms"] if "plan" in kern else 0.0
    t_enc, t_dec = kern["encode"]["ms"], kern["decode"]["ms"]
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "u8" if dt == 1 else "u16", "data": "synthetic (seeded generator: kvgen)",
        "config": {"workload": wl.name, "desc": wl.desc, "tensors_per_rank": T,
                   "launch": "one CUDA graph per step" if args.graph else "direct launches",
                   "codebooks": "reused from a calibration plan (no histogram pass per step)" if args.reuse
                   else "own plan per step",
                   "layout": ("paged: %d-token pages, random page order in and out" % args.paged) if args.paged
                   else "contiguous tensors",
                   "raw_blocks": bool(args.raw_blocks),
                   "raw_bytes_per_rank": wl.raw_bytes, "mode": "one batch" if args.mode == "batch" else "per layer",
                   "l2": "inputs larger than L2, no flush (%.2f GB per step per rank)" % (wl.raw_bytes / 1e9),
                   "parallelism": "replicas" if world == 1 else "dp%d (independent tensors)" % world},
        "step_stats": {"replays": reps, "median_ms": round(statistics.median(more), 4),
                       "p10_ms": round(more[reps // 10], 4), "p90_ms": round(more[(9 * reps) // 10], 4),
                       "value_at_median": round(wl.raw_bytes / (statistics.median(more) * 1e-3) / 1e9, 2),
                       "timed_steps_median_ms": round(statistics.median(step_ms), 4)},
        "encode_gbs": round(wl.raw_bytes / ((t_plan + t_enc) * 1e-3) / 1e9, 1),
        "decode_gbs": round(wl.raw_bytes / (t_dec * 1e-3) / 1e9, 1),
        "ratio": round(wl.raw_bytes / stream_bytes, 5),
        "escape_fraction": round(E_total / sum(wl.n), 6),
        "kernels": {k: {kk: (round(vv, 4) if kk != "gbs" else round(vv, 1)) for kk, vv in v.items()}
                    for k, v in kern.items()},
        "roofline": roof,
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    return res, wl


# ------------------------------------------------------ per-config records

L2_FLUSH_BYTES = 256 << 20   # written between measurements that must start with a cold L2 (2x its 126 MB)


def cold_l2(buf: torch.Tensor, tag: int = 0):
    """Leave L2 holding none of the data that follows and no dirty lines: write
    a buffer of twice its size (evicting everything, writing back what was
    dirty), then read it (the written lines go back to DRAM, clean copies stay)."""
    buf.fill_(tag & 0xFF)
    buf.view(torch.int32).sum()


def record_of(res: dict) -> dict:
    """The figures of one workload's run (run_ours) for the `configs` object."""
    keep = ("value", "unit", "ms_per_step", "ratio", "escape_fraction", "encode_gbs", "decode_gbs",
            "kernels", "roofline", "step_stats", "gpu_launches", "clocks")
    out = {"workload": res["config"]["workload"], "desc": res["config"]["desc"],
           "mode": res["config"]["mode"], "l2": res["config"]["l2"], "dtype": res["dtype"]}
    out.update({k: res[k] for k in keep if k in res})
    return out


def record_qwen3_stream(args, device, peak: float, peak_kind: str, layers: int = None) -> dict:
    """Qwen3-32B KV at 131072 tokens, as the config describes it: 64 layers x
    {K, V} x [131072, 8, 128] bf16 (34.4 GB), generated on the device one layer
    at a time and coded layer by layer -- plan, encode and decode of the layer's
    K and V, one batched call each (537 MB per call).  Before each layer's
    measured pass a 256 MB buffer is written and read back, so that the layer
    starts with a cold L2 holding no dirty lines (`cold`); the same calls are then repeated at once (`warm`: L2 holds
    what the first pass left).  Per-kernel figures are medians over the layers;
    every layer's decode is checked bit for bit against its input."""
    import fp8_kv_cache_exp_b200 as sz
    cfg = kvgen.CONFIGS["qwen3-32b"]
    nl = cfg.layers if layers is None else layers
    n = cfg.numel
    stream = torch.cuda.current_stream()
    ws = sz.new_workspace(0, [n, n])
    plans = sz.new_plans(2)
    outs = [torch.empty(sz.sz_max_compressed_size(0, n), dtype=torch.uint8, device=device) for _ in range(2)]
    decs = [torch.empty(cfg.shape, dtype=torch.bfloat16, device=device) for _ in range(2)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    raw_layer = 2 * n * 2
    names = ("plan", "encode", "decode")
    cold = {k: [] for k in names}
    warm = {k: [] for k in names}
    kb = {k: [] for k in names}
    stream_total = E_total = 0
    clocks = ClockSampler(gpu_uuid(device))
    clocks.start()
    for layer in range(nl):
        xs = [kvgen.kv_tensor(cfg, layer, kv, device=device) for kv in (0, 1)]
        b = sz.Batch(0, xs, outs, ws, plans, decs=decs)
        if layer == 0:  # first calls of these sizes (launch setup), not measured
            b.plan(); b.encode(); b.decode()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
        head_start()
        cold_l2(flush, layer)
        for rep in range(2):
            ev[4 * rep].record(stream)
            b.plan()
            ev[4 * rep + 1].record(stream)
            b.encode()
            ev[4 * rep + 2].record(stream)
            b.decode()
            ev[4 * rep + 3].record(stream)
        torch.cuda.synchronize()
        check_status(sz, [ws], "qwen3-32b layer %d" % layer)
        for x, d in zip(xs, decs):
            if not torch.equal(x.view(torch.uint8), d.view(torch.uint8)):
                raise RuntimeError("qwen3-32b layer %d: round trip mismatch" % layer)
        heads = torch.stack([o[:64] for o in outs]).cpu()
        sb = int(heads[:, 40:48].contiguous().view(torch.int64).sum().item())
        E_total += int(heads[:, 16:24].contiguous().view(torch.int64).sum().item())
        stream_total += sb
        layer_bytes = {"plan": raw_layer + 128, "encode": raw_layer + sb, "decode": raw_layer + sb}
        for i, k in enumerate(names):
            cold[k].append(ev[i].elapsed_time(ev[i + 1]))
            warm[k].append(ev[4 + i].elapsed_time(ev[4 + i + 1]))
            kb[k].append(layer_bytes[k])
        del xs, b
    clk = clocks.stop()
    del flush, outs, decs, ws
    torch.cuda.empty_cache()

    kern = {}
    for k in names:
        g_cold = [by / (t * 1e-3) / 1e9 for by, t in zip(kb[k], cold[k])]
        g_warm = [by / (t * 1e-3) / 1e9 for by, t in zip(kb[k], warm[k])]
        kern[k] = {"ms": round(statistics.median(cold[k]), 4), "gbs": round(statistics.median(g_cold), 1),
                   "frac": round(statistics.median(g_cold) / peak, 4),
                   "frac_min": round(min(g_cold) / peak, 4), "frac_max": round(max(g_cold) / peak, 4),
                   "warm_ms": round(statistics.median(warm[k]), 4),
                   "warm_frac": round(statistics.median(g_warm) / peak, 4)}
    dom = max(kern, key=lambda k: kern[k]["ms"])
    t_cold = sum(sum(cold[k]) for k in names)
    raw_all = raw_layer * nl
    return {
        "workload": "qwen3-32b", "desc": "Qwen3-32B KV at 131072 tokens: %d layers x {K,V} x [131072,8,128] bf16, "
                                         "generated on the device and coded layer by layer (537 MB per call)" % nl,
        "mode": "per layer, streamed", "dtype": "u16", "layers": nl,
        "l2": "cold: 256 MB written and read back before each layer (inputs 537 MB per layer); "
                    "warm: the layer's calls repeated at once",
        "value": round(raw_all / (t_cold * 1e-3) / 1e9, 2), "unit": UNIT,
        "ms_per_layer": round(t_cold / nl, 4),
        "ratio": round(raw_all / stream_total, 5), "escape_fraction": round(E_total / (2 * n * nl), 6),
        "encode_gbs": round(raw_layer / ((kern["plan"]["ms"] + kern["encode"]["ms"]) * 1e-3) / 1e9, 1),
        "decode_gbs": round(raw_layer / (kern["decode"]["ms"] * 1e-3) / 1e9, 1),
        "kernels": kern,
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": kern[dom]["gbs"], "peak": peak, "unit": "GB/s",
                     "frac": kern[dom]["frac"], "traffic": profiled_traffic(dom + "_kernel", "qwen3-32b"),
                     "algorithmic_bytes": int(statistics.median(kb[dom])), "peak_source": peak_kind,
                     "timing": "median over %d layers of one launch each, cold L2" % nl},
        "gpu_launches": 3 * 2 * nl,
        "clocks": clk,
    }


def run_transfer(args, wl, device, res):
    """Layer-pipelined transfer (fp8_kv_cache_exp_b200.transfer): per layer, plan +
    encode on the source, decode on the destination from the source's streams.
    One GPU: source and destination are the same device (the link is not crossed);
    the pipeline's device time is measured, and the transfer over a link of speed B
    is modelled from the measured per-layer codec times (FastKVComp page, Equation 1
    for the break-even)."""
    from fp8_kv_cache_exp_b200.transfer import LayerPipeline, break_even_gbs, pipelined_seconds
    layers = [[wl.xs[2 * i], wl.xs[2 * i + 1]] for i in range(len(wl.xs) // 2)]
    pipe = LayerPipeline(layers, device)
    for _ in range(args.warmup):
        pipe.run()
    pipe.synchronize()
    # per-layer stage times, from one instrumented pass (events around each call)
    enc_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in layers]
    dec_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in layers]
    import fp8_kv_cache_exp_b200 as sz
    for i, (b, outs, dec, ws) in enumerate(zip(pipe.batches, pipe.outs, pipe.decoded, pipe.ws_dst)):
        with torch.cuda.stream(pipe.s_src):
            enc_ev[i][0].record(pipe.s_src)
            b.plan(stream=pipe.s_src)
            b.encode(stream=pipe.s_src)
            enc_ev[i][1].record(pipe.s_src)
        pipe.s_dst.wait_stream(pipe.s_src)
        with torch.cuda.stream(pipe.s_dst):
            dec_ev[i][0].record(pipe.s_dst)
            sz.sz_decode_batched(wl.dtype, outs, dec, ws, stream=pipe.s_dst)
            dec_ev[i][1].record(pipe.s_dst)
        pipe.s_src.wait_stream(pipe.s_dst)
    pipe.synchronize()
    t_enc = [a.elapsed_time(b) * 1e-3 for a, b in enc_ev]
    t_dec = [a.elapsed_time(b) * 1e-3 for a, b in dec_ev]
    # the pipelined run itself
    K = args.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(pipe.s_src)
    for _ in range(K):
        pipe.run()
    pipe.s_src.wait_stream(pipe.s_dst)
    stop.record(pipe.s_src)
    pipe.synchronize()
    ms = start.elapsed_time(stop) / K
    for src, out in zip(layers, pipe.decoded):
        for x, y in zip(src, out):
            if not torch.equal(x.view(torch.uint8), y.view(torch.uint8)):
                raise RuntimeError("transfer round trip mismatch")
    ratio = res["ratio"]
    S = float(wl.raw_bytes)
    layer_bytes = [float(x.numel() * x.element_size() + y.numel() * y.element_size()) for x, y in layers]
    codec_s = sum(t_enc) + sum(t_dec)
    links = {}
    for name, gbs in (("RoCE 4x200 Gb/s (the SplitZip setup)", 100.0), ("NVLink 5, 900 GB/s nominal", 900.0)):
        B = gbs * 1e9
        raw_s = S / B
        serial_s = codec_s + S / (ratio * B)
        piped_s = pipelined_seconds([(te, lb / (ratio * B), td) for te, td, lb in zip(t_enc, t_dec, layer_bytes)])
        links[name] = {"link_gbs": gbs, "raw_ms": round(raw_s * 1e3, 4), "compressed_serial_ms": round(serial_s * 1e3, 4),
                       "compressed_pipelined_ms": round(piped_s * 1e3, 4),
                       "speedup_pipelined": round(raw_s / piped_s, 3)}
    return {
        "pipeline_ms_per_step": round(ms, 4),
        "pipeline_gbs": round(S / (ms * 1e-3) / 1e9, 1),
        "devices": "one GPU: source and destination are the same device (loopback)",
        "layers": len(layers),
        "encode_ms_per_layer": round(1e3 * sum(t_enc) / len(layers), 4),
        "decode_ms_per_layer": round(1e3 * sum(t_dec) / len(layers), 4),
        "break_even_gbs_serial": round(break_even_gbs(S, ratio, codec_s), 1),
        "model": links,
        "model_note": "link times are modelled from the measured per-layer codec times; the link is not measured",
    }


def run_e2e(args, wl, device):
    """Same metric through the C ABI with host buffers: every step copies its raw
    batch from pinned host memory to the device, runs plan + encode + decode, and
    copies the decoded batch back, all inside the timed region.  Steps are
    pipelined over three streams and two device buffer sets: while step k runs
    its kernels, step k+1's input crosses PCIe one way and step k-1's output the
    other way (PCIe is full duplex)."""
    import fp8_kv_cache_exp_b200 as sz
    dt = wl.dtype
    NB = 2  # device buffer sets in flight
    host_in = [x.cpu().pin_memory() for x in wl.xs]
    host_out = [torch.empty_like(h).pin_memory() for h in host_in]
    dev_in = [[torch.empty_like(x) for x in wl.xs] for _ in range(NB)]
    dev_out = [[torch.empty_like(x) for x in wl.xs] for _ in range(NB)]
    ws = sz.new_workspace(dt, wl.n)
    plans = sz.new_plans(len(wl.xs))
    outs = [torch.empty(sz.sz_max_compressed_size(dt, n), dtype=torch.uint8, device=device) for n in wl.n]
    batches = [sz.Batch(dt, dev_in[b], outs, ws, plans, decs=dev_out[b], raw_blocks=args.raw_blocks)
               for b in range(NB)]
    s_in, s_comp, s_out = (torch.cuda.Stream(device=device) for _ in range(3))
    in_done = [torch.cuda.Event() for _ in range(NB)]
    comp_done = [torch.cuda.Event() for _ in range(NB)]
    out_done = [torch.cuda.Event() for _ in range(NB)]
    used = [False] * NB

    def step(k):
        b = k % NB
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(comp_done[b])  # step k - NB has finished reading dev_in[b]
            for h, d in zip(host_in, dev_in[b]):
                d.copy_(h, non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[b])
            if used[b]:
                s_comp.wait_event(out_done[b])  # step k - NB's output has left dev_out[b]
            if args.reuse:
                batches[b].encode_reuse(stream=s_comp)  # codebooks of the calibration plan
            else:
                batches[b].plan(stream=s_comp)
                batches[b].encode(stream=s_comp)
            batches[b].decode(stream=s_comp)
            comp_done[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            for d, h in zip(dev_out[b], host_out):
                h.copy_(d, non_blocking=True)
            out_done[b].record(s_out)
        used[b] = True

    if args.reuse:  # calibration plan, outside the timed region
        for h, d in zip(host_in, dev_in[0]):
            d.copy_(h)
        batches[0].plan()
        torch.cuda.synchronize()

    step(0)
    torch.cuda.synchronize()
    for h, g in zip(host_out, host_in):
        if not torch.equal(h.view(torch.uint8), g.view(torch.uint8)):
            raise RuntimeError("e2e round trip mismatch")
    k = 1
    for _ in range(max(1, args.warmup // 2)):
        step(k)
        k += 1
    K = max(2, min(args.steps, 5))
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for _ in range(K):
        step(k)
        k += 1
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize()
    if sz.sz_last_device_status(ws) != 0:
        raise RuntimeError("device status in e2e")
    for h, g in zip(host_out, host_in):
        if not torch.equal(h.view(torch.uint8), g.view(torch.uint8)):
            raise RuntimeError("e2e round trip mismatch after timing")
    ms = a.elapsed_time(b) / K
    return {"value": round(wl.raw_bytes / (ms * 1e-3) / 1e9, 2), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": wl.raw_bytes, "d2h_bytes_per_step": wl.raw_bytes, "steps": K,
            "pipelining": "H2D of step k+1, kernels of step k and D2H of step k-1 overlap (3 streams, 2 buffer sets)"}


# ------------------------------------------------------- the oracle arm

def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class pinned_to_one_core:
    """Pin this process to one host core (the highest-numbered one it may use)
    for the duration of a with-block, then restore its affinity."""

    def __enter__(self):
        self.saved = None
        self.core = None
        try:
            self.saved = os.sched_getaffinity(0)
            self.core = max(self.saved)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            self.saved = None
        return self

    def __exit__(self, *exc):
        if self.saved is not None:
            os.sched_setaffinity(0, self.saved)
        return False


def oracle_host_sample(cfg_name: str):
    """(dtype, host byte arrays, description) of the reference arm's per-step
    sample: one layer's K and V (the stress workload: a 2^23-element tensor of
    the same generator)."""
    if cfg_name == "stress-uniform":
        xs = [kvgen.stress_tensor(STRESS_SAMPLE_N, None, stress_seed())]
        return 0, [x.contiguous().view(torch.uint8).reshape(-1).numpy() for x in xs], \
            "stress-uniform 2^23 elements"
    cfg = kvgen.CONFIGS[cfg_name]
    xs = [kvgen.kv_tensor(cfg, 0, kv) for kv in (0, 1)]
    return (1 if cfg.fp8 else 0), [x.contiguous().view(torch.uint8).reshape(-1).numpy() for x in xs], \
        "%s layer 0 K+V" % cfg_name


def oracle_sample(dt: int, raws, what: str, budget_s: float, raw_blocks: bool = False, max_reps: int = 1 << 30):
    """Time the CPU oracle (as it stands: plain single-threaded C), pinned to one
    host core, on the tensors `raws` (host byte arrays): plan + encode + decode
    of each, in order, repeated until budget_s seconds have passed (at least one
    tensor, at most max_reps passes).  A pass that runs out of budget stops
    after the tensor in progress; the sample says how many tensors were coded."""
    import numpy as np
    import oracle
    t_enc = t_dec = 0.0
    coded = 0
    nbytes = 0
    reps = 0
    with pinned_to_one_core() as pin:
        t_start = time.perf_counter()
        done = False
        while not done and reps < max_reps:
            for r in raws:
                n = r.size // (2 if dt == 0 else 1)
                t0 = time.perf_counter()
                s = oracle.encode(dt, r, raw_blocks=raw_blocks)
                t1 = time.perf_counter()
                back = oracle.decode(s, n, dt)
                t2 = time.perf_counter()
                t_enc += t1 - t0
                t_dec += t2 - t1
                if not np.array_equal(back, r):
                    raise RuntimeError("oracle round trip mismatch")
                coded += 1
                nbytes += r.size
                if time.perf_counter() - t_start > budget_s:
                    done = True
                    break
            reps += 1
        core = pin.core
    return {
        "value": round(nbytes / (t_enc + t_dec) / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
        "pinned_core": core, "host_cores": os.cpu_count(), "cpu_model": cpu_model(),
        "sample": "%s: %d tensor(s) coded, %.1f MB raw, single-threaded C oracle pinned to one core%s" % (
            what, coded, nbytes / 1e6, ", raw blocks allowed" if raw_blocks else ""),
        "encode_gbs": round(nbytes / t_enc / 1e9, 4), "decode_gbs": round(nbytes / t_dec / 1e9, 4),
        "seconds": round(t_enc + t_dec, 2),
    }


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cfg_name = WORKLOADS[args.workload][0]
    dt, raws, what = oracle_host_sample(cfg_name)
    sample = None
    times = []
    for k in range(args.warmup + args.steps):
        r = oracle_sample(dt, raws, what, 0.0, args.raw_blocks, max_reps=1)
        if k >= args.warmup:
            times.append(r)
        sample = r
    val = statistics.median(t["value"] for t in times)
    fp8 = dt == 1
    raw = sum(r.size for r in raws)
    ms = raw / (val * 1e9) * 1e3
    cpu = dict(sample)
    cpu["value"] = val
    cpu["sample"] = "%s per step (%d steps, median), single-threaded C oracle pinned to one core" % (
        what, args.steps)
    return {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8" if fp8 else "u16", "data": "synthetic",
        "config": {"workload": args.workload, "desc": WORKLOADS[args.workload][2],
                   "sample": cpu["sample"]},
        "cpu_baseline": cpu,
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama3-8b")
    ap.add_argument("--mode", choices=["batch", "per_layer"], default="batch")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers per step (default: the workload's); smaller batches are for profiler captures")
    ap.add_argument("--reuse", action="store_true",
                    help="codebook reuse: plan once, then every step is encode with those codebooks + decode")
    ap.add_argument("--paged", type=int, default=0, metavar="TOKENS",
                    help="hold the tensors in pages of TOKENS tokens (paged KV), in random page order")
    ap.add_argument("--transfer", action="store_true",
                    help="also run the layer-pipelined transfer (encode on the source, decode on the destination)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time the step with direct launches instead of one captured CUDA graph per step")
    ap.add_argument("--raw-blocks", action="store_true",
                    help="allow raw blocks (header flag): blocks that would expand are stored raw")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-records", action="store_true",
                    help="skip the other workloads' records (`configs`) of the default run")
    ap.add_argument("--qwen3-layers", type=int, default=None,
                    help="layers of the streamed Qwen3-32B record (default: all 64)")
    ap.add_argument("--kernel-reps", type=int, default=50,
                    help="replays of each kernel's graph for the per-kernel figures (at least --steps)")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=30.0,
                    help="bound on the CPU oracle's timed work (0: skip it)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    try:
        res, wl = run_ours(args, rank, world, device)
        if not args.no_e2e and not args.paged:  # e2e covers the contiguous path
            e2e = run_e2e(args, wl, device)
            e2e_val = sum_over_ranks(wl.raw_bytes, world, device) / (
                max_over_ranks(e2e["ms_per_step"], world, device) * 1e-3) / 1e9
            e2e["value"] = round(e2e_val, 2)
            res["e2e"] = e2e
        if args.transfer:
            res["transfer"] = run_transfer(args, wl, device, res)
        default_run = (args.workload == "llama3-8b" and args.mode == "batch" and not args.reuse and
                       not args.paged and not args.raw_blocks and args.layers is None and not args.transfer)
        if world == 1 and default_run and not args.no_records:
            # the other KV configurations, measured in the same run
            peak, peak_kind = load_peaks()
            recs = {}
            a2 = argparse.Namespace(**vars(args))
            a2.mode = "per_layer"
            r, _ = run_ours(a2, rank, world, device, wl=wl)
            recs["llama3-8b-per-layer"] = record_of(r)
            hosts = [x.cpu() for x in wl.xs] if args.cpu_baseline_seconds > 0 else None
            del wl
            torch.cuda.empty_cache()
            recs["qwen3-32b"] = record_qwen3_stream(args, device, peak, peak_kind, args.qwen3_layers)
            a3 = argparse.Namespace(**vars(args))
            a3.workload = "qwen3-30b-a3b-e5m2"
            r, wl5 = run_ours(a3, rank, world, device)
            recs["qwen3-30b-a3b-e5m2"] = record_of(r)
            del wl5
            torch.cuda.empty_cache()
            res["configs"] = recs
            if hosts is not None:
                raws = [h.contiguous().view(torch.uint8).reshape(-1).numpy() for h in hosts]
                res["cpu_baseline"] = oracle_sample(0, raws, "llama3-8b, all 64 K/V tensors of the batch",
                                                    args.cpu_baseline_seconds, max_reps=1)
        elif rank == 0 and world == 1 and args.cpu_baseline_seconds > 0:
            dt, raws, what = oracle_host_sample(WORKLOADS[args.workload][0])
            res["cpu_baseline"] = oracle_sample(dt, raws, what, args.cpu_baseline_seconds, args.raw_blocks,
                                                max_reps=30)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
