"""The seeded synthetic-input generator: shapes, determinism, value structure (no GPU)."""
import numpy as np
import torch

import kvgen


def test_shapes_and_sizes():
    c = kvgen.CONFIGS
    assert c["phi2"].shape == (1024, 32, 80) and c["phi2"].tensors == 2
    assert c["llama3-8b"].shape == (8192, 8, 128) and c["llama3-8b"].tensors == 64
    assert c["llama3-8b"].tensors * c["llama3-8b"].numel * 2 == 1 << 30
    assert c["qwen3-32b"].shape == (131072, 8, 128) and c["qwen3-32b"].tensors == 128
    assert c["qwen3-30b-a3b-e5m2"].shape == (32768, 4, 128) and c["qwen3-30b-a3b-e5m2"].fp8


def test_deterministic_and_distinct():
    cfg = kvgen.CONFIGS["phi2"]
    a = kvgen.kv_tensor(cfg, 0, 0)
    b = kvgen.kv_tensor(cfg, 0, 0)
    v = kvgen.kv_tensor(cfg, 0, 1)
    assert a.dtype == torch.bfloat16 and a.shape == (1024, 32, 80)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), v.view(torch.int16))
    assert kvgen.kv_seed(cfg, 0, 0) == 0 and kvgen.kv_seed(kvgen.CONFIGS["llama3-8b"], 3, 1) == 2_000_007


def test_value_structure():
    x = kvgen.kv_tensor(kvgen.CONFIGS["phi2"], 0, 0).view(torch.int16).numpy().astype(np.int64) & 0xFFFF
    n = x.size
    zeros = (x == 0).mean()
    assert 0.008 < zeros < 0.012
    sub = ((x & 0x7F80) == 0) & ((x & 0x7F) != 0)
    assert 0 < sub.sum() < 5e-4 * n
    # per-channel outliers: some channel has a much larger typical magnitude
    v = kvgen.kv_tensor(kvgen.CONFIGS["phi2"], 0, 0).float().abs().reshape(1024, -1).median(0).values
    assert float(v.max() / v.median()) > 20


def test_fp8_cast():
    cfg = kvgen.KVConfig("tiny-e5m2", 5, 1, 64, 4, 128, layer_scale=False, fp8=True)
    x = kvgen.kv_tensor(cfg, 0, 0)
    assert x.dtype == torch.float8_e5m2 and x.shape == (64, 4, 128)


def test_stress_exponents():
    n = 1 << 16
    for p, lo in ((0, 113), (10, 81), (50, 81)):
        w = kvgen.stress_tensor(n, p, 4_000_000 + p).view(torch.int16).numpy().astype(np.int64) & 0xFFFF
        e = (w >> 7) & 0xFF
        assert e.min() >= lo and e.max() <= 127
        rare = (e < 113).mean()
        assert abs(rare - p / 100) < 0.01
    u = kvgen.stress_tensor(n, None, 4_000_004).view(torch.int16).numpy()
    assert len(np.unique(u)) > 0.5 * n
