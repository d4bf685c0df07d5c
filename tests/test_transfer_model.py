"""Host logic of the layer-pipelined transfer (no GPU): the Equation-1 break-even and
the pipeline timing model, against values worked out by hand."""
import pytest

from fp8_kv_cache_exp_b200.transfer import break_even_gbs, pipelined_seconds


def test_break_even_by_hand():
    # 1.0 GB raw, ratio 4/3: 0.25 GB saved; the codec takes 1 ms -> 250 GB/s
    assert break_even_gbs(1e9, 4.0 / 3.0, 1e-3) == pytest.approx(250.0)
    # at exactly that link speed raw and compressed transfers take the same time
    B = break_even_gbs(2.5e9, 1.25, 4e-3) * 1e9
    assert 2.5e9 / B == pytest.approx(4e-3 + 2.5e9 / (1.25 * B))
    # no gain, no break-even
    assert break_even_gbs(1e9, 1.0, 1e-3) == 0.0


def test_pipeline_model_by_hand():
    # three layers through (encode 1, wire 2, decode 1): the wire is the bottleneck
    # layer 0 leaves at 1, 3, 4; layer 1 at 2, 5, 6; layer 2 at 3, 7, 8
    assert pipelined_seconds([(1, 2, 1)] * 3) == 8
    # equal stages: L layers through 3 stages of t take (L + 2) t
    for L in (1, 2, 7):
        assert pipelined_seconds([(0.5, 0.5, 0.5)] * L) == pytest.approx((L + 2) * 0.5)
    # uneven layers
    assert pipelined_seconds([(1, 1, 1), (3, 1, 1)]) == 6   # layer 1: 4, 5, 6
    assert pipelined_seconds([]) == 0.0

