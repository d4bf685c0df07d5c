"""The layer pipeline on one GPU (source and destination the same device): every
layer decodes to its input, the streams are the oracle's, and repeated runs reuse
the buffers safely.  With two GPUs the same code decodes on the peer, reading the
source's streams over NVLink; only one GPU is available to these tests."""
import numpy as np
import pytest
import torch

import kvgen
import oracle
from gpu_helpers import raw_of, sz

pytestmark = pytest.mark.gpu


def test_layer_pipeline_loopback():
    sz()
    from fp8_kv_cache_exp_b200.transfer import LayerPipeline
    cfg = kvgen.CONFIGS["phi2"]
    layers = [[kvgen.kv_tensor(cfg, 0, kv).cuda() for kv in (0, 1)] for _ in range(1)]
    llama = kvgen.CONFIGS["llama3-8b"]
    layers += [[kvgen.kv_tensor(llama, l, kv).cuda() for kv in (0, 1)] for l in (0, 1, 2)]
    pipe = LayerPipeline(layers, torch.cuda.current_device())
    for _ in range(2):
        dec = pipe.run()
        pipe.synchronize()
        for src, out in zip(layers, dec):
            for x, y in zip(src, out):
                assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    # the streams that crossed are the oracle's
    raw = raw_of(layers[1][0])
    ref = oracle.encode(0, raw)
    assert np.array_equal(pipe.outs[1][0][: ref.size].cpu().numpy(), ref)
