"""Layer-pipelined KV transfer: compress on the source GPU, decompress on the
destination GPU, which pulls the compressed streams straight out of the source's
memory.

The use the codec is made for (SplitZip project page, FAQ "How can I reduce KV
cache transfer time between prefill and decode nodes?"): the prefill GPU
compresses the KV cache, the decode GPU decompresses it, and the bytes saved
shorten the transfer.  Here the link is NVLink: after sz_enable_peer_access,
the decode kernel on the destination reads the source's stream buffers with its
own bulk copies, so each layer crosses the link inside the decode kernel, tile
by tile, and never lands in the destination's memory.  Layers are pipelined
over two streams: layer i+1 is planned and encoded on the source while layer i
crosses and is decoded.

Whether compressing pays at all is the question of the FastKVComp page
(Equation 1): encoding plus decoding must take less time than the wire time the
smaller payload saves.  break_even_gbs() gives the link speed below which it
pays when codec and link run one after the other.

Host orchestration only: every step on the data runs in the library's kernels.
"""
import torch

from . import (Batch, dtype_of, new_plans, new_workspace, numel_of, sz_decode_batched, sz_enable_peer_access,
               sz_max_compressed_size)


def break_even_gbs(raw_bytes: float, ratio: float, codec_seconds: float) -> float:
    """Link speed (GB/s) below which compressing pays when the codec and the link
    run one after the other (FastKVComp page, Equation 1): sending raw takes
    S / B, sending compressed takes t_codec + S / (r B); the second is shorter
    exactly when B < S (1 - 1/r) / t_codec."""
    if codec_seconds <= 0 or ratio <= 1.0:
        return 0.0
    return raw_bytes * (1.0 - 1.0 / ratio) / codec_seconds / 1e9


def pipelined_seconds(stages) -> float:
    """Time for layers to pass in order through stages that each serve one layer at
    a time (the source GPU, the link, the destination GPU): layer i enters stage
    s when it has left stage s - 1 and layer i - 1 has left stage s.
    stages: per layer, its stage times in stage order."""
    done = []  # completion time of the previous layer at each stage
    for t in stages:
        cur, prev_stage = [], 0.0
        for s, dt in enumerate(t):
            start = max(prev_stage, done[s] if done else 0.0)
            prev_stage = start + dt
            cur.append(prev_stage)
        done = cur
    return done[-1] if done else 0.0


class LayerPipeline:
    """Per layer: plan + encode on the source device, decode on the destination.

    layers: a list of layers, each a list of tensors (bf16 or float8_e5m2,
    contiguous) on the source device.  dst_device: where the decoded tensors go
    (may be the source itself).  After run(), decoded[i][j] holds layer i's
    tensor j on the destination.  Buffers are allocated once; run() may be
    repeated.
    """

    def __init__(self, layers, dst_device):
        self.layers = [list(l) for l in layers]
        first = self.layers[0][0]
        self.dtype = dtype_of(first)
        self.src = first.device
        self.dst = torch.device(dst_device)
        if self.src.index != self.dst.index:
            sz_enable_peer_access(self.dst.index, self.src.index)
        self.s_src = torch.cuda.Stream(device=self.src)
        self.s_dst = torch.cuda.Stream(device=self.dst)
        self.batches, self.outs, self.decoded, self.ws_dst = [], [], [], []
        self.encoded, self.consumed = [], []  # per layer: stream written (source) / read (destination)
        for layer in self.layers:
            ns = [numel_of(x, self.dtype) for x in layer]
            with torch.cuda.device(self.src):
                ws = new_workspace(self.dtype, ns, device=self.src)
                plans = new_plans(len(layer), device=self.src)
                outs = [torch.empty(sz_max_compressed_size(self.dtype, n), dtype=torch.uint8, device=self.src)
                        for n in ns]
            with torch.cuda.device(self.dst):
                self.ws_dst.append(new_workspace(self.dtype, ns, device=self.dst))
                self.decoded.append([torch.empty(x.shape, dtype=x.dtype, device=self.dst) for x in layer])
            self.batches.append(Batch(self.dtype, layer, outs, ws, plans))
            self.outs.append(outs)
            self.encoded.append(torch.cuda.Event())
            self.consumed.append(None)

    def run(self):
        """Enqueue every layer: encode on the source stream, decode (reading the
        source's streams) on the destination stream after that layer's encode.
        A layer's stream buffers are rewritten only after the previous run's
        decode of that layer has read them."""
        for i, (b, outs, dec, ws) in enumerate(zip(self.batches, self.outs, self.decoded, self.ws_dst)):
            with torch.cuda.device(self.src), torch.cuda.stream(self.s_src):
                if self.consumed[i] is not None:
                    self.s_src.wait_event(self.consumed[i])
                b.plan(stream=self.s_src)
                b.encode(stream=self.s_src)
                self.encoded[i].record(self.s_src)
            with torch.cuda.device(self.dst), torch.cuda.stream(self.s_dst):
                self.s_dst.wait_event(self.encoded[i])
                sz_decode_batched(self.dtype, outs, dec, ws, stream=self.s_dst)
                if self.consumed[i] is None:
                    self.consumed[i] = torch.cuda.Event()
                self.consumed[i].record(self.s_dst)
        return self.decoded

    def synchronize(self):
        self.s_src.synchronize()
        self.s_dst.synchronize()
