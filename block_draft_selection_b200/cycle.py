"""DraftCycle: one draft cycle on fixed shapes, replayed as a CUDA graph.

The cycle is the four stages of the C ABI in order -- the two-tap conv, the
fused LM head + log-softmax + top-16, and path selection fused with greedy
verification -- on buffers owned by the object.  `run()` copies one step's
inputs from pinned host buffers to the device, runs the cycle and copies its
results back, all captured once into a CUDA graph so a step costs one graph
launch on the host.  Weights (W, E, M, conv taps) stay on the device.

The step's inputs live in one pinned host arena and one device arena with the
same layout (each tensor at a 256-byte-aligned offset), and so do its results:
a step moves its inputs with one host-to-device copy and its results with one
device-to-host copy.
"""
from __future__ import annotations

import torch

from . import _binding as b


def _arena(specs, device, pinned=False, align=256):
    """One byte buffer holding tensors of the given (name, shape, dtype) at
    aligned offsets; returns (buffer, {name: view})."""
    offs, off = {}, 0
    for name, shape, dt in specs:
        off = (off + align - 1) // align * align
        n = 1
        for x in shape:
            n *= x
        offs[name] = (off, shape, dt)
        off += n * torch.tensor([], dtype=dt).element_size()
    buf = torch.empty(max(off, 1), dtype=torch.uint8, device=device, pin_memory=pinned)
    views = {}
    for name, (o, shape, dt) in offs.items():
        n = 1
        for x in shape:
            n *= x
        nb = n * torch.tensor([], dtype=dt).element_size()
        views[name] = buf[o:o + nb].view(dt).view(shape)
    return buf, views


class DraftCycle:
    def __init__(self, W, E, Msel, a0, a1, B: int, L: int, P: int, use_graph: bool = True):
        dev = W.device
        self.W, self.E, self.Msel, self.a0, self.a1 = W, E, Msel, a0, a1
        self.B, self.L, self.P = B, L, P
        V, d = W.shape
        M = B * L
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
        ins = [("H", (M, d), torch.bfloat16), ("x", (B, P, d), torch.bfloat16), ("prev", (B, d), torch.bfloat16),
               ("target", (B, L + 1), torch.int32)]
        outs = [("path_tok", (B, L), torch.int32), ("accept_len", (B,), torch.int32),
                ("next_token", (B,), torch.int32), ("y", (B, P, d), torch.bfloat16)]
        # device arenas (inputs, results) and their pinned host twins
        self._din, din = _arena(ins, dev)
        self._dout, dout = _arena(outs, dev)
        self._hin, self.host_in = _arena(ins, "cpu", pinned=True)
        self._hout, self.host_out = _arena(outs, "cpu", pinned=True)
        self.H, self.x, self.prev, self.target = din["H"], din["x"], din["prev"], din["target"]
        self.tok, self.acc, self.nxt, self.y = dout["path_tok"], dout["accept_len"], dout["next_token"], dout["y"]
        self.lp, self.ix, self.lse = e((M, 16), torch.float32), e((M, 16), torch.int32), e((M,), torch.float32)
        self.slot, self.score = e((B, L), torch.int32), e((B,), torch.float32)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws = b.workspace(M, V, d, dev)
        self._graph = None
        if use_graph:
            self._capture()

    def kernels(self):
        """Enqueue the cycle's kernels on the current stream (device buffers)."""
        b.dflash_conv2tap(self.x, self.a0, self.a1, self.prev, y=self.y)
        b.dflash_lmhead_topk(self.H, self.W, topk_logp=self.lp, topk_idx=self.ix, lse=self.lse, ws=self.ws,
                             dev_status=self.status)
        b.dflash_select_verify(self.lp, self.ix, self.E, self.Msel, self.target, self.B, self.L,
                               path_tok=self.tok, path_slot=self.slot, path_score=self.score,
                               accept_len=self.acc, next_token=self.nxt, dev_status=self.status)

    def _step(self):
        self._din.copy_(self._hin, non_blocking=True)      # one host-to-device copy
        self.kernels()
        self._hout.copy_(self._dout, non_blocking=True)    # one device-to-host copy

    def _capture(self):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self._step()                      # warm-up outside capture (first-call set-up)
        side.synchronize()
        self._graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self._graph, stream=side):
            self._step()
        torch.cuda.current_stream().wait_stream(side)

    def run(self):
        """One step: host inputs (self.host_in) -> device -> cycle -> host results."""
        if self._graph is not None:
            self._graph.replay()
        else:
            self._step()
        torch.cuda.current_stream().synchronize()
        return self.host_out

    def io_bytes(self):
        """Bytes a step copies host-to-device and device-to-host (the arenas,
        alignment padding included)."""
        return int(self._hin.numel()), int(self._hout.numel())
