"""DraftCycle: one draft cycle on fixed shapes, replayed as a CUDA graph.

The cycle is the four stages of the C ABI in order -- the two-tap conv, the
fused LM head + log-softmax + top-16, and path selection fused with greedy
verification -- on buffers owned by the object.  `run()` copies one step's
inputs from pinned host buffers to the device, runs the cycle and copies its
results back, all captured once into a CUDA graph so a step costs one graph
launch on the host.  Weights (W, E, M, conv taps) stay on the device.
"""
from __future__ import annotations

import torch

from . import _binding as b


class DraftCycle:
    def __init__(self, W, E, Msel, a0, a1, B: int, L: int, P: int, use_graph: bool = True):
        dev = W.device
        self.W, self.E, self.Msel, self.a0, self.a1 = W, E, Msel, a0, a1
        self.B, self.L, self.P = B, L, P
        V, d = W.shape
        M = B * L
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
        # device buffers
        self.H, self.x, self.prev = e((M, d), torch.bfloat16), e((B, P, d), torch.bfloat16), e((B, d), torch.bfloat16)
        self.target = e((B, L + 1), torch.int32)
        self.y = e((B, P, d), torch.bfloat16)
        self.lp, self.ix, self.lse = e((M, 16), torch.float32), e((M, 16), torch.int32), e((M,), torch.float32)
        self.tok, self.slot = e((B, L), torch.int32), e((B, L), torch.int32)
        self.score, self.acc, self.nxt = e((B,), torch.float32), e((B,), torch.int32), e((B,), torch.int32)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws = b.workspace(M, V, d, dev)
        # pinned host buffers: inputs the caller fills, results the cycle returns
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        self.host_in = {"H": pin(self.H), "x": pin(self.x), "prev": pin(self.prev), "target": pin(self.target)}
        self.host_out = {"path_tok": pin(self.tok), "accept_len": pin(self.acc), "next_token": pin(self.nxt),
                         "y": pin(self.y)}
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
        for name, dst in (("H", self.H), ("x", self.x), ("prev", self.prev), ("target", self.target)):
            dst.copy_(self.host_in[name], non_blocking=True)
        self.kernels()
        for name, src in (("path_tok", self.tok), ("accept_len", self.acc), ("next_token", self.nxt),
                          ("y", self.y)):
            self.host_out[name].copy_(src, non_blocking=True)

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
        nb = lambda d: int(sum(t.numel() * t.element_size() for t in d.values()))
        return nb(self.host_in), nb(self.host_out)
