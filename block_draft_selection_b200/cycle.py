"""DraftCycle: one draft cycle on fixed shapes, replayed as a CUDA graph.

The cycle is the four stages of the C ABI in order -- the two-tap conv, the
fused LM head + log-softmax + top-16, and path selection fused with greedy
verification -- on buffers owned by the object.  `run()` copies one step's
inputs from pinned host buffers to the device, runs the cycle and copies its
results back, all captured once into a CUDA graph so a step costs one graph
launch on the host.  Weights (W, E, M, conv taps) stay on the device.

A step has two lanes.  The selection lane's inputs (hidden states, target
tokens), a status word and its results live in one device buffer (each
tensor at a 256-byte-aligned offset), mirrored by a pinned host buffer for
the inputs and one for the results: one host-to-device copy moves the inputs
and a zero status word, one device-to-host copy the status word and the
results, and `run()` raises if the status is nonzero.  The conv does not feed
the LM head, so its lane (one copy of its inputs in, the conv, one copy of its
output out) runs on a second stream inside the same graph, overlapping the
LM head; the step ends when both lanes have.

`launch()` / `wait()` split `run()` in two, and DraftPipeline steps two
cycles over the same weights alternately on two streams, for independent
batches whose copies and kernels may overlap.
"""
from __future__ import annotations

import torch

from . import _binding as b


def _nbytes(shape, dt) -> int:
    n = 1
    for x in shape:
        n *= x
    return n * torch.tensor([], dtype=dt).element_size()


def _offsets(specs, align=256):
    """Offsets of (name, shape, dtype) tensors packed in order at `align`-byte
    boundaries: ({name: (offset, shape, dtype)}, end)."""
    offs, off = {}, 0
    for name, shape, dt in specs:
        off = (off + align - 1) // align * align
        offs[name] = (off, shape, dt)
        off += _nbytes(shape, dt)
    return offs, off


def _views(buf, offs, names, base=0):
    """Typed views of `buf` (a uint8 buffer that starts at byte `base` of the
    layout) for the listed names."""
    out = {}
    for name in names:
        o, shape, dt = offs[name]
        out[name] = buf[o - base:o - base + _nbytes(shape, dt)].view(dt).view(shape)
    return out


def _arena(specs, device, pinned=False, align=256):
    """One byte buffer holding tensors of the given (name, shape, dtype) at
    aligned offsets; returns (buffer, {name: view})."""
    offs, end = _offsets(specs, align)
    buf = torch.empty(max(end, 1), dtype=torch.uint8, device=device, pin_memory=pinned)
    return buf, _views(buf, offs, [n for n, _, _ in specs])


def io_layout(ins, outs):
    """Layout of a step's device buffer: the inputs, the status word, then the
    results.  The host-to-device copy covers [0, in_end) -- inputs and the
    status word, which the host side keeps at zero, so each step starts with
    a cleared status -- and the device-to-host copy covers [out_begin, end) --
    the status word and the results.  Returns (offsets, in_end, out_begin, end)."""
    offs, end = _offsets(list(ins) + [("status", (1,), torch.int32)] + list(outs))
    s_off = offs["status"][0]
    return offs, s_off + 4, s_off, end


class DraftCycle:
    def __init__(self, W, E, Msel, a0, a1, B: int, L: int, P: int, use_graph: bool = True):
        dev = W.device
        self.W, self.E, self.Msel, self.a0, self.a1 = W, E, Msel, a0, a1
        self.B, self.L, self.P = B, L, P
        V, d = W.shape
        M = B * L
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
        # selection lane: hidden states and targets in; status and the path's results out
        ins = [("H", (M, d), torch.bfloat16), ("target", (B, L + 1), torch.int32)]
        outs = [("path_tok", (B, L), torch.int32), ("accept_len", (B,), torch.int32),
                ("next_token", (B,), torch.int32)]
        # one device buffer (inputs | status | results) and pinned host twins
        # of its input span and its result span
        offs, in_end, out_begin, end = io_layout(ins, outs)
        in_names = [n for n, _, _ in ins] + ["status"]
        out_names = ["status"] + [n for n, _, _ in outs]
        self._dbuf = torch.zeros(end, dtype=torch.uint8, device=dev)
        dv = _views(self._dbuf, offs, in_names + out_names[1:])
        self._din, self._dout = self._dbuf[:in_end], self._dbuf[out_begin:]
        self._hin = torch.zeros(in_end, dtype=torch.uint8, pin_memory=True)    # its status word stays 0
        self._hout = torch.zeros(end - out_begin, dtype=torch.uint8, pin_memory=True)
        # conv lane: the conv's input and previous-position rows in, its output out
        cins = [("x", (B, P, d), torch.bfloat16), ("prev", (B, d), torch.bfloat16)]
        couts = [("y", (B, P, d), torch.bfloat16)]
        self._cdin, cdin = _arena(cins, dev)
        self._cdout, cdout = _arena(couts, dev)
        self._chin, chin = _arena(cins, "cpu", pinned=True)
        self._chout, chout = _arena(couts, "cpu", pinned=True)
        self.host_in = {**_views(self._hin, offs, in_names[:-1]), **chin}
        self.host_out = {**_views(self._hout, offs, out_names, base=out_begin), **chout}
        self.H, self.target = dv["H"], dv["target"]
        self.x, self.prev, self.y = cdin["x"], cdin["prev"], cdout["y"]
        self.tok, self.acc, self.nxt = dv["path_tok"], dv["accept_len"], dv["next_token"]
        self.lp, self.ix, self.lse = e((M, 16), torch.float32), e((M, 16), torch.int32), e((M,), torch.float32)
        self.slot, self.score = e((B, L), torch.int32), e((B,), torch.float32)
        self.status = dv["status"]
        self.ws = b.workspace(M, V, d, dev)
        self._side = torch.cuda.Stream(device=dev)
        self._done = None
        self._graph = None
        if use_graph:
            self._capture()

    def kernels(self):
        """Enqueue the cycle's kernels on the current stream (device buffers)."""
        b.dflash_conv2tap(self.x, self.a0, self.a1, self.prev, y=self.y)
        self.selection_kernels()

    def selection_kernels(self):
        b.dflash_lmhead_topk(self.H, self.W, topk_logp=self.lp, topk_idx=self.ix, lse=self.lse, ws=self.ws,
                             dev_status=self.status)
        b.dflash_select_verify(self.lp, self.ix, self.E, self.Msel, self.target, self.B, self.L,
                               path_tok=self.tok, path_slot=self.slot, path_score=self.score,
                               accept_len=self.acc, next_token=self.nxt, dev_status=self.status)

    def _step(self):
        """The conv does not feed the LM head, so its lane (copy in, conv,
        copy out) runs on a side stream alongside the selection lane (copy
        in, LM head, selection + verification, copy out); the step ends when
        both have.  The conv lane starts once the selection lane's input copy
        is done, so the copy that gates the LM head has the host link to
        itself and the conv lane's copies overlap the LM head."""
        main = torch.cuda.current_stream()
        self._din.copy_(self._hin, non_blocking=True)
        self._side.wait_stream(main)
        with torch.cuda.stream(self._side):
            self._cdin.copy_(self._chin, non_blocking=True)
            b.dflash_conv2tap(self.x, self.a0, self.a1, self.prev, y=self.y)
            self._chout.copy_(self._cdout, non_blocking=True)
        self.selection_kernels()
        self._hout.copy_(self._dout, non_blocking=True)
        main.wait_stream(self._side)

    def _capture(self):
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            self._step()                      # warm-up outside capture (first-call set-up)
        cap.synchronize()
        self._graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self._graph, stream=cap):
            self._step()
        torch.cuda.current_stream().wait_stream(cap)

    def run(self):
        """One step: host inputs (self.host_in) -> device -> cycle -> host
        results.  Raises DFlashError when a kernel of the step recorded a
        device-side error (a bounded wait that ran out, a token index out of
        range): the results of such a step are not valid."""
        self.launch()
        return self.wait()

    def launch(self, stream=None):
        """Enqueue one step on `stream` (the current stream if None) without
        waiting for it; self.host_in must not change until wait() returns."""
        stream = stream or torch.cuda.current_stream()
        with torch.cuda.stream(stream):
            if self._graph is not None:
                self._graph.replay()
            else:
                self._step()
            if self._done is None:
                self._done = torch.cuda.Event()
            self._done.record(stream)

    def wait(self):
        """Wait for the step launch() enqueued and return its host results
        (raises DFlashError as run() does)."""
        self._done.synchronize()
        code = int(self.host_out["status"][0])
        if code != 0:
            raise b.DFlashError("DraftCycle.run", code)
        return self.host_out

    def io_bytes(self):
        """Bytes a step copies host-to-device and device-to-host (both lanes'
        arenas, alignment padding included)."""
        return (int(self._hin.numel() + self._chin.numel()), int(self._hout.numel() + self._chout.numel()))


class DraftPipeline:
    """Two DraftCycles over the same device-resident weights, stepping
    independent batches alternately on two streams, so that one batch's
    copies overlap the other's kernels.  Step i runs on cycle i % 2: its host
    inputs are filled after that cycle's previous step has been waited for,
    and every step's results are read back to the host.  For serving
    independent groups of blocks; a loop whose next inputs depend on the
    previous step's results uses DraftCycle.run()."""

    def __init__(self, W, E, Msel, a0, a1, B: int, L: int, P: int):
        self.cycles = [DraftCycle(W, E, Msel, a0, a1, B, L, P) for _ in range(2)]
        self.streams = [torch.cuda.Stream(device=W.device) for _ in range(2)]
        self._pending = [False, False]
        self._i = 0

    def host_in(self):
        """The host input views of the next step's cycle; waits for that
        cycle's previous step and returns its results first (None if none)."""
        k = self._i % 2
        prev = None
        if self._pending[k]:
            prev = self.cycles[k].wait()
            self._pending[k] = False
        return self.cycles[k].host_in, prev

    def launch(self):
        """Enqueue the next step (its inputs filled through host_in())."""
        k = self._i % 2
        if self._pending[k]:
            raise RuntimeError("DraftPipeline.launch: call host_in() first")
        self.cycles[k].launch(self.streams[k])
        self._pending[k] = True
        self._i += 1

    def drain(self):
        """Wait for the steps still in flight, oldest first; their results."""
        out = []
        for j in (self._i % 2, (self._i + 1) % 2):
            if self._pending[j]:
                out.append(self.cycles[j].wait())
                self._pending[j] = False
        return out

    def io_bytes(self):
        return self.cycles[0].io_bytes()
