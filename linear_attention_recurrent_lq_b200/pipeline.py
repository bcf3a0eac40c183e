"""Decode windows fed from, and read back to, pinned host memory, with the
transfers overlapped with the kernels.

Each layer-state of a step has device input buffers (q, k, v, beta, decay
for W tokens), a device output buffer, and pinned host copies of both.  Per
layer l, the upload stream copies l's inputs host->device, the compute
stream runs l's window (W decode calls and the window flush, captured as one
CUDA graph per layer) once they have landed, and the download stream copies
l's outputs back once the window has written them.  So layer l+1's upload
and layer l-1's download run while layer l computes, on the GPU's separate
copy engines.  Buffers are reused from step to step, ordered by events: an
upload waits for the previous step's window to be done with that layer's
input buffers, a window for the previous step's download of its output
buffer.
"""
from __future__ import annotations

from dataclasses import dataclass, field

NAMES = ("q", "k", "v", "beta", "decay")


@dataclass
class Layer:
    state: object          # an LQState
    dev_in: dict           # name -> device tensor [W, ...]
    dev_out: object        # device tensor [W, rows, H, dv]
    host_in: dict          # name -> pinned host tensor, same shapes
    host_out: object       # pinned host tensor, same shape as dev_out
    graph: object = field(default=None)


class HostIOPipeline:
    def __init__(self, layers: list[Layer], window: int, flush: bool = True):
        import torch
        self.torch = torch
        self.layers = layers
        self.window = window
        self.flush = flush
        self.up = torch.cuda.Stream()
        self.comp = torch.cuda.Stream()
        self.down = torch.cuda.Stream()
        n = len(layers)
        self.up_done = [torch.cuda.Event() for _ in range(n)]
        self.comp_done = [torch.cuda.Event() for _ in range(n)]
        self.down_done = [torch.cuda.Event() for _ in range(n)]

    def _window(self, lay: Layer):
        x = lay.dev_in
        for t in range(self.window):
            lay.state.step(x["q"][t], x["k"][t], x["v"][t], x["beta"][t], x["decay"][t], lay.dev_out[t])
        if self.flush:
            lay.state.flush()

    def capture(self):
        """One graph per layer (run once eagerly first, which also sets the
        kernels' launch attributes outside the capture)."""
        torch = self.torch
        with torch.cuda.stream(self.comp):
            for lay in self.layers:
                self._window(lay)
        torch.cuda.synchronize()
        for lay in self.layers:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.comp):
                self._window(lay)
            lay.graph = g
        torch.cuda.synchronize()

    def bytes_per_step(self) -> tuple[int, int]:
        h2d = sum(t.numel() * t.element_size() for lay in self.layers for t in lay.host_in.values())
        d2h = sum(lay.host_out.numel() * lay.host_out.element_size() for lay in self.layers)
        return h2d, d2h

    def step(self):
        """Enqueue one step: every layer's upload, window and download."""
        torch = self.torch
        for i, lay in enumerate(self.layers):
            with torch.cuda.stream(self.up):
                self.up.wait_event(self.comp_done[i])
                for name in NAMES:
                    lay.dev_in[name].copy_(lay.host_in[name], non_blocking=True)
                self.up_done[i].record(self.up)
            with torch.cuda.stream(self.comp):
                self.comp.wait_event(self.up_done[i])
                self.comp.wait_event(self.down_done[i])
                lay.graph.replay()
                self.comp_done[i].record(self.comp)
            with torch.cuda.stream(self.down):
                self.down.wait_event(self.comp_done[i])
                lay.host_out.copy_(lay.dev_out, non_blocking=True)
                self.down_done[i].record(self.down)

    def join(self, stream=None):
        """Make `stream` (default: the current one) wait for all enqueued work."""
        torch = self.torch
        s = stream or torch.cuda.current_stream()
        for ev in (self.up_done[-1], self.comp_done[-1], self.down_done[-1]):
            s.wait_event(ev)

    def fork(self, stream=None):
        """Make the three streams wait for the work enqueued so far on `stream`."""
        torch = self.torch
        s = stream or torch.cuda.current_stream()
        ev = torch.cuda.Event()
        ev.record(s)
        for st in (self.up, self.comp, self.down):
            st.wait_event(ev)
