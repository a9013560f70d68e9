"""A stack of transformer-layer products on one GPU, enqueued back to back.

This is the runner behind the benchmark and the tests of the timed
configuration: one stream, one shared workspace, every product launched with
programmatic dependent launch, and the whole step capturable as one CUDA graph.
It only arranges calls into the library (``exl3.py``); every step of every
product runs in the library's kernels.

Two ways to chain the layer's seven matrices (q, k, v, o, gate, up, down):

* ``"sweep"`` -- every matrix takes its own input rows (the 64-layer verify
  sweep: independent problems).  With ``grouped=True`` a layer is ONE grouped
  call (``exl3_gemm_grouped``): one input-rotation pre-pass and one product
  launch whose work split covers the whole layer.  With ``grouped=False`` each
  matrix is a separate call.
* ``"chain"`` -- the output of layer l feeds layer l+1, as in a decode step
  through a parallel-block transformer layer: q, k, v, gate and up take the
  layer input h (one sibling call, ``exl3_gemm_siblings``), o takes q's output
  (the stand-in for attention is the identity), down takes up's output (the
  stand-in for the activation is the identity), and down's output is the next
  layer's h.  o and down depend only on the sibling call, so with
  ``grouped=True`` they run as one grouped call: two dependent steps per
  layer (three with ``grouped=False``).

Buffers: inputs and outputs of all products live in one flat device buffer
each (x and y), a layer's slices contiguous, so an end-to-end step moves one
slice per layer between pinned host memory and the device.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from . import synth

KINDS = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass
class Product:
    spec: synth.MatrixSpec
    packed: object          # device int32 words
    scale: object
    su: object
    sv: object
    x: object               # device view (m, k_in) into Stack.x_dev
    y: object               # device view (m, n_out) into Stack.y_dev
    kind: str = ""


@dataclass
class Layer:
    index: int
    products: List[Product] = field(default_factory=list)
    x0: int = 0
    x1: int = 0
    y0: int = 0
    y1: int = 0

    def by_kind(self, kind):
        for p in self.products:
            if p.kind == kind:
                return p
        raise KeyError(kind)


class Stack:
    """The products of ``specs`` (grouped by layer in spec order) at ``m`` rows.

    ``weights``: device int32 packed words per spec (e.g. from
    ``synth.splitmix64_words_torch``).  Input rows are ``synth.small_inputs``'s
    (chained runs: its chain scales), repeated when m exceeds them (many-row
    runs).  ``large``: use the many-row call (default: m > 32).  ``run_e2e``
    moves every layer's x and y slices, so it is meant for the sweep."""

    def __init__(self, ex, torch, device, m: int, specs, weights, mode: str = "sweep",
                 grouped: bool = True, large: Optional[bool] = None):
        if mode not in ("sweep", "chain"):
            raise ValueError(mode)
        self.ex, self.torch, self.device = ex, torch, device
        self.m, self.mode = m, mode
        self.large = (m > 32) if large is None else large
        self.grouped = grouped and not self.large
        self.specs = list(specs)
        x_off, y_off, xo, yo = [], [], 0, 0
        for s in self.specs:
            x_off.append(xo)
            y_off.append(yo)
            xo += m * s.k_in
            yo += m * s.n_out
        self.x_dev = torch.empty(xo, dtype=torch.float16, device=device)
        self.y_dev = torch.empty(yo, dtype=torch.float16, device=device)
        self.x_pin = torch.empty(xo, dtype=torch.float16).pin_memory()
        self.y_pin = torch.empty(yo, dtype=torch.float16).pin_memory()
        self.products: List[Product] = []
        self.layers: List[Layer] = []
        for i, (spec, packed) in enumerate(zip(self.specs, weights)):
            scale, x, su, sv = synth.small_inputs(spec, chain=(mode == "chain"))
            if x.shape[0] < m:                  # many-row runs: the synthetic rows repeated
                x = np.tile(x, ((m + x.shape[0] - 1) // x.shape[0], 1))
            xs = slice(x_off[i], x_off[i] + m * spec.k_in)
            ys = slice(y_off[i], y_off[i] + m * spec.n_out)
            self.x_pin[xs].copy_(torch.from_numpy(np.ascontiguousarray(x[:m]).reshape(-1)))
            self.x_dev[xs].copy_(self.x_pin[xs])
            dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
            kind = spec.name.split(".")[-1]
            p = Product(spec, packed, dev(scale), dev(su), dev(sv), self.x_dev[xs].view(m, spec.k_in),
                        self.y_dev[ys].view(m, spec.n_out), kind)
            self.products.append(p)
            if not self.layers or self.layers[-1].index != spec.layer:
                self.layers.append(Layer(spec.layer, [], x_off[i], 0, y_off[i], 0))
            lay = self.layers[-1]
            lay.products.append(p)
            lay.x1 = x_off[i] + m * spec.k_in
            lay.y1 = y_off[i] + m * spec.n_out
        if mode == "chain":
            for lay in self.layers:
                kinds = sorted(p.kind for p in lay.products)
                if kinds != sorted(KINDS):
                    raise ValueError("a chained layer needs all seven matrices")
                h = lay.by_kind("q").spec
                if any(p.spec.bits != h.bits for p in lay.products):
                    raise ValueError("a chained layer has one bit width")
        self.ws = torch.zeros(self._workspace_bytes(), dtype=torch.uint8, device=device)
        self.s_in = torch.cuda.Stream(device=device)
        self.s_out = torch.cuda.Stream(device=device)
        self.packed_bytes = sum(s.packed_bytes for s in self.specs)
        self.io_bytes = sum(2 * m * (s.k_in + s.n_out) + 2 * (s.k_in + 2 * s.n_out) for s in self.specs)
        self.h2d = self.x_pin.numel() * 2
        self.d2h = self.y_pin.numel() * 2

    # ------------------------------------------------------------ sizes ---

    def _calls(self):
        """(kind, payload) of every library call one step makes, in order."""
        calls = []
        for lay in self.layers:
            if self.mode == "chain":
                P = {p.kind: p for p in lay.products}
                calls.append(("siblings", [P["q"], P["k"], P["v"], P["gate"], P["up"]]))
                if self.grouped:
                    calls.append(("grouped", [P["o"], P["down"]]))
                else:
                    calls.append(("single", P["o"]))
                    calls.append(("single", P["down"]))
            elif self.grouped:
                calls.append(("grouped", lay.products))
            else:
                calls.extend(("single", p) for p in lay.products)
        return calls

    def _workspace_bytes(self):
        ex, m, need = self.ex, self.m, 0
        for kind, pl in self._calls():
            if kind == "single":
                s = pl.spec
                if self.large:
                    n = int(ex.lib.exl3_large_m_workspace_bytes(m, s.k_in, s.n_out, s.bits))
                else:
                    n = ex.workspace_bytes(m, s.k_in, s.n_out, s.bits)
            elif kind == "siblings":
                s = pl[0].spec
                n = ex.workspace_bytes(m, s.k_in, sum(p.spec.n_out for p in pl), s.bits)
            else:
                n = ex.grouped_workspace_bytes(m, [(p.spec.k_in, p.spec.n_out) for p in pl], pl[0].spec.bits)
            need = max(need, n)
        return need

    def launches(self) -> int:
        """Kernel launches of one step (the library's own count per call)."""
        ex, m, total = self.ex, self.m, 0
        for kind, pl in self._calls():
            if kind == "single":
                s = pl.spec
                total += 3 if self.large else ex.kernel_launches(m, s.k_in, s.n_out, s.bits)
            elif kind == "siblings":
                s = pl[0].spec
                total += ex.kernel_launches(m, s.k_in, sum(p.spec.n_out for p in pl), s.bits)
            else:
                total += ex.grouped_kernel_launches(m)
        return total

    # -------------------------------------------------------------- run ---

    def _inputs_for_chain(self, li):
        """Device input rows of chained layer li: layer 0 takes its q input
        slice; layer l > 0 takes layer l-1's down output."""
        if li == 0:
            return self.layers[0].by_kind("q").x
        return self.layers[li - 1].by_kind("down").y

    def run_layer(self, li):
        ex, lay = self.ex, self.layers[li]
        if self.mode == "chain":
            P = {p.kind: p for p in lay.products}
            h = self._inputs_for_chain(li)
            q = P["q"]
            sib = [P["q"], P["k"], P["v"], P["gate"], P["up"]]
            ex.gemm_siblings(h, q.su, [(p.packed, p.scale, p.sv) for p in sib], q.spec.bits,
                             outs=[p.y for p in sib], workspace=self.ws)
            o, d = P["o"], P["down"]
            if self.grouped:
                ex.gemm_grouped([(P["q"].y, o.packed, o.scale, o.su, o.sv, o.y),
                                 (P["up"].y, d.packed, d.scale, d.su, d.sv, d.y)],
                                o.spec.bits, workspace=self.ws)
            else:
                ex.gemm(P["q"].y, o.packed, o.scale, o.su, o.sv, o.spec.bits, out=o.y, workspace=self.ws)
                ex.gemm(P["up"].y, d.packed, d.scale, d.su, d.sv, d.spec.bits, out=d.y, workspace=self.ws)
            return
        if self.grouped:
            ex.gemm_grouped([(p.x, p.packed, p.scale, p.su, p.sv, p.y) for p in lay.products],
                            lay.products[0].spec.bits, workspace=self.ws)
            return
        call = ex.gemm_large if self.large else ex.gemm
        for p in lay.products:
            call(p.x, p.packed, p.scale, p.su, p.sv, p.spec.bits, out=p.y, workspace=self.ws)

    def run(self):
        for li in range(len(self.layers)):
            self.run_layer(li)

    def _copy_chunks(self, growth: float = 1.6):
        """Layer ranges [a, b) whose inputs go up in one copy: 1, 1, 2, 3, 5, ...
        layers, each range growing by ``growth`` -- slow enough that a range has
        landed by the time the products reach it (a layer's inputs copy in about
        half the time its products take)."""
        n = len(self.layers)
        b = [0, 1]
        while b[-1] < n:
            b.append(min(n, int(b[-1] * growth) + 1))
        return list(zip(b[:-1], b[1:]))

    def _out_chunks(self):
        """{last layer of a chunk: its layer range [a, b)} for the output
        copies: the input chunks mirrored, so they shrink towards the last
        layer, whose output goes down alone."""
        n = len(self.layers)
        return {n - 1 - a: (n - b, n - a) for a, b in self._copy_chunks()}

    def run_e2e(self):
        """One end-to-end step from pinned host buffers: the inputs go up on one
        stream in growing chunks of layers (``_copy_chunks``), the products run
        on the current stream, the outputs come down on a third stream in
        chunks that shrink towards the last layer, so the copies overlap the
        products and the step ends one layer's output copy after its last
        product.  Every copy is inside the step.  Chunks rather than one copy
        per layer: each cross-stream wait in front of a product costs the
        overlap of that product with the previous one's tail (measured with 64
        layers at M = 32: 7.94 ms per step with a wait per layer, 7.66 ms with
        nine)."""
        torch = self.torch
        n = len(self.layers)
        for prev, lay in zip(self.layers, self.layers[1:]):
            assert lay.x0 == prev.x1 and lay.y0 == prev.y1, "layer slices must be contiguous"
        cs = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(cs)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        landed = {}
        with torch.cuda.stream(self.s_in):
            for a, b in self._copy_chunks():
                xs = slice(self.layers[a].x0, self.layers[b - 1].x1)
                self.x_dev[xs].copy_(self.x_pin[xs], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.s_in)
                landed[a] = ev
        out_chunks = self._out_chunks()
        for li in range(n):
            if li in landed:
                cs.wait_event(landed[li])
            self.run_layer(li)
            if li in out_chunks:
                a, b = out_chunks[li]
                ev = torch.cuda.Event()
                ev.record(cs)
                self.s_out.wait_event(ev)
                with torch.cuda.stream(self.s_out):
                    ys = slice(self.layers[a].y0, self.layers[b - 1].y1)
                    self.y_pin[ys].copy_(self.y_dev[ys], non_blocking=True)
        cs.wait_stream(self.s_in)
        cs.wait_stream(self.s_out)

    def capture(self, fn=None):
        """A CUDA graph of one step (``fn`` defaults to ``run``); the first,
        configuring call must have run outside the capture."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            (fn or self.run)()
        return g
