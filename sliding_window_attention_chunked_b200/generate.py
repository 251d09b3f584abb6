"""Prefill -> decode generation loop over a Rodimus+ mixer stack, decode steps from a CUDA graph.

SALA blog §3.3: the prompt is prefilled in chunks, then tokens are decoded one at a time with
the recurrent state updated in place and the sliding window kept in a circular buffer; §4.3
(third tip) and §4.1: decode steps are replayed from CUDA graphs to remove per-kernel launch
cost. CodeFuse Rodimus* article: Rodimus+ alternates the gated recurrence (Rodimus block) and
SW-SKA layers.

`MixerStack` holds, for N sequences, every layer's decode state: the fp32 recurrence state of
the recurrence layers and the shared-K / per-head-V ring buffers of the SW-SKA layers. One
decode step runs every layer's decode kernel on per-step inputs held in static buffers (q, k,
v, g for a recurrence layer; q, k_new, v_new for an SW-SKA layer) and then advances the token
position; `capture()` records that step once into a CUDA graph and `step()` replays it. The
inputs of a step are the caller's (here: synthetic; in a model they are the projections of the
previous layer's output). Every kernel is the library's; this module only orders the calls.
"""
from __future__ import annotations

import torch

from . import _binding as rod


class MixerStack:
    """Decode-time state of an alternating stack: layer l is a recurrence layer when l is even
    and an SW-SKA layer when l is odd."""

    def __init__(self, n_layers: int, N: int, H: int, d: int, window: int,
                 dtype=torch.bfloat16, device="cuda"):
        self.n_layers, self.N, self.H, self.d, self.W = n_layers, N, H, d, int(window)
        self.dtype, self.device = dtype, torch.device(device)
        dev, dt = self.device, dtype
        self.pos = torch.zeros(N, dtype=torch.int64, device=dev)  # position of the next token
        self.layers = []
        for l in range(n_layers):
            if self.kind(l) == "gla":
                self.layers.append(dict(
                    state=torch.zeros(N, H, d, d, dtype=torch.float32, device=dev),
                    q=torch.zeros(N, H, d, dtype=dt, device=dev),
                    k=torch.zeros(N, H, d, dtype=dt, device=dev),
                    v=torch.zeros(N, H, d, dtype=dt, device=dev),
                    g=torch.ones(N, H, d, dtype=torch.float32, device=dev),
                    o=torch.zeros(N, H, d, dtype=dt, device=dev)))
            else:
                self.layers.append(dict(
                    k_cache=torch.zeros(N, self.W, d, dtype=dt, device=dev),
                    v_cache=torch.zeros(N, H, self.W, d, dtype=dt, device=dev),
                    q=torch.zeros(N, H, d, dtype=dt, device=dev),
                    k_new=torch.zeros(N, d, dtype=dt, device=dev),
                    v_new=torch.zeros(N, H, d, dtype=dt, device=dev),
                    o=torch.zeros(N, H, d, dtype=dt, device=dev)))
        self.graph = None

    @staticmethod
    def kind(layer: int) -> str:
        return "gla" if layer % 2 == 0 else "swska"

    # ---- prefill and hand-off ------------------------------------------------------------
    def prefill(self, inputs, chunk: int = 64, stream=None):
        """inputs[l]: (q, k, v, g) with q, k, v [N,H,T,d] (g fp32) for a recurrence layer,
        (q, k, v) with q, v [N,H,T,d] and the shared k [N,T,d] for an SW-SKA layer. Runs every
        layer's prefill, leaves each recurrence layer's final state and each SW-SKA layer's
        ring buffers (last W tokens, slot = position mod W) ready for decode, and sets the next
        position to T. Returns the prefill outputs [N,H,T,d] per layer."""
        outs, T = [], None
        for l, (lay, ins) in enumerate(zip(self.layers, inputs)):
            if self.kind(l) == "gla":
                q, k, v, g = ins
                lay["state"].zero_()
                outs.append(rod.gla_prefill(q, k, v, g, lay["state"], chunk=chunk, stream=stream))
            else:
                q, k, v = ins
                outs.append(rod.swska_prefill(q, k, v, self.W, stream=stream))
                rod.swska_cache_fill(k, v, lay["k_cache"], lay["v_cache"], self.W, stream=stream)
            T = q.shape[2]
        self.pos.fill_(int(T or 0))
        return outs

    # ---- decode ----------------------------------------------------------------------------
    def set_step_inputs(self, layer: int, *tensors):
        """Copy one token's inputs of a layer into its static buffers (device copies, so they can
        run on the stream right before a replay): (q, k, v, g) [N,H,d] for a recurrence layer,
        (q, k_new [N,d], v_new [N,H,d]) for an SW-SKA layer."""
        lay = self.layers[layer]
        names = ("q", "k", "v", "g") if self.kind(layer) == "gla" else ("q", "k_new", "v_new")
        for n, t in zip(names, tensors):
            lay[n].copy_(t, non_blocking=True)

    def step_eager(self, stream=None):
        """One decode token for every sequence through every layer, then position + 1."""
        for l, lay in enumerate(self.layers):
            if self.kind(l) == "gla":
                rod.gla_decode_step(lay["q"], lay["k"], lay["v"], lay["g"], lay["state"], o=lay["o"],
                                    stream=stream)
            else:
                rod.swska_decode(lay["q"], lay["k_new"], lay["v_new"], lay["k_cache"], lay["v_cache"],
                                 self.pos, self.W, o=lay["o"], stream=stream)
        self.pos.add_(1)

    def capture(self):
        """Record one decode step into a CUDA graph (after one eager step has run on this device,
        so that every kernel attribute and launch plan is already set up)."""
        s = torch.cuda.Stream(device=self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                self.step_eager()
        torch.cuda.current_stream(self.device).wait_stream(s)
        self.graph = g
        return g

    def step(self):
        """Replay the captured decode step (capture() first)."""
        if self.graph is None:
            raise RuntimeError("capture() has not been called")
        self.graph.replay()

    def kernels_per_step(self) -> int:
        """Library kernel launches in one decode step (one per layer)."""
        return self.n_layers

    def outputs(self):
        return [lay["o"] for lay in self.layers]
