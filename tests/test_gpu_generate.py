"""Prefill -> decode hand-off and the CUDA-graph decode loop, against the oracle.

SALA blog §3.3: a prompt is prefilled, then tokens are decoded one at a time from the
recurrent state and the circular window buffer. The ring-buffer fill is byte work, so the GPU
caches must equal the oracle's bit for bit. Decoding positions T, T+1, ... after a T-token
prefill must reproduce the rows of a prefill over the whole sequence (the oracle's), and a
decode step replayed from a CUDA graph must give exactly what the same step gives eagerly.
"""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_attention_chunked_b200 as rod
from sliding_window_attention_chunked_b200 import workloads as wl
from sliding_window_attention_chunked_b200.generate import MixerStack

from .parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("T,W,d", [(5, 8, 128), (8, 8, 128), (300, 64, 128), (77, 1, 64),
                                   (1000, 96, 32)])
def test_cache_fill_matches_oracle_bit_exact(T, W, d):
    B, H = 2, 3
    _, k, v = wl.swska_inputs(B, H, T, d, d, seed=T + W)
    kc = torch.full((B, W, d), 3.0, dtype=torch.bfloat16)
    vc = torch.full((B, H, W, d), 3.0, dtype=torch.bfloat16)
    kc_ref, vc_ref = oracle.swska_cache_fill(k, v, kc, vc, W)
    kg, vg = kc.to(DEV), vc.to(DEV)
    rod.swska_cache_fill(k.to(DEV), v.to(DEV), kg, vg, W)
    rod.check()
    np.testing.assert_array_equal(kg.float().cpu().numpy(), kc_ref)
    np.testing.assert_array_equal(vg.float().cpu().numpy(), vc_ref)


def test_cache_fill_fp32_and_empty():
    B, H, T, W, d = 1, 2, 40, 16, 16
    _, k, v = wl.swska_inputs(B, H, T, d, d, seed=3, dtype="fp32")
    kc = torch.zeros(B, W, d)
    vc = torch.zeros(B, H, W, d)
    kc_ref, vc_ref = oracle.swska_cache_fill(k, v, kc, vc, W)
    kg, vg = kc.to(DEV), vc.to(DEV)
    rod.swska_cache_fill(k.to(DEV), v.to(DEV), kg, vg, W)
    rod.swska_cache_fill(k[:, :0].to(DEV).contiguous(), v[:, :, :0].to(DEV).contiguous(),
                         kg, vg, W)  # T = 0: nothing happens
    rod.check()
    np.testing.assert_array_equal(kg.cpu().numpy(), kc_ref)
    np.testing.assert_array_equal(vg.cpu().numpy(), vc_ref)


def _stack_inputs(L, N, H, T, d, seed):
    ins = []
    for l in range(L):
        if MixerStack.kind(l) == "gla":
            ins.append(wl.gla_inputs(N, H, T, d, d, dist="l2", seed=seed + l))
        else:
            ins.append(wl.swska_inputs(N, H, T, d, d, seed=seed + l))
    return ins


def _token(ins, kind, t):
    """The inputs of position t of one layer, on the device."""
    if kind == "gla":
        q, k, v, g = ins
        return [x[:, :, t].contiguous().to(DEV) for x in (q, k, v, g)]
    q, k, v = ins
    return [q[:, :, t].contiguous().to(DEV), k[:, t].contiguous().to(DEV),
            v[:, :, t].contiguous().to(DEV)]


def test_generation_loop_continues_the_prefill():
    """A 4-layer stack: prefill T tokens on the GPU, then decode S more, the first step eagerly
    and the rest from the captured graph; every decode output equals the oracle's prefill of the
    whole T + S sequence at that position (recurrence: o_t = q_t S_t; SW-SKA: window rows)."""
    L, N, H, d, W, T, S = 4, 2, 4, 128, 64, 150, 6
    ins = _stack_inputs(L, N, H, T + S, d, seed=500)
    ref = []
    for l in range(L):
        if MixerStack.kind(l) == "gla":
            ref.append(oracle.gla_prefill(*ins[l])[0])
        else:
            ref.append(oracle.swska_prefill(*ins[l], W))
    stack = MixerStack(L, N, H, d, W)
    pre = [tuple(x[:, :, :T].contiguous().to(DEV) if x.dim() == 4 else x[:, :T].contiguous().to(DEV)
                 for x in lay) for lay in ins]
    outs = stack.prefill(pre)
    rod.check()
    for l in range(L):
        compare(outs[l], ref[l][:, :, :T], "bf16", f"prefill layer {l}")
    for s in range(S):
        for l in range(L):
            stack.set_step_inputs(l, *_token(ins[l], MixerStack.kind(l), T + s))
        if s == 0:
            stack.step_eager()
            torch.cuda.synchronize()
            got = [o.clone() for o in stack.outputs()]
            stack.capture()
        else:
            stack.step()
            got = [o.clone() for o in stack.outputs()]
        rod.check()
        for l in range(L):
            compare(got[l], ref[l][:, :, T + s], "bf16", f"decode step {s} layer {l}")
    assert int(stack.pos[0]) == T + S


def test_graph_replay_equals_eager_step():
    L, N, H, d, W, T, S = 2, 3, 2, 128, 32, 40, 4
    ins = _stack_inputs(L, N, H, T + S, d, seed=700)
    pre = [tuple(x[:, :, :T].contiguous().to(DEV) if x.dim() == 4 else x[:, :T].contiguous().to(DEV)
                 for x in lay) for lay in ins]
    eager, graphed = MixerStack(L, N, H, d, W), MixerStack(L, N, H, d, W)
    eager.prefill(pre)
    graphed.prefill(pre)
    for s in range(S):
        for stk in (eager, graphed):
            for l in range(L):
                stk.set_step_inputs(l, *_token(ins[l], MixerStack.kind(l), T + s))
        eager.step_eager()
        if s == 0:
            graphed.step_eager()
            graphed.capture()
        else:
            graphed.step()
        torch.cuda.synchronize()
        for a, b in zip(eager.outputs(), graphed.outputs()):
            assert torch.equal(a, b)
    rod.check()
    for la, lb in zip(eager.layers, graphed.layers):
        for key in la:
            assert torch.equal(la[key], lb[key]), key
    assert torch.equal(eager.pos, graphed.pos)
