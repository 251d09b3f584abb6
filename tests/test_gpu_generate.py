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


# ------------------------------------------------------------------------------------------
# paged window cache
# ------------------------------------------------------------------------------------------


@pytest.mark.parametrize("N,H,W,page,full", [(3, 16, 4096, 64, True), (2, 16, 4096, 8, False),
                                             (5, 4, 512, 128, True), (1, 16, 2048, 2048, True),
                                             (7, 3, 96, 16, False)])
def test_swska_decode_paged_matches_oracle(N, H, W, page, full):
    """Random pool contents, a shuffled block table with spare pages, full and partial windows:
    outputs within the bf16 tolerance, pools bit-exact after the new tokens are written."""
    d = 128
    dd = wl.decode_inputs(N, H, d, d, W, seed=N + W + page, dtype="bf16", full=full)
    pps = W // page
    P = N * pps + 5
    g = torch.Generator().manual_seed(W + page)
    k_pool = torch.randn(P, page, d, generator=g).to(torch.bfloat16)
    v_pool = torch.randn(P, H, page, d, generator=g).to(torch.bfloat16)
    table = torch.randperm(P, generator=g)[:N * pps].to(torch.int32).reshape(N, pps)
    ref, kp_ref, vp_ref = oracle.swska_decode_paged(dd["sq"], dd["k_new"], dd["v_new"], k_pool,
                                                    v_pool, table, page, dd["pos"], W)
    kp, vp = k_pool.to(DEV), v_pool.to(DEV)
    o = rod.swska_decode_paged(dd["sq"].to(DEV), dd["k_new"].to(DEV), dd["v_new"].to(DEV), kp, vp,
                               table.to(DEV), page, dd["pos"].to(DEV), W)
    rod.check()
    compare(o, ref, "bf16", "paged o")
    np.testing.assert_array_equal(kp.float().cpu().numpy(), kp_ref)
    np.testing.assert_array_equal(vp.float().cpu().numpy(), vp_ref)


def test_swska_decode_paged_identity_table_equals_ring():
    """With the pool laid out as [N*pages][page] and the identity table, the K pool is the ring
    buffer itself: paged and ring decode give the same outputs bit for bit."""
    N, H, d, W, page = 4, 16, 128, 1024, 128
    dd = wl.decode_inputs(N, H, d, d, W, seed=9, dtype="bf16", full=True)
    pps = W // page
    kc, vc = dd["k_cache"].to(DEV), dd["v_cache"].to(DEV)
    k_pool = kc.reshape(N * pps, page, d).clone()
    v_pool = vc.reshape(N, H, pps, page, d).permute(0, 2, 1, 3, 4).reshape(N * pps, H, page, d).contiguous()
    table = torch.arange(N * pps, dtype=torch.int32, device=DEV).reshape(N, pps)
    args = (dd["sq"].to(DEV), dd["k_new"].to(DEV), dd["v_new"].to(DEV))
    pos = dd["pos"].to(DEV)
    o_ring = rod.swska_decode(*args, kc, vc, pos, W)
    o_paged = rod.swska_decode_paged(*args, k_pool, v_pool, table, page, pos, W)
    rod.check()
    assert torch.equal(o_ring, o_paged)
    assert torch.equal(kc.reshape(N * pps, page, d), k_pool)
