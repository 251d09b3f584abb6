"""GPU parity: every entry point of librod.so against the fp64 CPU oracle on the same seeded
inputs, through the C ABI (via the ctypes binding), with the tolerances in tests/parity.py.

Sizes: small cases the oracle finishes in seconds that still span several tiles and a ragged
tail, the edge cases of the method (T = 1, T < chunk, W = 1, W >= T, g = 0, g = 1, partially
filled decode windows, a negative decode position), and the full workload sizes in the launch
configuration the benchmark times, checked on sampled outputs the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_attention_chunked_b200 as rod
from sliding_window_attention_chunked_b200 import workloads as wl

from .parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cuda(*ts):
    return [t.to(DEV) for t in ts]


# ------------------------------------------------------------------------------------------
# gated linear recurrence: prefill
# ------------------------------------------------------------------------------------------


def _gla_check(B, H, T, dk, dv, chunk, dtype, dist, seed=0, state0_scale=0.0, gate=None):
    q, k, v, g = wl.gla_inputs(B, H, T, dk, dv, dist=dist, seed=seed, dtype=dtype)
    if gate is not None:
        g = torch.full_like(g, float(gate))
    S0 = torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(seed + 7)) * state0_scale
    o_ref, S_ref = oracle.gla_prefill(q, k, v, g, S0)
    qd, kd, vd, gd = _cuda(q, k, v, g)
    S = S0.to(DEV).contiguous()
    o = rod.gla_prefill(qd, kd, vd, gd, S, chunk=chunk)
    rod.check()
    compare(o, o_ref, dtype, "o")
    compare(S, S_ref, dtype, "state")
    return o, S


def test_gla_prefill_tiny_fp32():
    d = wl.WORKLOADS["tiny_fp32"].dims
    _gla_check(d["B"], d["H"], d["T"], d["dk"], d["dv"], d["chunk"], "fp32", "tiny")


@pytest.mark.parametrize("dk,dv", [(16, 32), (32, 16), (64, 64), (128, 128), (16, 128)])
def test_gla_prefill_fp32_dims(dk, dv):
    _gla_check(2, 2, 77, dk, dv, 32, "fp32", "tiny", seed=dk + dv, state0_scale=0.5)


def test_gla_prefill_bf16_ragged_with_initial_state():
    _gla_check(2, 3, 1000, 128, 128, 64, "bf16", "l2", seed=1, state0_scale=0.3)


@pytest.mark.parametrize("T", [1, 17, 64, 65])
def test_gla_prefill_bf16_short(T):
    _gla_check(1, 2, T, 128, 128, 64, "bf16", "l2", seed=T)


@pytest.mark.parametrize("chunk", [16, 32, 128])
def test_gla_prefill_bf16_chunk_sizes_cuda_core_kernel(chunk):
    """Chunk sizes other than 64 run the sequential CUDA-core kernel (only bf16, d = 128,
    chunk 64 takes the tensor-core path): the chunk size must not change the result."""
    _gla_check(1, 2, 300, 128, 128, chunk, "bf16", "l2", seed=chunk)


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64)])
def test_gla_prefill_gate_zero_resets(dk, dv):
    _gla_check(1, 2, 130, dk, dv, 64, "bf16", "l2", seed=3, gate=0.0)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_gla_prefill_gate_one_linear_attention(dk, dv):
    _gla_check(1, 2, 130, dk, dv, 64, "bf16", "l2", seed=4, gate=1.0)


def test_gla_prefill_mixed_strong_and_mild_decay():
    """Chunks where a channel decays below 2^-60 take the exact CUDA-core path for the
    intra-chunk scores; the others use the tensor cores. Both must agree with the oracle."""
    B, H, T, d = 1, 2, 700, 128
    q, k, v, g = wl.gla_inputs(B, H, T, d, d, dist="l2", seed=31)
    g[:, :, 100:110, 5] = 1e-9     # chunk 1: strong decay in one channel
    g[:, 1, 400:464, :] = 0.3      # chunk 6 of head 1: every channel decays hard
    g[:, 0, 650, 77] = 0.0         # an exact zero gate in the tail chunk
    o_ref, S_ref = oracle.gla_prefill(q, k, v, g)
    S = torch.zeros(B, H, d, d, device=DEV)
    o = rod.gla_prefill(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), S, chunk=64)
    rod.check()
    compare(o, o_ref, "bf16", "o")
    compare(S, S_ref, "bf16", "state")


@pytest.mark.parametrize("B,H,T", [(1, 2, 5000), (1, 1, 64 * 40 + 3), (3, 5, 777), (5, 14, 700)])
def test_gla_prefill_many_segments(B, H, T):
    """Small B*H spreads the sequence over many segments (segment pass + state scan); at B5 H14
    the segment pass cuts each segment into two pieces and the scan chains the pieces."""
    _gla_check(B, H, T, 128, 128, 64, "bf16", "l2", seed=T, state0_scale=0.2)


@pytest.mark.parametrize("gates", ["one", "one_minus_2^-10", "sigmoid(N(8,1))"])
def test_gla_prefill_long_sequence_gates_near_one(gates):
    """Gates at or near 1 over a long sequence (g = 1 is linear attention, SALA blog §2.2): the
    state sums thousands of k^T v terms and grows with T, the regime where the readout's bf16
    copy of the state would be most likely to lose accuracy. B1 H2 T16384 cuts each head into
    many segments, so the segment pass, the scan and the output pass all run. v is scaled by
    sqrt(128 / T) so that outputs and states stay O(1) and the absolute bound keeps its
    meaning; relative accuracy, which is what the long state tests, does not depend on it."""
    B, H, T, d = 1, 2, 16384, 128
    q, k, v, g = wl.gla_inputs(B, H, T, d, d, dist="l2", seed=61)
    v = (v.float() * (128.0 / T) ** 0.5).to(v.dtype)
    if gates == "one":
        g = torch.ones_like(g)
    elif gates == "one_minus_2^-10":
        g = torch.full_like(g, 1.0 - 2.0 ** -10)
    else:
        gen = torch.Generator().manual_seed(62)
        g = torch.sigmoid(torch.randn(g.shape, generator=gen) + 8.0)
    assert rod.gla_prefill_workspace_size(B, H, T, d, d, 64) > 0  # several segments
    o_ref, S_ref = oracle.gla_prefill(q, k, v, g)
    S = torch.zeros(B, H, d, d, device=DEV)
    o = rod.gla_prefill(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), S, chunk=64)
    rod.check()
    compare(o, o_ref, "bf16", f"o ({gates})")
    compare(S, S_ref, "bf16", f"state ({gates})")


def test_gla_prefill_deterministic():
    q, k, v, g = [t.to(DEV) for t in wl.gla_inputs(1, 4, 3000, 128, 128, dist="l2", seed=32)]
    S1 = torch.zeros(1, 4, 128, 128, device=DEV)
    S2 = torch.zeros_like(S1)
    o1 = rod.gla_prefill(q, k, v, g, S1)
    o2 = rod.gla_prefill(q, k, v, g, S2)
    rod.check()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_gla_prefill_split_hands_off_state():
    B, H, T, d = 1, 2, 500, 128
    q, k, v, g = [t.to(DEV) for t in wl.gla_inputs(B, H, T, d, d, dist="l2", seed=5)]
    S = torch.zeros(B, H, d, d, device=DEV)
    o = rod.gla_prefill(q, k, v, g, S)
    S2 = torch.zeros_like(S)
    o1 = rod.gla_prefill(q[:, :, :211].contiguous(), k[:, :, :211].contiguous(),
                         v[:, :, :211].contiguous(), g[:, :, :211].contiguous(), S2)
    o2 = rod.gla_prefill(q[:, :, 211:].contiguous(), k[:, :, 211:].contiguous(),
                         v[:, :, 211:].contiguous(), g[:, :, 211:].contiguous(), S2)
    rod.check()
    compare(torch.cat([o1, o2], dim=2), o.float(), "bf16", "split o")
    compare(S2, S, "bf16", "split state")


def test_gla_prefill_full_workload():
    """B=4, T=4096, H=16, d=128, chunk 64, bf16 in / fp32 state: every output vs the oracle."""
    d = wl.WORKLOADS["gla_prefill_b4_t4096"].dims
    _gla_check(d["B"], d["H"], d["T"], d["dk"], d["dv"], d["chunk"], "bf16", "l2")


# ------------------------------------------------------------------------------------------
# gated linear recurrence: decode
# ------------------------------------------------------------------------------------------


# dv = 128 with few (n, h) pairs splits the columns over 4 (N H <= 64) or 2 (<= 128) CTAs
@pytest.mark.parametrize("dtype,N,H,dk,dv", [("fp32", 3, 2, 16, 32), ("fp32", 5, 3, 128, 64),
                                             ("bf16", 256, 16, 128, 128), ("bf16", 1, 16, 128, 128),
                                             ("fp32", 2, 3, 64, 128), ("bf16", 5, 20, 128, 128)])
def test_gla_decode_step(dtype, N, H, dk, dv):
    dd = wl.decode_inputs(N, H, dk, dv, 8, seed=N + dk, dtype=dtype)
    o_ref, S_ref = oracle.gla_decode_step(dd["q"], dd["k"], dd["v"], dd["g"], dd["state"])
    q, k, v, g, S = _cuda(dd["q"], dd["k"], dd["v"], dd["g"], dd["state"])
    o = rod.gla_decode_step(q, k, v, g, S)
    rod.check()
    compare(o, o_ref, dtype, "o")
    compare(S, S_ref, dtype, "state")


def test_gla_decode_steps_equal_prefill_fp32():
    B, H, T, dk, dv = 2, 2, 40, 32, 16
    q, k, v, g = [t.to(DEV) for t in wl.gla_inputs(B, H, T, dk, dv, dist="tiny", seed=9,
                                                   dtype="fp32")]
    S_pre = torch.zeros(B, H, dk, dv, device=DEV)
    o_pre = rod.gla_prefill(q, k, v, g, S_pre, chunk=16)
    S = torch.zeros_like(S_pre)
    outs = [rod.gla_decode_step(q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                v[:, :, t].contiguous(), g[:, :, t].contiguous(), S)
            for t in range(T)]
    rod.check()
    compare(torch.stack(outs, dim=2), o_pre, "fp32", "decode vs prefill o")
    compare(S, S_pre, "fp32", "decode vs prefill state")


# ------------------------------------------------------------------------------------------
# SW-SKA prefill
# ------------------------------------------------------------------------------------------


def _ska_check(B, H, T, dk, dv, W, dtype, dist, seed=0, rows=None, scale=None):
    q, k, v = wl.swska_inputs(B, H, T, dk, dv, dist=dist, seed=seed, dtype=dtype)
    qd, kd, vd = _cuda(q, k, v)
    o = rod.swska_prefill(qd, kd, vd, W, scale=scale)
    rod.check()
    if rows is None:
        ref = oracle.swska_prefill(q, k, v, W, scale=scale)
        compare(o, ref, dtype, "o")
    else:
        ref = oracle.swska_prefill(q, k, v, W, scale=scale, rows=rows)
        compare(o.reshape(-1, dv)[torch.as_tensor(rows, device=DEV)], ref, dtype, "o rows")
    return o


def test_swska_prefill_tiny_fp32():
    d = wl.WORKLOADS["tiny_fp32"].dims
    _ska_check(d["B"], d["H"], d["T"], d["dk"], d["dv"], d["window"], "fp32", "tiny")


@pytest.mark.parametrize("dk,dv,W", [(16, 32, 1), (32, 16, 7), (64, 64, 100), (128, 128, 300),
                                     (16, 128, 1000)])
def test_swska_prefill_fp32_dims(dk, dv, W):
    _ska_check(2, 2, 333, dk, dv, W, "fp32", "tiny", seed=dk + W)


def test_swska_prefill_bf16_ragged():
    _ska_check(2, 3, 1500, 128, 128, 300, "bf16", "normal", seed=2)


@pytest.mark.parametrize("T,W", [(1, 4096), (130, 1), (200, 4096), (700, 129), (700, 128)])
def test_swska_prefill_bf16_edges(T, W):
    _ska_check(1, 2, T, 128, 128, W, "bf16", "normal", seed=T + W)


def test_swska_prefill_window_one_is_v():
    q, k, v = [t.to(DEV) for t in wl.swska_inputs(1, 2, 257, 128, 128, seed=3)]
    o = rod.swska_prefill(q, k, v, 1)
    rod.check()
    assert torch.equal(o, v)


def test_swska_prefill_full_workload_sampled():
    """B=2, T=32768, H=16, d=128, W=4096, scale 1/sqrt(128): the whole launch runs; the first
    W rows of (b=0, h=0) (sub-sampled) and random rows elsewhere are checked one by one."""
    d = wl.WORKLOADS["swska_prefill_b2_t32768"].dims
    B, H, T, W = d["B"], d["H"], d["T"], d["window"]
    r = np.random.default_rng(0)
    rows = np.concatenate([np.arange(0, W + 256, 37),
                           r.integers(0, B * H * T, 512),
                           [B * H * T - 1, T - 1, T, (B * H - 1) * T]])
    _ska_check(B, H, T, d["dk"], d["dv"], W, "bf16", "normal", rows=np.unique(rows))


# ------------------------------------------------------------------------------------------
# SW-SKA decode (ring buffer)
# ------------------------------------------------------------------------------------------


def _ska_decode_check(N, H, dk, dv, W, dtype, full, seed=0, check_n=None):
    dd = wl.decode_inputs(N, H, dk, dv, W, seed=seed, dtype=dtype, full=full)
    sq, kn, vn, kc, vc, pos = _cuda(dd["sq"], dd["k_new"], dd["v_new"], dd["k_cache"],
                                    dd["v_cache"], dd["pos"])
    o = rod.swska_decode(sq, kn, vn, kc, vc, pos, W)
    rod.check()
    sel = np.arange(N) if check_n is None else np.unique(
        np.concatenate([np.arange(min(4, N)), np.random.default_rng(seed).integers(0, N, check_n)]))
    ref, kc_ref, vc_ref = oracle.swska_decode(dd["sq"][sel], dd["k_new"][sel], dd["v_new"][sel],
                                              dd["k_cache"][sel], dd["v_cache"][sel],
                                              dd["pos"][sel], W)
    compare(o[torch.as_tensor(sel, device=DEV)], ref, dtype, "o")
    # the ring-buffer write is a copy: bit-exact
    s = torch.as_tensor(sel, device=DEV)
    np.testing.assert_array_equal(kc[s].float().cpu().numpy(), kc_ref)
    np.testing.assert_array_equal(vc[s].float().cpu().numpy(), vc_ref)


def test_swska_decode_tiny_fp32():
    _ska_decode_check(5, 2, 16, 32, 64, "fp32", full=False, seed=1)


@pytest.mark.parametrize("W", [600, 1030])
def test_swska_decode_bf16_cluster_split(W):
    _ska_decode_check(7, 4, 128, 128, W, "bf16", full=False, seed=W)
    _ska_decode_check(7, 4, 128, 128, W, "bf16", full=True, seed=W + 1)


@pytest.mark.parametrize("H", [1, 3, 16, 20])
def test_swska_decode_bf16_heads(H):
    """H <= 16 runs one warp per head, H = 20 the general kernel: both against the oracle."""
    _ska_decode_check(6, H, 128, 128, 300, "bf16", full=False, seed=40 + H)
    _ska_decode_check(6, H, 128, 128, 300, "bf16", full=True, seed=50 + H)


@pytest.mark.parametrize("W", [1, 2, 7, 8, 9, 17])
def test_swska_decode_bf16_small_windows(W):
    """Windows shorter than, equal to and just past one stage of slots; W = 1 gives o = v_new."""
    _ska_decode_check(9, 2, 128, 128, W, "bf16", full=False, seed=60 + W)
    _ska_decode_check(9, 2, 128, 128, W, "bf16", full=True, seed=70 + W)


@pytest.mark.parametrize("N,H,W", [(1, 16, 4096), (2, 16, 4096), (3, 12, 1000), (1, 3, 4096),
                                   (5, 16, 2048), (12, 16, 4096), (16, 16, 4096), (32, 16, 4096)])
def test_swska_decode_bf16_small_batches(N, H, W):
    """Small batches split the heads over CTAs (K read once per head group) and the window over
    clusters of up to 16 CTAs: full and partially filled windows against the oracle."""
    _ska_decode_check(N, H, 128, 128, W, "bf16", full=True, seed=80 + N + H)
    _ska_decode_check(N, H, 128, 128, W, "bf16", full=False, seed=90 + N + H)


@pytest.mark.parametrize("N", [1, 4, 16, 48])
def test_swska_decode_repeatable(N):
    """Thirty identical calls give bit-identical outputs. For a fixed launch shape the decode is
    deterministic, so a stage read before its copies landed (a broken ring hand-off between the
    consumer warps that share a head) would show as a mismatch; the first call is also checked
    against the oracle."""
    H, W = 16, 4096
    dd = wl.decode_inputs(N, H, 128, 128, W, seed=300 + N, dtype="bf16", full=True)
    o_ref, _, _ = oracle.swska_decode(dd["sq"], dd["k_new"], dd["v_new"], dd["k_cache"], dd["v_cache"],
                                      dd["pos"], W)
    sq, kn, vn, kc, vc, p = _cuda(dd["sq"], dd["k_new"], dd["v_new"], dd["k_cache"], dd["v_cache"],
                                  dd["pos"])
    first = rod.swska_decode(sq, kn, vn, kc, vc, p, W)
    rod.check()
    compare(first, o_ref, "bf16", f"swska_decode N{N}")
    for _ in range(30):
        o = rod.swska_decode(sq, kn, vn, kc, vc, p, W)
        assert torch.equal(o, first)
    rod.check()


def test_swska_decode_full_workload_sampled():
    d = wl.WORKLOADS["decode_n256"].dims
    _ska_decode_check(d["N"], d["H"], d["dk"], d["dv"], d["window"], "bf16", full=True,
                      check_n=20)


@pytest.mark.parametrize("d", [64, 128])
def test_swska_decode_negative_position_gives_nan_and_keeps_cache(d):
    N, H, W = 3, 2, 32
    dd = wl.decode_inputs(N, H, d, d, W, seed=5, dtype="bf16", full=False)
    pos = dd["pos"].clone()
    pos[1] = -5
    sq, kn, vn, kc, vc, p = _cuda(dd["sq"], dd["k_new"], dd["v_new"], dd["k_cache"],
                                  dd["v_cache"], pos)
    kc0, vc0 = kc.clone(), vc.clone()
    o = rod.swska_decode(sq, kn, vn, kc, vc, p, W)
    rod.check()
    assert torch.isnan(o[1].float()).all()
    assert torch.isfinite(o[0].float()).all() and torch.isfinite(o[2].float()).all()
    assert torch.equal(kc[1], kc0[1]) and torch.equal(vc[1], vc0[1])


def test_swska_decode_equals_prefill_rows():
    """Fill the ring from a prefix of one sequence and decode position P: equals prefill row P."""
    H, d, W, T = 4, 128, 96, 400
    q, k, v = [t.to(DEV) for t in wl.swska_inputs(1, H, T, d, d, seed=8)]
    o_pre = rod.swska_prefill(q, k, v, W)
    positions = [0, 5, 95, 96, 97, 250, 399]
    N = len(positions)
    kc = torch.zeros(N, W, d, device=DEV, dtype=q.dtype)
    vc = torch.zeros(N, H, W, d, device=DEV, dtype=q.dtype)
    for n, P in enumerate(positions):
        for p in range(max(0, P - W + 1), P):
            kc[n, p % W] = k[0, p]
            vc[n, :, p % W] = v[0, :, p]
    P = torch.tensor(positions, device=DEV)
    o = rod.swska_decode(q[0][:, P].transpose(0, 1).contiguous(), k[0, P].contiguous(),
                         v[0][:, P].transpose(0, 1).contiguous(), kc, vc, P, W)
    rod.check()
    compare(o, o_pre[0][:, P].transpose(0, 1).float(), "bf16", "decode vs prefill")


# ------------------------------------------------------------------------------------------
# long-context stack: one layer of each kind at full length, sampled
# ------------------------------------------------------------------------------------------


def test_stack_layers_full_length_sampled():
    d = wl.WORKLOADS["stack_t131072"].dims
    B, H, T, dk, dv, W = d["B"], d["H"], d["T"], d["dk"], d["dv"], d["window"]
    # layer 0: recurrence, every head on the GPU; head 0 and head H-1 vs the oracle in full
    q, k, v, g = wl.stack_layer_inputs(0, B, H, T, dk, dv, device=DEV)
    S = torch.zeros(B, H, dk, dv, device=DEV)
    o = rod.gla_prefill(q, k, v, g, S, chunk=d["chunk"])
    rod.check()
    for h in (0, H - 1):
        o_ref, S_ref = oracle.gla_prefill(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], g[:, h:h + 1])
        compare(o[:, h:h + 1], o_ref, "bf16", f"stack gla head {h}")
        compare(S[:, h:h + 1], S_ref, "bf16", f"stack gla state head {h}")
    del q, k, v, g, o
    # layer 1: SW-SKA, sampled rows
    q, k, v = wl.stack_layer_inputs(1, B, H, T, dk, dv, device=DEV)
    o = rod.swska_prefill(q, k, v, W)
    rod.check()
    rows = np.unique(np.concatenate([np.arange(0, 300, 7),
                                     np.random.default_rng(1).integers(0, B * H * T, 400)]))
    ref = oracle.swska_prefill(q, k, v, W, rows=rows)
    compare(o.reshape(-1, dv)[torch.as_tensor(rows, device=DEV)], ref, "bf16", "stack swska")


# ------------------------------------------------------------------------------------------
# tensor-core SW-SKA specifics: lazy rescaling, odd head counts, tile edges, determinism
# ------------------------------------------------------------------------------------------


@pytest.mark.parametrize("qscale", [4.0, 16.0])
def test_swska_prefill_large_logits_exercise_rescaling(qscale):
    """Scores with a spread of many units of log2 force the running-maximum rescale path."""
    B, H, T, d, W = 1, 2, 1100, 128, 700
    q, k, v = wl.swska_inputs(B, H, T, d, d, seed=21)
    q = (q.float() * qscale).to(torch.bfloat16)
    o = rod.swska_prefill(q.to(DEV), k.to(DEV), v.to(DEV), W)
    rod.check()
    compare(o, oracle.swska_prefill(q, k, v, W), "bf16", "large logits")


@pytest.mark.parametrize("B,H,T,W", [(2, 1, 128, 64), (1, 3, 129, 128), (1, 5, 385, 257),
                                     (3, 2, 640, 4096)])
def test_swska_prefill_tile_edges(B, H, T, W):
    _ska_check(B, H, T, 128, 128, W, "bf16", "normal", seed=B * 1000 + H * 100 + W)


def test_swska_prefill_deterministic():
    q, k, v = [t.to(DEV) for t in wl.swska_inputs(1, 4, 2000, 128, 128, seed=22)]
    a = rod.swska_prefill(q, k, v, 512)
    b = rod.swska_prefill(q, k, v, 512)
    rod.check()
    assert torch.equal(a, b)
