"""Backward of the gated linear recurrence on the GPU against the oracle's reverse-mode sweep.

The oracle's gradients are pinned on the CPU (central differences, PyTorch autograd through a
float64 loop, and the gate identity); here every gradient the library returns (dq, dk, dv in the
input dtype; dg and the initial-state gradient in fp32) is compared with them element by
element: fp32 inputs within the fp32 tolerance, bf16 inputs within the bf16 tolerance for the
bf16 outputs and the fp32 tolerance for the fp32 ones (their arithmetic is fp32 throughout).
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


def _case(B, H, T, dk, dv, dtype, seed, gate=None, final=True, dO_scale=0.2):
    q, k, v, g = wl.gla_inputs(B, H, T, dk, dv, dist="l2", seed=seed, dtype=dtype)
    if gate is not None:
        g = torch.full_like(g, float(gate))
    # loss gradients and initial state scaled so the gradients are O(1): the bf16 bound (2e-2
    # absolute) is stated for outputs of that size (bf16 rounding alone is |x| 2^-9)
    gen = torch.Generator().manual_seed(seed + 1)
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.1
    dO = (torch.randn(B, H, T, dv, generator=gen) * dO_scale).to(q.dtype)
    dSf = torch.randn(B, H, dk, dv, generator=gen) * 0.1 if final else None
    return q, k, v, g, S0, dO, dSf


def _check(B, H, T, dk, dv, dtype, seed, gate=None, final=True, g=None, dO_scale=0.2):
    q, k, v, g0, S0, dO, dSf = _case(B, H, T, dk, dv, dtype, seed, gate, final, dO_scale)
    g = g0 if g is None else g
    ref = oracle.gla_backward(q, k, v, g, dO, S0.double(), dSf)
    got = rod.gla_backward(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), dO.to(DEV), S0.to(DEV),
                           None if dSf is None else dSf.to(DEV))
    rod.check()
    # bf16 with 128-wide heads runs the chunkwise tensor-core backward, whose products take bf16
    # operands (the chunk's states and state gradients included): every gradient there, the fp32
    # dg and dstate0 too, is held to the bf16 tolerance. The CUDA-core route keeps fp32
    # arithmetic throughout, and its fp32 outputs the fp32 tolerance.
    tensor_cores = dtype == "bf16" and dk == 128 and dv == 128
    names = ("dq", "dk", "dv", "dg", "dstate0")
    for name, a, b in zip(names, got, ref):
        tol = dtype if (name in ("dq", "dk", "dv") or tensor_cores) else "fp32"
        compare(a, b, tol, f"{name} B{B} H{H} T{T} dk{dk} dv{dv} {dtype}")


@pytest.mark.parametrize("dk,dv", [(16, 32), (32, 16), (64, 64), (128, 128), (16, 128)])
def test_gla_backward_fp32(dk, dv):
    _check(2, 3, 200, dk, dv, "fp32", seed=dk + dv)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 300])
def test_gla_backward_bf16_lengths_across_checkpoints(T):
    _check(1, 2, T, 128, 128, "bf16", seed=T)


@pytest.mark.parametrize("gate", [0.0, 1.0])
def test_gla_backward_gate_edges(gate):
    """g = 0 (the state resets every step: no gradient flows back through it) and g = 1."""
    _check(1, 2, 130, 64, 32, "fp32", seed=7, gate=gate)


def test_gla_backward_without_final_state_loss():
    _check(2, 2, 150, 32, 64, "fp32", seed=9, final=False)


# ---- the chunkwise tensor-core backward (bf16, d = 128) ----------------------------------------


@pytest.mark.parametrize("gate", [0.0, 1.0])
def test_gla_backward_tensor_core_gate_edges(gate):
    """g = 0 sends every chunk to the exact route (gates below 2^-8: the product form would
    divide by them); g = 1 keeps every chunk on the product route. With g = 1 nothing decays
    and the states sum every token, so dO is scaled down to keep the gradients O(1), the size
    the absolute bound is stated for (bf16 rounding of an output alone is |x| 2^-9)."""
    _check(1, 2, 200, 128, 128, "bf16", seed=17, gate=gate, dO_scale=0.2 if gate == 0.0 else 0.05)


def test_gla_backward_tensor_core_mixed_routes():
    """Chunks with a gate of exactly 0, a strongly decaying channel and a whole chunk below
    2^-8 take the exact route; the rest the product route. Both must agree with the oracle."""
    B, H, T, d = 1, 2, 700, 128
    q, k, v, g, S0, dO, dSf = _case(B, H, T, d, d, "bf16", 19)
    g = g.clone()
    g[:, :, 100:110, 5] = 1e-9
    g[:, 1, 400:464, :] = 0.3 ** 4
    g[:, 0, 650, 77] = 0.0
    g[:, 0, 200, 3] = 2.0 ** -9
    _check(B, H, T, d, d, "bf16", seed=19, g=g)


@pytest.mark.parametrize("B,H,T,final", [(2, 3, 300, False), (3, 1, 129, True), (1, 4, 1000, True)])
def test_gla_backward_tensor_core_shapes(B, H, T, final):
    _check(B, H, T, 128, 128, "bf16", seed=B * 100 + H * 10 + T, final=final)


def test_gla_backward_tensor_core_full_workload():
    """The benchmarked backward workload (B4 H16 T4096, bf16, d = 128): every gradient element
    against the oracle's reverse sweep. dO is drawn at 0.1 N(0,1), which keeps the largest
    gradients near 2.7: at 0.2 N(0,1) they reach 5.5, where bf16 rounding of the exact result
    alone is up to 0.0156 of the 2e-2 absolute bound (measured there: max error 0.022 on dq and
    0.031 on dk, relative Frobenius 2.9e-3 on every gradient; every error is linear in dO)."""
    _check(4, 16, 4096, 128, 128, "bf16", seed=4096, dO_scale=0.1)


def test_gla_backward_empty_sequence_passes_the_final_gradient_through():
    B, H, d = 2, 3, 32
    dSf = torch.randn(B, H, d, d, device=DEV)
    z = torch.zeros(B, H, 0, d, device=DEV)
    _, _, _, _, dS0 = rod.gla_backward(z, z, z, z, z, torch.zeros(B, H, d, d, device=DEV), dSf)
    rod.check()
    assert torch.equal(dS0, dSf)
    _, _, _, _, dS0 = rod.gla_backward(z, z, z, z, z, torch.zeros(B, H, d, d, device=DEV), None)
    rod.check()
    assert torch.equal(dS0, torch.zeros_like(dSf))


# ------------------------------------------------------------------------------------------
# SW-SKA
# ------------------------------------------------------------------------------------------


def _ska_check(B, H, T, dk, dv, W, dtype, seed):
    q, k, v = wl.swska_inputs(B, H, T, dk, dv, seed=seed, dtype=dtype)
    dO = (torch.randn(B, H, T, dv, generator=torch.Generator().manual_seed(seed + 5)) * 0.5).to(q.dtype)
    ref = oracle.swska_backward(q, k, v, dO, W)
    got = rod.swska_backward(q.to(DEV), k.to(DEV), v.to(DEV), dO.to(DEV), W)
    rod.check()
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        compare(a, b, dtype, f"{name} B{B} H{H} T{T} dk{dk} dv{dv} W{W} {dtype}")


@pytest.mark.parametrize("dk,dv,W", [(16, 32, 7), (32, 16, 64), (64, 64, 1), (128, 128, 40)])
def test_swska_backward_fp32(dk, dv, W):
    _ska_check(2, 3, 150, dk, dv, W, "fp32", seed=dk + dv + W)


@pytest.mark.parametrize("T,W", [(1, 64), (200, 64), (300, 300), (257, 128)])
def test_swska_backward_bf16(T, W):
    _ska_check(1, 4, T, 128, 128, W, "bf16", seed=T + W)


# bf16 with head dim 128 and T >= 128 runs on the tensor cores: one 128-query tile, ragged
# tails, windows of 1, below, at and above the tile size, a window longer than the sequence,
# several batches, and head counts that give one or several heads per key-tile group
@pytest.mark.parametrize("B,H,T,W", [(1, 2, 128, 128), (2, 3, 384, 1), (1, 5, 640, 200),
                                     (2, 2, 129, 1000), (1, 16, 1024, 256), (1, 3, 1000, 129),
                                     (3, 1, 700, 64), (1, 4, 2048, 700)])
def test_swska_backward_bf16_tensor_core(B, H, T, W):
    _ska_check(B, H, T, 128, 128, W, "bf16", seed=B * 1000 + H * 100 + T + W)


@pytest.mark.parametrize("d", [32, 64])
def test_swska_backward_bf16_small_head_dim(d):
    """Head dims other than 128 keep the CUDA-core kernels in bf16."""
    _ska_check(2, 3, 300, d, d, 100, "bf16", seed=d)


def test_swska_backward_full_size():
    """The benchmarked backward workload (B1 H16 T8192 W4096, bf16, head dim 128), every
    gradient element against the oracle (about ten seconds of fp64 on the host)."""
    _ska_check(1, 16, 8192, 128, 128, 4096, "bf16", seed=42)


# SW-SKA with the forward's saved statistics
# ------------------------------------------------------------------------------------------


def _ska_lse_check(B, H, T, dk, dv, W, dtype, seed):
    """swska_prefill_lse (output and natural log-sum-exp per row) and swska_backward_lse (the
    gradients from that output and log-sum-exp) against the oracle. The output must equal
    swska_prefill's bit for bit (the same arithmetic); the log-sum-exp is a sum of fp32
    exponentials of fp32 scores on both routes, held to 1e-4 relative (its terms carry the SFU's
    2^-22 and the scores' fp32 rounding); the gradients to the backward's tolerances."""
    q, k, v = wl.swska_inputs(B, H, T, dk, dv, seed=seed, dtype=dtype)
    dO = (torch.randn(B, H, T, dv, generator=torch.Generator().manual_seed(seed + 5)) * 0.5).to(q.dtype)
    o_ref, lse_ref = oracle.swska_prefill_lse(q, k, v, W)
    qd, kd, vd, dOd = q.to(DEV), k.to(DEV), v.to(DEV), dO.to(DEV)
    o, lse = rod.swska_prefill_lse(qd, kd, vd, W)
    o_plain = rod.swska_prefill(qd, kd, vd, W)
    rod.check()
    what = f"B{B} H{H} T{T} dk{dk} dv{dv} W{W} {dtype}"
    assert torch.equal(o, o_plain), f"o of swska_prefill_lse differs from swska_prefill ({what})"
    compare(o, o_ref, dtype, f"o {what}")
    lse_err = np.abs(lse.double().cpu().numpy() - lse_ref)
    lim = 1e-4 * np.maximum(1.0, np.abs(lse_ref))
    assert np.all(lse_err <= lim), f"lse {what}: max error {lse_err.max():.3e}"
    ref = oracle.swska_backward(q, k, v, dO, W)
    got = rod.swska_backward_lse(qd, kd, vd, o, lse, dOd, W)
    rod.check()
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        compare(a, b, dtype, f"{name} from saved statistics, {what}")


# tensor-core route (bf16, head dim 128, T >= 128): one tile, ragged tails, windows of 1 and
# beyond the sequence, several heads and batches
@pytest.mark.parametrize("B,H,T,W", [(1, 2, 128, 128), (2, 3, 300, 1), (1, 4, 1000, 4096),
                                     (1, 16, 1024, 256), (3, 1, 700, 64)])
def test_swska_saved_statistics_tensor_core(B, H, T, W):
    _ska_lse_check(B, H, T, 128, 128, W, "bf16", seed=7 * B + 11 * H + T + W)


# CUDA-core route (fp32, other head dims, or T < 128): the prefill writes the log-sum-exp, the
# backward recomputes its statistics
@pytest.mark.parametrize("B,H,T,d,W,dtype", [(2, 3, 150, 32, 7, "fp32"), (2, 3, 300, 64, 100, "bf16"),
                                             (1, 2, 100, 128, 40, "bf16")])
def test_swska_saved_statistics_cuda_cores(B, H, T, d, W, dtype):
    _ska_lse_check(B, H, T, d, d, W, dtype, seed=T + d + W)


def test_swska_saved_statistics_full_size():
    """The benchmarked backward workload (B1 H16 T8192 W4096, bf16) through the saved-statistics
    path, every element against the oracle."""
    _ska_lse_check(1, 16, 8192, 128, 128, 4096, "bf16", seed=43)
