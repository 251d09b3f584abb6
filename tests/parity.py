"""Comparison rules for GPU-vs-oracle parity.

bf16 inputs with fp32 accumulation: pass iff max|x - ref| <= 2e-2 AND
    ||x - ref||_F / ||ref||_F <= 5e-3, applied to every output and to the final state.
fp32 inputs: pass iff ||x - ref||_F / ||ref||_F <= 1e-4 AND
    max|x - ref| <= 1e-4 * max(1, max|ref|).
"""
import numpy as np
import torch

BF16_MAX_ABS = 2e-2
BF16_REL_FRO = 5e-3
FP32_REL = 1e-4


def _np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def compare(got, ref, dtype, what=""):
    """Assert parity; returns (max_abs, rel_fro) for reporting."""
    g, r = _np(got), _np(ref)
    assert g.shape == r.shape, f"{what}: shape {g.shape} vs {r.shape}"
    assert np.all(np.isfinite(g)), f"{what}: non-finite values in the GPU output"
    diff = g - r
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    nref = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(diff)) / nref if nref > 0 else float(np.linalg.norm(diff))
    if dtype in ("bf16", torch.bfloat16):
        assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_FRO, \
            f"{what}: max_abs {max_abs:.3e} (<= {BF16_MAX_ABS}), rel_fro {rel:.3e} (<= {BF16_REL_FRO})"
    else:
        lim = FP32_REL * max(1.0, float(np.max(np.abs(r))) if r.size else 1.0)
        assert rel <= FP32_REL and max_abs <= lim, \
            f"{what}: rel_fro {rel:.3e} (<= {FP32_REL}), max_abs {max_abs:.3e} (<= {lim:.3e})"
    return max_abs, rel
