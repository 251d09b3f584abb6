"""Seeded synthetic inputs for the Rodimus+ mixers -- shared by the CUDA path and the oracle.

This module holds only input recipes (shapes, distributions, seeds, rounding). It contains
none of the mixers' arithmetic, and it imports neither the CUDA binding nor the oracle.

Recipes (the pages publish no dataset for this path; these stand in for the model-level
shapes of the Rodimus+ 1.6B config -- hidden 2048 = 16 heads x 128, window 4096, 24
alternating layers, up to 131072 positions -- given in the setup blog's §3 config):

  "tiny"   q, k ~ N(0,1)/sqrt(dk); v ~ N(0,1)/sqrt(dv); g = sigmoid(N(3,1))
  "l2"     q, k ~ N(0,1)/sqrt(dk), then each (b,h,t) vector L2-normalised over dk;
           v ~ N(0,1); g = sigmoid(N(4, 1.5))
  "normal" q, k, v ~ N(0,1)
Everything is drawn in fp32 from one seeded ``torch.Generator`` in a fixed order
(q, k, v, g for the recurrence; q, shared k, v for attention) and then rounded once to the
compute dtype (bf16 round-to-nearest-even); gates and states stay fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

# ------------------------------------------------------------------------------------------
# named workloads
# ------------------------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "tiny" | "gla_prefill" | "swska_prefill" | "decode" | "stack"
    dtype: str           # "fp32" | "bf16"
    dims: dict = field(default_factory=dict)


WORKLOADS = {
    # tiny fp32 correctness case: both mixers
    "tiny_fp32": Workload("tiny_fp32", "tiny", "fp32",
                          dict(B=1, T=256, H=2, dk=16, dv=32, chunk=32, window=64)),
    # Rodimus block prefill: bf16 in, fp32 state
    "gla_prefill_b4_t4096": Workload("gla_prefill_b4_t4096", "gla_prefill", "bf16",
                                     dict(B=4, T=4096, H=16, dk=128, dv=128, chunk=64)),
    # SW-SKA prefill
    "swska_prefill_b2_t32768": Workload("swska_prefill_b2_t32768", "swska_prefill", "bf16",
                                        dict(B=2, T=32768, H=16, dk=128, dv=128, window=4096)),
    # batched decode: 256 sequences x 1 token, both mixers
    "decode_n256": Workload("decode_n256", "decode", "bf16",
                            dict(N=256, H=16, dk=128, dv=128, window=4096)),
    # long-context mixer stack: 24 alternating layers
    "stack_t131072": Workload("stack_t131072", "stack", "bf16",
                              dict(B=1, T=131072, H=16, dk=128, dv=128, layers=24, chunk=64,
                                   window=4096)),
}

TORCH_DTYPE = {"fp32": torch.float32, "bf16": torch.bfloat16}


def _gen(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev.type if dev.type != "cuda" else dev)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen, device):
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


# ------------------------------------------------------------------------------------------
# gated linear recurrence inputs
# ------------------------------------------------------------------------------------------


def gla_inputs(B, H, T, dk, dv, *, dist="l2", seed=0, dtype="bf16", device="cpu"):
    """q, k [B,H,T,dk] and v [B,H,T,dv] in ``dtype``; g [B,H,T,dk] fp32 in (0,1)."""
    gen = _gen(seed, device)
    dt = TORCH_DTYPE[dtype]
    q = _randn((B, H, T, dk), gen, device)
    k = _randn((B, H, T, dk), gen, device)
    v = _randn((B, H, T, dv), gen, device)
    z = _randn((B, H, T, dk), gen, device)
    if dist == "tiny":
        q, k, v = q / math.sqrt(dk), k / math.sqrt(dk), v / math.sqrt(dv)
        g = torch.sigmoid(z + 3.0)
    elif dist == "l2":
        q, k = _l2norm(q / math.sqrt(dk)), _l2norm(k / math.sqrt(dk))
        g = torch.sigmoid(z * 1.5 + 4.0)
    elif dist == "normal":
        g = torch.sigmoid(z * 1.5 + 4.0)
    else:
        raise ValueError(dist)
    return q.to(dt), k.to(dt), v.to(dt), g.contiguous()


# ------------------------------------------------------------------------------------------
# sliding-window shared-key attention inputs
# ------------------------------------------------------------------------------------------


def swska_inputs(B, H, T, dk, dv, *, dist="normal", seed=0, dtype="bf16", device="cpu"):
    """q [B,H,T,dk], shared k [B,T,dk], v [B,H,T,dv], all in ``dtype``."""
    gen = _gen(seed, device)
    dt = TORCH_DTYPE[dtype]
    q = _randn((B, H, T, dk), gen, device)
    k = _randn((B, T, dk), gen, device)
    v = _randn((B, H, T, dv), gen, device)
    if dist == "tiny":
        q, k, v = q / math.sqrt(dk), k / math.sqrt(dk), v / math.sqrt(dv)
    elif dist == "l2":
        q, k = _l2norm(q), _l2norm(k)
    elif dist != "normal":
        raise ValueError(dist)
    return q.to(dt), k.to(dt), v.to(dt)


# ------------------------------------------------------------------------------------------
# batched decode inputs
# ------------------------------------------------------------------------------------------


def decode_positions(N, W, *, full=True, device="cpu"):
    """Position of each sequence's new token. ``full``: every window is full and the ring head
    differs per sequence (pos_n = W + (n*997 mod W)); else pos_n = n*997 mod (2W) (a mix of
    partially filled and full windows)."""
    n = torch.arange(N, dtype=torch.int64)
    pos = W + (n * 997) % W if full else (n * 997) % (2 * W)
    return pos.to(device)


def decode_inputs(N, H, dk, dv, W, *, seed=0, dtype="bf16", device="cpu", full=True):
    """Returns a dict with the recurrence part (q, k, v, g, state) and the attention part
    (sq, k_new, v_new, k_cache, v_cache, pos)."""
    gen = _gen(seed, device)
    dt = TORCH_DTYPE[dtype]
    q = _l2norm(_randn((N, H, dk), gen, device))
    k = _l2norm(_randn((N, H, dk), gen, device))
    v = _randn((N, H, dv), gen, device)
    g = torch.sigmoid(_randn((N, H, dk), gen, device) * 1.5 + 4.0)
    state = _randn((N, H, dk, dv), gen, device)
    sq = _randn((N, H, dk), gen, device)
    k_new = _randn((N, dk), gen, device)
    v_new = _randn((N, H, dv), gen, device)
    k_cache = _randn((N, W, dk), gen, device)
    v_cache = _randn((N, H, W, dv), gen, device)
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), g=g, state=state,
                sq=sq.to(dt), k_new=k_new.to(dt), v_new=v_new.to(dt),
                k_cache=k_cache.to(dt), v_cache=v_cache.to(dt),
                pos=decode_positions(N, W, full=full, device=device))


def fp8_codes(shape, *, seed=0, device="cpu"):
    """Random E4M3 cache contents as codes (uint8): sign uniform, exponent field uniform in
    4 .. 9 (magnitudes 2^-3 .. 7.5), mantissa field uniform. Bit assembly only."""
    gen = _gen(seed, device)
    sign = torch.randint(0, 2, shape, generator=gen, device=device, dtype=torch.uint8)
    expo = torch.randint(4, 10, shape, generator=gen, device=device, dtype=torch.uint8)
    mant = torch.randint(0, 8, shape, generator=gen, device=device, dtype=torch.uint8)
    return (sign << 7) | (expo << 3) | mant


# ------------------------------------------------------------------------------------------
# long-context stack: layer l even = recurrence, odd = SW-SKA; per-layer seed = l
# ------------------------------------------------------------------------------------------


def stack_layer_kind(layer: int) -> str:
    return "gla" if layer % 2 == 0 else "swska"


def stack_layer_inputs(layer, B, H, T, dk, dv, *, seed_base=0, dtype="bf16", device="cpu"):
    seed = seed_base + layer
    if stack_layer_kind(layer) == "gla":
        return gla_inputs(B, H, T, dk, dv, dist="l2", seed=seed, dtype=dtype, device=device)
    return swska_inputs(B, H, T, dk, dv, dist="l2", seed=seed, dtype=dtype, device=device)
