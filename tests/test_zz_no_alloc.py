"""rod_gla_prefill_noalloc: the recurrence prefill for callers that cannot allocate.

Callers embedded in a host program that owns the GPU memory pool, plug-ins forbidden to call
cudaMalloc or a framework allocator, and paths that must not allocate after start-up cannot
hand rod_gla_prefill a workspace; rod_gla_prefill_noalloc uses a fixed device array inside the
library instead. These tests call it through the C ABI on sizes that need scratch (several
segments, so the segment pass and state scan run), twice in a row on different inputs, and
compare each result with the workspace-taking entry point within the parity tolerances. They
also check that the fixed array covers every problem: the prefill keeps its segment pass to one
wave of CTAs, so its scratch is bounded by the SM count (one and a half states per SM) whatever
the shape
(the entry point still refuses a larger need with ROD_ERR_WORKSPACE before launching). The file
is collected last and sets up everything it needs itself, so it passes both alone in a fresh
process and after the other tests.
"""
import ctypes

import pytest
import torch

import sliding_window_attention_chunked_b200 as rod
from sliding_window_attention_chunked_b200 import build as rbuild
from sliding_window_attention_chunked_b200 import workloads as wl

from .parity import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_SCRATCH = 48 << 20  # ROD_GLA_PREFILL_NOALLOC_MAX_SCRATCH in include/rod.h


def _noalloc(lib, q, k, v, g, state, o, chunk=64):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.rod_gla_prefill_noalloc(p(q), p(k), p(v), p(g), p(state), p(o), B, H, T, dk, dv,
                                       chunk, 1, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_prefill_matches_workspace_prefill_twice():
    rbuild.build()
    lib = rod.load_library()
    B, H, T, d = 2, 3, 2500, 128
    need = rod.gla_prefill_workspace_size(B, H, T, d, d, 64)
    assert 0 < need <= MAX_SCRATCH  # the case really uses scratch, and it fits
    for seed in (41, 42):           # two calls in a row share (and reuse) the fixed array
        q, k, v, g = [t.to(DEV) for t in wl.gla_inputs(B, H, T, d, d, dist="l2", seed=seed)]
        S0 = torch.randn(B, H, d, d, device=DEV) * 0.1
        S_ref, S_na = S0.clone(), S0.clone()
        o_ref = rod.gla_prefill(q, k, v, g, S_ref, chunk=64)
        o_na = torch.full_like(o_ref, float("nan"))
        assert _noalloc(lib, q, k, v, g, S_na, o_na) == 0
        rod.check()
        compare(o_na, o_ref.float(), "bf16", f"noalloc o (seed {seed})")
        compare(S_na, S_ref, "bf16", f"noalloc state (seed {seed})")


def test_noalloc_scratch_covers_every_plan():
    lib = rod.load_library()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # one fp32 state + decay per workspace slot; the plan keeps the segment pass to one wave
    # (at most `sms` pieces in all) plus one slot per (batch, head), and with more than one
    # segment there are at most sms / 2 (batch, head) pairs
    bound = (sms + sms // 2) * (128 * 128 + 128) * 4
    assert bound <= MAX_SCRATCH
    for B, H, T in [(1, 1, 1 << 20), (1, 16, 131072), (4, 16, 4096), (2, 3, 2500),
                    (1, sms, 8192), (1, sms + 1, 8192), (591, 1, 128)]:
        assert rod.gla_prefill_workspace_size(B, H, T, 128, 128, 64) <= bound
    # more (batch, head) pairs than SMs: one segment each, no scratch, same result
    B, H, T, d = 591, 1, 200, 128
    assert rod.gla_prefill_workspace_size(B, H, T, d, d, 64) == 0
    q, k, v, g = [t.to(DEV) for t in wl.gla_inputs(B, H, T, d, d, dist="l2", seed=7)]
    S_ref = torch.randn(B, H, d, d, device=DEV) * 0.1
    S_na = S_ref.clone()
    o_ref = rod.gla_prefill(q, k, v, g, S_ref, chunk=64)
    o_na = torch.full_like(o_ref, float("nan"))
    assert _noalloc(lib, q, k, v, g, S_na, o_na) == 0
    rod.check()
    compare(o_na, o_ref.float(), "bf16", "noalloc o, 591 pairs")
    compare(S_na, S_ref, "bf16", "noalloc state, 591 pairs")
