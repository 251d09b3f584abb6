"""FP8 (E4M3) window cache on the GPU against the oracle (SALA blog §4.3: the KV cache in FP8).

The cache bytes are the method's quantized codes, an encoding: the GPU's codes must equal the
oracle's bit for bit (the hand-off fill, and the decode's write of the new token). The decode
outputs are compared with the oracle's fp64 attention over the dequantized cache within the bf16
tolerance. A decode that continues a quantized prefill hand-off reproduces the oracle's prefill of
the dequantized keys and values.
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


def _caches(N, H, W, d, seed):
    """Seeded E4M3 cache contents (codes), host copies for the oracle."""
    kc = wl.fp8_codes((N, W, d), seed=seed).numpy()
    vc = wl.fp8_codes((N, H, W, d), seed=seed + 1).numpy()
    return kc, vc


@pytest.mark.parametrize("N,H,W,full,ks,vs", [(3, 16, 4096, True, 1.0, 1.0), (2, 16, 4096, False, 0.25, 2.0),
                                              (5, 4, 512, True, 0.5, 0.5), (1, 16, 2048, True, 2.0, 0.125),
                                              (7, 3, 96, False, 1.0, 1.0), (1, 1, 1, True, 1.0, 1.0)])
def test_swska_decode_fp8_matches_oracle(N, H, W, full, ks, vs):
    d = 128
    dd = wl.decode_inputs(N, H, d, d, W, seed=N + W, dtype="bf16", full=full)
    kc, vc = _caches(N, H, W, d, seed=N + W)
    ref, kc_ref, vc_ref = oracle.swska_decode_fp8(dd["sq"], dd["k_new"], dd["v_new"], kc, vc, dd["pos"], W,
                                                  k_scale=ks, v_scale=vs)
    kg, vg = torch.from_numpy(kc).to(DEV), torch.from_numpy(vc).to(DEV)
    o = rod.swska_decode_fp8(dd["sq"].to(DEV), dd["k_new"].to(DEV), dd["v_new"].to(DEV), kg, vg,
                             dd["pos"].to(DEV), W, k_scale=ks, v_scale=vs)
    rod.check()
    compare(o, ref, "bf16", f"fp8 decode N{N} H{H} W{W}")
    np.testing.assert_array_equal(kg.cpu().numpy(), kc_ref)  # the new token's codes, bit for bit
    np.testing.assert_array_equal(vg.cpu().numpy(), vc_ref)


def test_swska_decode_fp8_full_batch():
    """The benchmarked decode shape (N 256, H 16, W 4096, full windows), every output. Inputs are
    drawn on the device (the host copies feed the oracle)."""
    N, H, d, W = 256, 16, 128, 4096
    gen = torch.Generator(device=DEV)
    gen.manual_seed(77)
    sq = torch.randn(N, H, d, generator=gen, device=DEV).to(torch.bfloat16)
    kn = torch.randn(N, d, generator=gen, device=DEV).to(torch.bfloat16)
    vn = torch.randn(N, H, d, generator=gen, device=DEV).to(torch.bfloat16)
    pos = wl.decode_positions(N, W, full=True, device=DEV)
    kg = wl.fp8_codes((N, W, d), seed=78, device=DEV)
    vg = wl.fp8_codes((N, H, W, d), seed=79, device=DEV)
    kc, vc = kg.cpu().numpy(), vg.cpu().numpy()
    ref, kc_ref, vc_ref = oracle.swska_decode_fp8(sq, kn, vn, kc, vc, pos, W)
    o = rod.swska_decode_fp8(sq, kn, vn, kg, vg, pos, W)
    rod.check()
    compare(o, ref, "bf16", "fp8 decode N256")
    np.testing.assert_array_equal(kg.cpu().numpy(), kc_ref)
    np.testing.assert_array_equal(vg.cpu().numpy(), vc_ref)


def test_swska_decode_fp8_negative_position():
    N, H, d, W = 3, 4, 128, 64
    dd = wl.decode_inputs(N, H, d, d, W, seed=5, dtype="bf16", full=True)
    pos = dd["pos"].clone()
    pos[1] = -1
    kc, vc = _caches(N, H, W, d, seed=5)
    kg, vg = torch.from_numpy(kc).to(DEV), torch.from_numpy(vc).to(DEV)
    o = rod.swska_decode_fp8(dd["sq"].to(DEV), dd["k_new"].to(DEV), dd["v_new"].to(DEV), kg, vg, pos.to(DEV), W)
    rod.check()
    assert torch.isnan(o[1]).all() and torch.isfinite(o[0]).all() and torch.isfinite(o[2]).all()
    np.testing.assert_array_equal(kg[1].cpu().numpy(), kc[1])
    np.testing.assert_array_equal(vg[1].cpu().numpy(), vc[1])


@pytest.mark.parametrize("T,W,ks,vs", [(5, 8, 1.0, 1.0), (300, 64, 0.5, 2.0), (1000, 96, 1.0, 1.0), (77, 1, 4.0, 0.25)])
def test_swska_cache_fill_fp8_bit_exact(T, W, ks, vs):
    B, H, d = 2, 3, 128
    _, k, v = wl.swska_inputs(B, H, T, d, d, seed=T + W)
    kc = np.full((B, W, d), 0x55, np.uint8)
    vc = np.full((B, H, W, d), 0x55, np.uint8)
    kc_ref, vc_ref = oracle.swska_cache_fill_fp8(k, v, kc, vc, W, ks, vs)
    kg, vg = torch.from_numpy(kc).to(DEV), torch.from_numpy(vc).to(DEV)
    rod.swska_cache_fill_fp8(k.to(DEV), v.to(DEV), kg, vg, W, ks, vs)
    rod.check()
    np.testing.assert_array_equal(kg.cpu().numpy(), kc_ref)
    np.testing.assert_array_equal(vg.cpu().numpy(), vc_ref)


def test_swska_fp8_generation_continues_the_quantized_prefill():
    """Fill FP8 rings from a T-token prefill, then decode S more tokens: every decode output equals
    the oracle's prefill row of the whole sequence over the dequantized keys and values."""
    N, H, d, W, T, S = 2, 4, 128, 64, 150, 5
    q, k, v = wl.swska_inputs(N, H, T + S, d, d, seed=600)
    ks, vs = 0.5, 2.0
    kq = (oracle.e4m3_decode(oracle.e4m3_encode(k, ks)) * ks).astype(np.float32)
    vq = (oracle.e4m3_decode(oracle.e4m3_encode(v, vs)) * vs).astype(np.float32)
    ref = oracle.swska_prefill(q, kq, vq, W)
    kg = torch.zeros(N, W, d, dtype=torch.uint8, device=DEV)
    vg = torch.zeros(N, H, W, d, dtype=torch.uint8, device=DEV)
    rod.swska_cache_fill_fp8(k[:, :T].contiguous().to(DEV), v[:, :, :T].contiguous().to(DEV), kg, vg, W, ks, vs)
    for s in range(S):
        P = T + s
        o = rod.swska_decode_fp8(q[:, :, P].contiguous().to(DEV), k[:, P].contiguous().to(DEV),
                                 v[:, :, P].contiguous().to(DEV), kg, vg,
                                 torch.full((N,), P, dtype=torch.int64, device=DEV), W, k_scale=ks, v_scale=vs)
        rod.check()
        compare(o, ref[:, :, P], "bf16", f"fp8 generation step {s}")
