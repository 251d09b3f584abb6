"""C-ABI checks that need no GPU: librod.so loads, exports every entry point include/rod.h
declares, and rejects bad arguments on the host with the documented status codes before
anything is launched (no call below reaches a kernel)."""
import ctypes
import os
import re
import subprocess

import pytest

import sliding_window_attention_chunked_b200 as rod
from sliding_window_attention_chunked_b200 import build as rbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rod.h")

OK, NULL, SHAPE, ALIGN, DTYPE, WS, CUDA, TIMEOUT = 0, -1, -2, -3, -4, -5, -6, -7


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return rod.load_library()


def declared_symbols():
    src = open(HEADER).read()
    return re.findall(r"ROD_API\s+[\w\s\*]+?\b(rod_\w+)\s*\(", src)


def test_header_declares_the_four_entry_points():
    names = set(declared_symbols())
    for n in ("rod_gla_prefill", "rod_gla_decode_step", "rod_swska_prefill", "rod_swska_decode",
              "rod_gla_prefill_workspace_size", "rod_check", "rod_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert names
    out = subprocess.run(["nm", "-D", "--defined-only", rod.library_path()], check=True,
                         capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, f"{n} declared in rod.h but not exported"
        assert getattr(lib, n) is not None
    # the library exports exactly the declared ABI (no C++ or CUDA-runtime internals)
    assert exported == set(names), sorted(exported ^ set(names))


def test_status_strings_and_version(lib):
    for st in (OK, NULL, SHAPE, ALIGN, DTYPE, WS, CUDA, TIMEOUT):
        assert lib.rod_status_string(st)
    assert lib.rod_status_string(12345) == b"unknown status"
    assert lib.rod_abi_version() == 1


def test_wait_expiry_arming_is_host_only(lib):
    # arming and disarming the wait-expiry diagnostic touches no device state
    assert lib.rod_test_expire_waits(4096) == OK
    assert lib.rod_test_expire_waits(0) == OK


P = ctypes.c_void_p(0x10000)   # aligned, never dereferenced (every call below fails first)
MIS = ctypes.c_void_p(0x10008)  # 8-byte aligned only


def gla(lib, **kw):
    a = dict(q=P, k=P, v=P, g=P, s=P, o=P, B=1, H=2, T=8, dk=16, dv=32, chunk=32, dtype=2,
             ws=None, wsb=0)
    a.update(kw)
    return lib.rod_gla_prefill(a["q"], a["k"], a["v"], a["g"], a["s"], a["o"], a["B"], a["H"],
                               a["T"], a["dk"], a["dv"], a["chunk"], a["dtype"], a["ws"],
                               a["wsb"], None)


def test_gla_prefill_validation(lib):
    assert gla(lib, dtype=3) == DTYPE
    assert gla(lib, dk=24) == SHAPE
    assert gla(lib, dv=256) == SHAPE
    assert gla(lib, chunk=24) == SHAPE
    assert gla(lib, chunk=144) == SHAPE
    assert gla(lib, T=-1) == SHAPE
    assert gla(lib, q=None) == NULL
    assert gla(lib, g=None) == NULL
    assert gla(lib, o=MIS) == ALIGN
    assert gla(lib, T=0, q=None) == OK          # empty: a no-op that touches nothing
    assert gla(lib, B=0, q=None) == OK


def test_gla_prefill_workspace_size_is_deterministic(lib):
    a = lib.rod_gla_prefill_workspace_size(4, 16, 4096, 128, 128, 64, 1)
    b = lib.rod_gla_prefill_workspace_size(4, 16, 4096, 128, 128, 64, 1)
    assert a == b
    assert lib.rod_gla_prefill_workspace_size(4, 16, 4096, 100, 128, 64, 1) == 0


def test_gla_decode_validation(lib):
    f = lib.rod_gla_decode_step
    assert f(P, P, P, P, P, P, 4, 2, 16, 32, 7, None) == DTYPE
    assert f(P, P, P, P, P, P, 4, 2, 48, 32, 2, None) == SHAPE
    assert f(None, P, P, P, P, P, 4, 2, 16, 32, 2, None) == NULL
    assert f(P, P, P, P, MIS, P, 4, 2, 16, 32, 2, None) == ALIGN
    assert f(None, None, None, None, None, None, 0, 2, 16, 32, 2, None) == OK


def test_swska_prefill_validation(lib):
    f = lib.rod_swska_prefill
    assert f(P, P, P, P, 1, 2, 8, 16, 32, 0, 0.0, 2, None) == SHAPE      # window < 1
    assert f(P, P, P, P, 1, 65, 8, 16, 32, 4, 0.0, 2, None) == SHAPE     # too many heads
    assert f(P, P, P, P, 1, 2, 8, 16, 32, 4, float("nan"), 2, None) == SHAPE
    assert f(P, P, P, P, 1, 2, 8, 16, 32, 4, 0.0, 0, None) == DTYPE
    assert f(P, None, P, P, 1, 2, 8, 16, 32, 4, 0.0, 2, None) == NULL
    assert f(P, P, MIS, P, 1, 2, 8, 16, 32, 4, 0.0, 2, None) == ALIGN
    assert f(None, None, None, None, 1, 2, 0, 16, 32, 4, 0.0, 2, None) == OK


def test_swska_decode_validation(lib):
    f = lib.rod_swska_decode
    assert f(P, P, P, P, P, P, P, 4, 2, 16, 32, 0, 0.0, 2, None) == SHAPE
    assert f(P, P, P, P, P, P, P, 4, 0, 16, 32, 8, 0.0, 2, None) == SHAPE
    assert f(P, P, P, P, P, None, P, 4, 2, 16, 32, 8, 0.0, 2, None) == NULL
    assert f(P, P, P, P, MIS, P, P, 4, 2, 16, 32, 8, 0.0, 2, None) == ALIGN
    assert f(P, P, P, P, P, P, P, 4, 2, 16, 32, 8, 0.0, 9, None) == DTYPE
    assert f(None, None, None, None, None, None, None, 0, 2, 16, 32, 8, 0.0, 2, None) == OK


def test_swska_decode_paged_validation(lib):
    f = lib.rod_swska_decode_paged
    # (q, k_new, v_new, k_pool, v_pool, table, page, pps, pos, o, N, H, dk, dv, W, scale, dtype, s)
    ok = (P, P, P, P, P, P, 64, 4, P, P, 2, 16, 128, 128, 256, 0.0, 1, None)
    args = lambda **kw: tuple(kw.get(k, v) for k, v in zip(
        ("q", "kn", "vn", "kp", "vp", "t", "page", "pps", "pos", "o", "N", "H", "dk", "dv", "W",
         "scale", "dt", "s"), ok))
    assert f(*args(W=255)) == SHAPE                   # window != pages x page size
    assert f(*args(page=12, W=48)) == SHAPE            # page size not a multiple of 8
    assert f(*args(pps=513, W=64 * 513)) == SHAPE      # more pages than a CTA's table slice holds
    assert f(*args(H=17)) == SHAPE
    assert f(*args(dk=64, dv=64)) == SHAPE             # only 128-wide heads
    assert f(*args(dt=2)) == DTYPE                     # bf16 only
    assert f(*args(t=None)) == NULL
    assert f(*args(kp=MIS)) == ALIGN
    assert f(*args(N=0, q=None, kn=None, vn=None, kp=None, vp=None, t=None, pos=None, o=None)) == OK


def test_swska_cache_fill_validation(lib):
    f = lib.rod_swska_cache_fill
    assert f(P, P, P, P, 1, 2, 8, 16, 32, 0, 2, None) == SHAPE    # window < 1
    assert f(P, P, P, P, 1, 0, 8, 16, 32, 4, 2, None) == SHAPE    # no heads
    assert f(P, P, P, P, 1, 2, 8, 16, 32, 4, 0, None) == DTYPE
    assert f(P, None, P, P, 1, 2, 8, 16, 32, 4, 2, None) == NULL
    assert f(P, P, MIS, P, 1, 2, 8, 16, 32, 4, 2, None) == ALIGN
    assert f(None, None, None, None, 1, 2, 0, 16, 32, 4, 2, None) == OK   # T = 0


def test_swska_fp8_validation(lib):
    """FP8 cache entry points: argument checks before any launch (no GPU needed)."""
    d = lib.rod_swska_decode_fp8
    args = lambda N=2, H=4, dk=128, dv=128, W=64, s=0.0, ks=1.0, vs=1.0, q=P, kc=P: (
        q, P, P, kc, P, P, P, N, H, dk, dv, W, s, ks, vs, None)
    assert d(*args(W=0)) == SHAPE
    assert d(*args(dk=64, dv=64)) == SHAPE             # only 128-wide heads
    assert d(*args(H=17)) == SHAPE
    assert d(*args(ks=0.0)) == SHAPE                   # scales positive and finite
    assert d(*args(vs=-1.0)) == SHAPE
    assert d(*args(ks=float("inf"))) == SHAPE
    assert d(*args(vs=float("nan"))) == SHAPE
    assert d(*args(q=None)) == NULL
    assert d(*args(kc=MIS)) == ALIGN
    assert d(*args(N=0, q=None, kc=None)) == OK
    f = lib.rod_swska_cache_fill_fp8
    assert f(P, P, P, P, 1, 2, 8, 128, 128, 0, 1.0, 1.0, None) == SHAPE   # window < 1
    assert f(P, P, P, P, 1, 2, 8, 64, 64, 4, 1.0, 1.0, None) == SHAPE     # only 128-wide heads
    assert f(P, P, P, P, 1, 2, 8, 128, 128, 4, 0.0, 1.0, None) == SHAPE
    assert f(P, None, P, P, 1, 2, 8, 128, 128, 4, 1.0, 1.0, None) == NULL
    assert f(P, P, MIS, P, 1, 2, 8, 128, 128, 4, 1.0, 1.0, None) == ALIGN
    assert f(None, None, None, None, 1, 2, 0, 128, 128, 4, 1.0, 1.0, None) == OK   # T = 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 2, 8, 16)
    with pytest.raises(ValueError, match="CUDA"):
        rod.swska_prefill(q, torch.zeros(1, 8, 16), torch.zeros(1, 2, 8, 32), 4)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from sliding_window_attention_chunked_b200 import _binding
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "_PKG", str(tmp_path))
    with pytest.raises(RuntimeError, match="not built"):
        _binding.load_library()
