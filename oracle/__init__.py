"""fp64 CPU oracle for the Rodimus+ token mixers -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. It shares no code with the CUDA library and never imports it.

The arithmetic lives in ``rodref.c`` (plain double-precision loops); this module only
marshals numpy/torch CPU arrays into it. Inputs are converted to float32, which holds every
bf16 and fp32 input exactly, so the oracle sees exactly the values the GPU sees.

Definitions (see ``rodref.c`` for the citations):
  gla_prefill      S_t = diag(g_t) S_{t-1} + k_t^T v_t,  o_t = q_t S_t
  gla_decode_step  one step of the same recurrence
  swska_prefill    o_t = softmax_j(scale q_t . k_j) v_j over j in [t-W+1, t], K shared by heads
  swska_decode     ring-buffer write at slot pos mod W, then the same softmax over the window
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build


class OracleLib:
    """ctypes view of one build of rodref.c (the default build, or a test's mutated copy)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.rodref_gla_prefill.argtypes = [f32p, f32p, f32p, f32p, f64p, f64p,
                                           i64, i64, i64, i64, i64, ctypes.c_int]
        lib.rodref_gla_decode_step.argtypes = [f32p, f32p, f32p, f32p, f64p, f64p,
                                               i64, i64, i64, i64, ctypes.c_int]
        lib.rodref_swska_prefill.argtypes = [f32p, f32p, f32p, f64p, i64, i64, i64, i64, i64,
                                             i64, ctypes.c_double, i64p, i64, ctypes.c_int]
        lib.rodref_swska_prefill_lse.argtypes = [f32p, f32p, f32p, f64p, f64p, i64, i64, i64, i64, i64,
                                                 i64, ctypes.c_double, i64p, i64, ctypes.c_int]
        lib.rodref_swska_decode.argtypes = [f32p, f32p, f32p, f32p, f32p, i64p, f64p,
                                            i64, i64, i64, i64, i64, ctypes.c_double,
                                            ctypes.c_int]
        lib.rodref_swska_cache_fill.argtypes = [f32p, f32p, f32p, f32p, i64, i64, i64, i64, i64,
                                                i64]
        lib.rodref_swska_decode_paged.argtypes = [f32p, f32p, f32p, f32p, f32p,
                                                  ctypes.POINTER(ctypes.c_int32), i64, i64, i64p,
                                                  f64p, i64, i64, i64, i64, i64, ctypes.c_double,
                                                  ctypes.c_int]
        lib.rodref_swska_backward.argtypes = [f32p, f32p, f32p, f32p, f64p, f64p, f64p, i64, i64,
                                              i64, i64, i64, i64, ctypes.c_double, ctypes.c_int]
        lib.rodref_gla_backward.argtypes = [f32p, f32p, f32p, f32p, f64p, f32p, f32p, f64p, f64p,
                                            f64p, f64p, f64p, i64, i64, i64, i64, i64, ctypes.c_int]
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.rodref_e4m3_encode_array.argtypes = [f32p, u8p, i64, ctypes.c_float]
        lib.rodref_e4m3_decode_array.argtypes = [u8p, f64p, i64]
        lib.rodref_swska_decode_fp8.argtypes = [f32p, f32p, f32p, u8p, u8p, i64p, f64p, i64, i64, i64,
                                                i64, i64, ctypes.c_double, ctypes.c_double,
                                                ctypes.c_double, ctypes.c_int]
        lib.rodref_swska_cache_fill_fp8.argtypes = [f32p, f32p, u8p, u8p, i64, i64, i64, i64, i64, i64,
                                                    ctypes.c_float, ctypes.c_float]
        for name in ("rodref_gla_backward", "rodref_swska_backward", "rodref_gla_prefill", "rodref_gla_decode_step",
                     "rodref_swska_prefill", "rodref_swska_prefill_lse",
                     "rodref_swska_decode", "rodref_swska_cache_fill", "rodref_swska_decode_paged",
                     "rodref_e4m3_encode_array", "rodref_e4m3_decode_array", "rodref_swska_decode_fp8",
                     "rodref_swska_cache_fill_fp8"):
            getattr(lib, name).restype = ctypes.c_int
        self.lib = lib
        self.path = path


_default = None


def _load() -> ctypes.CDLL:
    global _default
    if _default is None:
        _default = OracleLib(_build.build())
    return _default.lib


_active = None  # set by ``using`` to route the module functions through another build


class using:
    """Context manager: route this module's functions through another build of rodref.c."""

    def __init__(self, lib: OracleLib):
        self._lib = lib

    def __enter__(self):
        global _active
        self._prev, _active = _active, self._lib
        return self._lib

    def __exit__(self, *exc):
        global _active
        _active = self._prev
        return False


def _L() -> ctypes.CDLL:
    return _active.lib if _active is not None else _load()


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _f32(x) -> np.ndarray:
    """Any numpy array or CPU/GPU torch tensor -> contiguous float32 numpy (exact for bf16)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p32(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _p64(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _pi64(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _pu8(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def _u8(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").contiguous().view(__import__("torch").uint8).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint8))


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: oracle rejected its arguments (status {rc})")


def gla_prefill(q, k, v, g, state0=None, nthreads=None):
    """Gated linear recurrence over [B,H,T,*] inputs. Returns (o [B,H,T,dv], state [B,H,dk,dv]),
    both float64. ``state0`` defaults to zeros."""
    q, k, v, g = _f32(q), _f32(k), _f32(v), _f32(g)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, T, dk) and g.shape == (B, H, T, dk) and v.shape == (B, H, T, dv)
    S = np.zeros((B, H, dk, dv)) if state0 is None else _f64(state0).copy()
    assert S.shape == (B, H, dk, dv)
    o = np.empty((B, H, T, dv))
    rc = _L().rodref_gla_prefill(_p32(q), _p32(k), _p32(v), _p32(g), _p64(S), _p64(o),
                                 B, H, T, dk, dv, nthreads or default_threads())
    _check(rc, "gla_prefill")
    return o, S


def gla_decode_step(q, k, v, g, state, nthreads=None):
    """One recurrence step for [N,H,*] inputs. Returns (o [N,H,dv], new state), float64."""
    q, k, v, g = _f32(q), _f32(k), _f32(v), _f32(g)
    N, H, dk = q.shape
    dv = v.shape[-1]
    S = _f64(state).copy()
    assert S.shape == (N, H, dk, dv)
    o = np.empty((N, H, dv))
    rc = _L().rodref_gla_decode_step(_p32(q), _p32(k), _p32(v), _p32(g), _p64(S), _p64(o),
                                     N, H, dk, dv, nthreads or default_threads())
    _check(rc, "gla_decode_step")
    return o, S


def swska_prefill(q, k, v, window, scale=None, rows=None, nthreads=None):
    """Sliding-window shared-key attention. q [B,H,T,dk], k [B,T,dk], v [B,H,T,dv].

    ``rows`` (optional) is a 1-D array of flat output-row indices (b*H + h)*T + t; then the
    result is [len(rows), dv], else [B,H,T,dv]. float64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, dk) and v.shape == (B, H, T, dv)
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(dk)
    if rows is None:
        o = np.empty((B, H, T, dv))
        rp, n = None, 0
    else:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        o = np.empty((rows.shape[0], dv))
        rp, n = _pi64(rows), rows.shape[0]
    rc = _L().rodref_swska_prefill(_p32(q), _p32(k), _p32(v), _p64(o), B, H, T, dk, dv,
                                   int(window), float(scale), rp, n,
                                   nthreads or default_threads())
    _check(rc, "swska_prefill")
    return o


def swska_prefill_lse(q, k, v, window, scale=None, rows=None, nthreads=None):
    """swska_prefill and each output row's natural log-sum-exp of its scaled scores
    (rodref_swska_prefill_lse). Returns (o, lse): [B,H,T,dv] and [B,H,T], or [len(rows), dv]
    and [len(rows)] for the given flat rows. float64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, dk) and v.shape == (B, H, T, dv)
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(dk)
    if rows is None:
        o, lse = np.empty((B, H, T, dv)), np.empty((B, H, T))
        rp, n = None, 0
    else:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        o, lse = np.empty((rows.shape[0], dv)), np.empty(rows.shape[0])
        rp, n = _pi64(rows), rows.shape[0]
    rc = _L().rodref_swska_prefill_lse(_p32(q), _p32(k), _p32(v), _p64(o), _p64(lse), B, H, T, dk, dv,
                                       int(window), float(scale), rp, n, nthreads or default_threads())
    _check(rc, "swska_prefill_lse")
    return o, lse


def swska_decode(q, k_new, v_new, k_cache, v_cache, pos, window, scale=None, nthreads=None):
    """Ring-buffer decode. Returns (o [N,H,dv] float64, k_cache', v_cache') with the caches
    (float32 copies) updated at slot pos mod W."""
    q, k_new, v_new = _f32(q), _f32(k_new), _f32(v_new)
    kc, vc = _f32(k_cache).copy(), _f32(v_cache).copy()
    N, H, dk = q.shape
    dv = v_new.shape[-1]
    W = int(window)
    assert kc.shape == (N, W, dk) and vc.shape == (N, H, W, dv)
    if hasattr(pos, "detach"):
        pos = pos.detach().cpu().numpy()
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(dk)
    o = np.empty((N, H, dv))
    rc = _L().rodref_swska_decode(_p32(q), _p32(k_new), _p32(v_new), _p32(kc), _p32(vc),
                                  _pi64(pos), _p64(o), N, H, dk, dv, W, float(scale),
                                  nthreads or default_threads())
    _check(rc, "swska_decode")
    return o, kc, vc


def swska_cache_fill(k, v, k_cache, v_cache, window):
    """Prefill -> decode hand-off (rodref_swska_cache_fill). Returns float32 copies of the
    caches with positions max(0, T-W) .. T-1 of k [B,T,dk] and v [B,H,T,dv] in slots p mod W."""
    k, v = _f32(k), _f32(v)
    kc, vc = _f32(k_cache).copy(), _f32(v_cache).copy()
    B, T, dk = k.shape
    H, dv = v.shape[1], v.shape[-1]
    W = int(window)
    assert v.shape == (B, H, T, dv) and kc.shape == (B, W, dk) and vc.shape == (B, H, W, dv)
    rc = _L().rodref_swska_cache_fill(_p32(k), _p32(v), _p32(kc), _p32(vc), B, H, T, dk, dv, W)
    _check(rc, "swska_cache_fill")
    return kc, vc


def swska_decode_paged(q, k_new, v_new, k_pool, v_pool, block_table, page_size, pos, window,
                       scale=None, nthreads=None):
    """Decode over a paged window cache (rodref_swska_decode_paged). Returns (o [N,H,dv] float64,
    k_pool', v_pool') with float32 copies of the pools, the new tokens written to their pages."""
    q, k_new, v_new = _f32(q), _f32(k_new), _f32(v_new)
    kp, vp = _f32(k_pool).copy(), _f32(v_pool).copy()
    N, H, dk = q.shape
    dv = v_new.shape[-1]
    W, page = int(window), int(page_size)
    if hasattr(block_table, "detach"):
        block_table = block_table.detach().cpu().numpy()
    table = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32)).reshape(-1)
    pps = W // page
    assert table.size == N * pps and kp.shape[1:] == (page, dk) and vp.shape[1:] == (H, page, dv)
    if hasattr(pos, "detach"):
        pos = pos.detach().cpu().numpy()
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(dk)
    o = np.empty((N, H, dv))
    rc = _L().rodref_swska_decode_paged(_p32(q), _p32(k_new), _p32(v_new), _p32(kp), _p32(vp),
                                        table.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), page,
                                        pps, _pi64(pos), _p64(o), N, H, dk, dv, W, float(scale),
                                        nthreads or default_threads())
    _check(rc, "swska_decode_paged")
    return o, kp, vp


def gla_backward(q, k, v, g, dO, state0=None, dS_final=None, nthreads=None):
    """Gradients of the recurrence (rodref_gla_backward) for loss gradients dO [B,H,T,dv] and
    dS_final [B,H,dk,dv] (None: no loss on the final state). Returns float64
    (dq, dk, dv, dg, dstate0)."""
    q, k, v, g, dO = _f32(q), _f32(k), _f32(v), _f32(g), _f32(dO)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    S0 = np.zeros((B, H, dk, dv)) if state0 is None else np.ascontiguousarray(_f64(state0))
    dSf = None if dS_final is None else _f32(dS_final)
    outs = [np.empty((B, H, T, dk)), np.empty((B, H, T, dk)), np.empty((B, H, T, dv)),
            np.empty((B, H, T, dk)), np.empty((B, H, dk, dv))]
    dq, dk_, dv_, dg, dS0 = outs
    rc = _L().rodref_gla_backward(_p32(q), _p32(k), _p32(v), _p32(g), _p64(S0), _p32(dO),
                                  None if dSf is None else _p32(dSf), _p64(dq), _p64(dk_),
                                  _p64(dv_), _p64(dg), _p64(dS0), B, H, T, dk, dv,
                                  nthreads or default_threads())
    _check(rc, "gla_backward")
    return dq, dk_, dv_, dg, dS0


def swska_backward(q, k, v, dO, window, scale=None, nthreads=None):
    """Gradients of SW-SKA prefill (rodref_swska_backward) for the loss gradient dO [B,H,T,dv].
    Returns float64 (dq [B,H,T,dk], dk [B,T,dk] summed over heads, dv [B,H,T,dv])."""
    q, k, v, dO = _f32(q), _f32(k), _f32(v), _f32(dO)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(dk)
    dq, dk_, dv_ = np.empty((B, H, T, dk)), np.empty((B, T, dk)), np.empty((B, H, T, dv))
    rc = _L().rodref_swska_backward(_p32(q), _p32(k), _p32(v), _p32(dO), _p64(dq), _p64(dk_),
                                    _p64(dv_), B, H, T, dk, dv, int(window), float(scale),
                                    nthreads or default_threads())
    _check(rc, "swska_backward")
    return dq, dk_, dv_


# ------------------------------------------------------------------------------------------
# FP8 (E4M3) window cache (SALA blog §4.3; format and rounding as read in rodref.c's header)
# ------------------------------------------------------------------------------------------


def e4m3_encode(x, scale=1.0):
    """E4M3 codes (uint8) of x / scale: the quotient in fp32, the nearest code, ties to the even
    code, magnitudes past 448 saturated."""
    x = _f32(x)
    out = np.empty(x.shape, dtype=np.uint8)
    rc = _L().rodref_e4m3_encode_array(_p32(x), _pu8(out), x.size, float(np.float32(scale)))
    _check(rc, "e4m3_encode")
    return out


def e4m3_decode(codes):
    """Values (float64) of E4M3 codes."""
    c = _u8(codes)
    out = np.empty(c.shape, dtype=np.float64)
    rc = _L().rodref_e4m3_decode_array(_pu8(c), _p64(out), c.size)
    _check(rc, "e4m3_decode")
    return out


def swska_decode_fp8(q, k_new, v_new, k_cache, v_cache, pos, window, scale=None, k_scale=1.0,
                     v_scale=1.0, nthreads=None):
    """Decode over FP8 rings (codes k_cache [N,W,dk], v_cache [N,H,W,dv]). Returns
    (o [N,H,dv] float64, k_cache', v_cache') with the new token's codes written."""
    q, k_new, v_new = _f32(q), _f32(k_new), _f32(v_new)
    kc, vc = _u8(k_cache).copy(), _u8(v_cache).copy()
    pos = np.ascontiguousarray(np.asarray(pos.cpu() if hasattr(pos, "cpu") else pos, dtype=np.int64))
    N, H, dk = q.shape
    dv = v_new.shape[-1]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(dk)
    o = np.empty((N, H, dv))
    rc = _L().rodref_swska_decode_fp8(_p32(q), _p32(k_new), _p32(v_new), _pu8(kc), _pu8(vc), _pi64(pos),
                                      _p64(o), N, H, dk, dv, int(window), float(scale),
                                      float(np.float32(k_scale)), float(np.float32(v_scale)),
                                      nthreads or default_threads())
    _check(rc, "swska_decode_fp8")
    return o, kc, vc


def swska_cache_fill_fp8(k, v, k_cache, v_cache, window, k_scale=1.0, v_scale=1.0):
    """Hand-off into FP8 rings: positions [max(0,T-W), T) of k [B,T,dk], v [B,H,T,dv] to slot
    p mod W as E4M3 codes of x / scale. Returns the updated (k_cache, v_cache) copies (uint8)."""
    k, v = _f32(k), _f32(v)
    kc, vc = _u8(k_cache).copy(), _u8(v_cache).copy()
    B, T, dk = k.shape
    H, dv = v.shape[1], v.shape[-1]
    rc = _L().rodref_swska_cache_fill_fp8(_p32(k), _p32(v), _pu8(kc), _pu8(vc), B, H, T, dk, dv,
                                          int(window), float(np.float32(k_scale)), float(np.float32(v_scale)))
    _check(rc, "swska_cache_fill_fp8")
    return kc, vc
