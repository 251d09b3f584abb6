"""ctypes marshalling for librod.so. Argument checks and pointer passing only -- no arithmetic.

Each function mirrors one entry point of include/rod.h and takes torch CUDA tensors in the
layouts documented there. Outputs are allocated with torch when not supplied (plumbing);
the computation itself is entirely inside the library's kernels.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))

ROD_BF16 = 1
ROD_FP32 = 2
_DT = {torch.bfloat16: ROD_BF16, torch.float32: ROD_FP32}

_lib = None


class RodError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str, cuda_error: int = 0):
        extra = f", cudaError {cuda_error}" if cuda_error else ""
        super().__init__(f"{fn}: status {status} ({msg}{extra})")
        self.status = status


def library_path() -> str:
    return os.path.join(_PKG, "librod.so")


def load_library() -> ctypes.CDLL:
    """Load librod.so (built in-tree by ``python -m sliding_window_attention_chunked_b200.build``).
    Raises if it is missing: there is deliberately no fallback path."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"librod.so is not built ({path}); run "
                           "`python -m sliding_window_attention_chunked_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    lib.rod_status_string.argtypes = [i]
    lib.rod_status_string.restype = ctypes.c_char_p
    lib.rod_last_cuda_error.argtypes = []
    lib.rod_last_cuda_error.restype = i
    lib.rod_check.argtypes = [vp]
    lib.rod_check.restype = i
    lib.rod_abi_version.argtypes = []
    lib.rod_abi_version.restype = i
    lib.rod_launch_count.argtypes = []
    lib.rod_launch_count.restype = ctypes.c_uint64
    lib.rod_test_expire_waits.argtypes = [ctypes.c_uint32]
    lib.rod_test_expire_waits.restype = i
    lib.rod_gla_prefill_workspace_size.argtypes = [i, i, i, i, i, i, i]
    lib.rod_gla_prefill_workspace_size.restype = sz
    lib.rod_gla_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.rod_gla_prefill.restype = i
    lib.rod_gla_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.rod_gla_prefill_noalloc.restype = i
    lib.rod_gla_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.rod_gla_decode_step.restype = i
    lib.rod_swska_prefill.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
    lib.rod_swska_prefill.restype = i
    lib.rod_swska_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    lib.rod_swska_decode.restype = i
    lib.rod_swska_cache_fill.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.rod_swska_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, i, i, vp, vp, i, i, i, i, i, f,
                                           i, vp]
    lib.rod_swska_decode_paged.restype = i
    lib.rod_gla_backward_workspace_size.argtypes = [i, i, i, i, i]
    lib.rod_gla_backward_workspace_size.restype = sz
    lib.rod_gla_backward.argtypes = [vp] * 12 + [i] * 6 + [vp, sz, vp]
    lib.rod_gla_backward.restype = i
    lib.rod_swska_backward_workspace_size.argtypes = [i, i, i]
    lib.rod_swska_backward_workspace_size.restype = sz
    lib.rod_swska_backward.argtypes = [vp] * 7 + [i] * 6 + [f, i, vp, sz, vp]
    lib.rod_swska_backward.restype = i
    lib.rod_swska_prefill_lse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
    lib.rod_swska_prefill_lse.restype = i
    lib.rod_swska_backward_lse.argtypes = [vp] * 9 + [i] * 6 + [f, i, vp, sz, vp]
    lib.rod_swska_backward_lse.restype = i
    lib.rod_swska_cache_fill.restype = i
    lib.rod_swska_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, vp]
    lib.rod_swska_decode_fp8.restype = i
    lib.rod_swska_cache_fill_fp8.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, f, vp]
    lib.rod_swska_cache_fill_fp8.restype = i
    _lib = lib
    return lib


def _raise_on(fn: str, status: int):
    if status != 0:
        lib = load_library()
        raise RodError(fn, status, lib.rod_status_string(status).decode(),
                       lib.rod_last_cuda_error() if status == -6 else 0)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library computes only on the GPU)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise ValueError(f"unsupported dtype {t.dtype} (bf16 or fp32)")
    return _DT[t.dtype]


def abi_version() -> int:
    return load_library().rod_abi_version()


def launch_count() -> int:
    """Kernels launched by librod.so in this process so far."""
    return int(load_library().rod_launch_count())


def test_expire_waits(probes: int) -> None:
    """Diagnostics (rod_test_expire_waits): arm the next tensor-core recurrence prefill call so
    that its producers issue no copies and its bounded waits give up after `probes` probes;
    check() then raises RodError with status ROD_ERR_TIMEOUT (-7). 0 disarms."""
    _raise_on("rod_test_expire_waits", load_library().rod_test_expire_waits(int(probes)))


def check(stream=None) -> None:
    """Synchronise the stream and raise if a kernel reported a CUDA error or a wait timeout."""
    _raise_on("rod_check", load_library().rod_check(_stream(stream)))


def gla_prefill_workspace_size(B, H, T, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    return load_library().rod_gla_prefill_workspace_size(B, H, T, dk, dv, chunk, _DT[dtype])


def gla_prefill(q, k, v, g, state, o=None, chunk=64, workspace=None, stream=None):
    """Chunkwise prefill. q,k [B,H,T,dk], v [B,H,T,dv] (bf16|fp32), g [B,H,T,dk] fp32,
    state [B,H,dk,dv] fp32 (initial on entry, final on return, updated in place).
    Returns o [B,H,T,dv]."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype, 4)
    _need(g, "g", torch.float32, 4)
    _need(state, "state", torch.float32, 4)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or tuple(v.shape[:3]) != (B, H, T):
        raise ValueError("q, k, g must be [B,H,T,dk] and v [B,H,T,dv]")
    if tuple(state.shape) != (B, H, dk, dv):
        raise ValueError("state must be [B,H,dk,dv]")
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, 4)
    lib = load_library()
    ws_need = lib.rod_gla_prefill_workspace_size(B, H, T, dk, dv, chunk, _dtype_code(q))
    if ws_need and workspace is None:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.rod_gla_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(state), _ptr(o),
                             B, H, T, dk, dv, chunk, _dtype_code(q), _ptr(workspace), ws_bytes,
                             _stream(stream))
    _raise_on("rod_gla_prefill", st)
    return o


def gla_prefill_noalloc(q, k, v, g, state, o=None, chunk=64, stream=None):
    """rod_gla_prefill_noalloc: the same prefill as gla_prefill, but the library uses its own
    fixed device scratch instead of a caller-provided workspace (for callers that cannot
    allocate per call). ``o`` must be supplied by such callers; when omitted it is allocated
    here for convenience. Returns o."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype, 4)
    _need(g, "g", torch.float32, 4)
    _need(state, "state", torch.float32, 4)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or tuple(v.shape[:3]) != (B, H, T):
        raise ValueError("q, k, g must be [B,H,T,dk] and v [B,H,T,dv]")
    if tuple(state.shape) != (B, H, dk, dv):
        raise ValueError("state must be [B,H,dk,dv]")
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, 4)
    st = load_library().rod_gla_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(state),
                                                _ptr(o), B, H, T, dk, dv, chunk, _dtype_code(q),
                                                _stream(stream))
    _raise_on("rod_gla_prefill_noalloc", st)
    return o


def gla_decode_step(q, k, v, g, state, o=None, stream=None):
    """One decode step. q,k [N,H,dk], v [N,H,dv], g [N,H,dk] fp32, state [N,H,dk,dv] fp32
    (updated in place). Returns o [N,H,dv]."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype, 3)
    _need(g, "g", torch.float32, 3)
    _need(state, "state", torch.float32, 4)
    N, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or tuple(state.shape) != (N, H, dk, dv):
        raise ValueError("shape mismatch")
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, 3)
    st = load_library().rod_gla_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(state),
                                            _ptr(o), N, H, dk, dv, _dtype_code(q), _stream(stream))
    _raise_on("rod_gla_decode_step", st)
    return o


def swska_prefill(q, k, v, window, scale=None, o=None, stream=None):
    """Sliding-window shared-key attention. q [B,H,T,dk], k [B,T,dk] (shared by the heads),
    v [B,H,T,dv]. Returns o [B,H,T,dv]."""
    _need(q, "q", None, 4)
    _need(k, "k", q.dtype, 3)
    _need(v, "v", q.dtype, 4)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (B, T, dk) or tuple(v.shape[:3]) != (B, H, T):
        raise ValueError("k must be [B,T,dk] and v [B,H,T,dv]")
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, 4)
    st = load_library().rod_swska_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, T, dk, dv,
                                          int(window), float(scale or 0.0), _dtype_code(q),
                                          _stream(stream))
    _raise_on("rod_swska_prefill", st)
    return o


def swska_prefill_lse(q, k, v, window, scale=None, o=None, lse=None, stream=None):
    """swska_prefill that also returns each row's natural log-sum-exp of the scaled scores.
    Returns (o [B,H,T,dv], lse [B,H,T] fp32), the pair swska_backward_lse takes."""
    _need(q, "q", None, 4)
    _need(k, "k", q.dtype, 3)
    _need(v, "v", q.dtype, 4)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (B, T, dk) or tuple(v.shape[:3]) != (B, H, T):
        raise ValueError("k must be [B,T,dk] and v [B,H,T,dv]")
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _need(o, "o", q.dtype, 4)
    _need(lse, "lse", torch.float32, 3)
    if tuple(o.shape) != (B, H, T, dv) or tuple(lse.shape) != (B, H, T):
        raise ValueError("o must be [B,H,T,dv] and lse [B,H,T]")
    st = load_library().rod_swska_prefill_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, T, dk, dv,
                                              int(window), float(scale or 0.0), _dtype_code(q), _stream(stream))
    _raise_on("rod_swska_prefill_lse", st)
    return o, lse


def swska_decode(q, k_new, v_new, k_cache, v_cache, pos, window, scale=None, o=None,
                 stream=None):
    """Ring-buffer decode. q [N,H,dk], k_new [N,dk], v_new [N,H,dv], k_cache [N,W,dk] and
    v_cache [N,H,W,dv] (updated in place at slot pos mod W), pos [N] int64. Returns o [N,H,dv]."""
    _need(q, "q", None, 3)
    for n, t, nd in (("k_new", k_new, 2), ("v_new", v_new, 3), ("k_cache", k_cache, 3),
                     ("v_cache", v_cache, 4)):
        _need(t, n, q.dtype, nd)
    _need(pos, "pos", torch.int64, 1)
    N, H, dk = q.shape
    dv = v_new.shape[-1]
    W = int(window)
    if (tuple(k_new.shape) != (N, dk) or tuple(k_cache.shape) != (N, W, dk)
            or tuple(v_cache.shape) != (N, H, W, dv) or pos.shape[0] != N):
        raise ValueError("shape mismatch")
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, 3)
    st = load_library().rod_swska_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                         _ptr(v_cache), _ptr(pos), _ptr(o), N, H, dk, dv, W,
                                         float(scale or 0.0), _dtype_code(q), _stream(stream))
    _raise_on("rod_swska_decode", st)
    return o


def swska_cache_fill(k, v, k_cache, v_cache, window, stream=None):
    """Prefill -> decode hand-off: k [B,T,dk], v [B,H,T,dv] into the ring buffers k_cache
    [B,W,dk], v_cache [B,H,W,dv] (position p of the last W goes to slot p mod W)."""
    _need(k, "k", None, 3)
    _need(v, "v", k.dtype, 4)
    _need(k_cache, "k_cache", k.dtype, 3)
    _need(v_cache, "v_cache", k.dtype, 4)
    B, T, dk = k.shape
    H, dv = v.shape[1], v.shape[-1]
    W = int(window)
    if (tuple(v.shape) != (B, H, T, dv) or tuple(k_cache.shape) != (B, W, dk)
            or tuple(v_cache.shape) != (B, H, W, dv)):
        raise ValueError("shape mismatch")
    st = load_library().rod_swska_cache_fill(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), B, H, T,
                                             dk, dv, W, _dtype_code(k), _stream(stream))
    _raise_on("rod_swska_cache_fill", st)
    return k_cache, v_cache


def swska_decode_paged(q, k_new, v_new, k_pool, v_pool, block_table, page_size, pos, window,
                       scale=None, o=None, stream=None):
    """Ring-buffer decode over a paged window cache: k_pool [P,page,dk], v_pool [P,H,page,dv]
    (bf16), block_table [N, W/page] int32 (logical page -> physical page). Returns o [N,H,dv]."""
    _need(q, "q", None, 3)
    for n, t, nd in (("k_new", k_new, 2), ("v_new", v_new, 3), ("k_pool", k_pool, 3),
                     ("v_pool", v_pool, 4)):
        _need(t, n, q.dtype, nd)
    _need(pos, "pos", torch.int64, 1)
    _need(block_table, "block_table", torch.int32, 2)
    N, H, dk = q.shape
    dv = v_new.shape[-1]
    W, page = int(window), int(page_size)
    pps = W // page if page > 0 else 0
    if (tuple(k_new.shape) != (N, dk) or tuple(block_table.shape) != (N, pps)
            or tuple(k_pool.shape[1:]) != (page, dk) or tuple(v_pool.shape[1:]) != (H, page, dv)
            or v_pool.shape[0] != k_pool.shape[0] or pos.shape[0] != N):
        raise ValueError("shape mismatch")
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, 3)
    st = load_library().rod_swska_decode_paged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool),
                                               _ptr(v_pool), _ptr(block_table), page, pps, _ptr(pos),
                                               _ptr(o), N, H, dk, dv, W, float(scale or 0.0),
                                               _dtype_code(q), _stream(stream))
    _raise_on("rod_swska_decode_paged", st)
    return o


def gla_backward(q, k, v, g, dO, state0=None, dstate_final=None, workspace=None, stream=None):
    """Gradients of gla_prefill: q, k, v, dO [B,H,T,*] (dtype), g fp32, state0 [B,H,dk,dv] fp32
    (None: zeros), dstate_final [B,H,dk,dv] fp32 or None. Returns (dq, dk, dv, dg, dstate0)."""
    _need(q, "q", None, 4)
    for n, t in (("k", k), ("v", v), ("dO", dO)):
        _need(t, n, q.dtype, 4)
    _need(g, "g", torch.float32, 4)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (B, H, T, dk) or tuple(g.shape) != (B, H, T, dk) or tuple(dO.shape) != (B, H, T, dv):
        raise ValueError("shape mismatch")
    if state0 is None:
        state0 = torch.zeros(B, H, dk, dv, dtype=torch.float32, device=q.device)
    _need(state0, "state0", torch.float32, 4)
    if dstate_final is not None:
        _need(dstate_final, "dstate_final", torch.float32, 4)
    lib = load_library()
    need = lib.rod_gla_backward_workspace_size(B, H, T, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg = torch.empty_like(g)
    dS0 = torch.empty_like(state0)
    st = lib.rod_gla_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(state0), _ptr(dO),
                              None if dstate_final is None else _ptr(dstate_final), _ptr(dq),
                              _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(dS0), B, H, T, dk, dv,
                              _dtype_code(q), _ptr(workspace), workspace.numel(), _stream(stream))
    _raise_on("rod_gla_backward", st)
    return dq, dk_, dv_, dg, dS0


def swska_backward(q, k, v, dO, window, scale=None, workspace=None, stream=None):
    """Gradients of swska_prefill: q [B,H,T,dk], shared k [B,T,dk], v and dO [B,H,T,dv].
    Returns (dq, dk, dv) in the layouts and dtype of q, k, v."""
    _need(q, "q", None, 4)
    _need(k, "k", q.dtype, 3)
    _need(v, "v", q.dtype, 4)
    _need(dO, "dO", q.dtype, 4)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if tuple(k.shape) != (B, T, dk) or tuple(v.shape[:3]) != (B, H, T) or tuple(dO.shape) != tuple(v.shape):
        raise ValueError("shape mismatch")
    lib = load_library()
    need = lib.rod_swska_backward_workspace_size(B, H, T)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = lib.rod_swska_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dq), _ptr(dk_), _ptr(dv_),
                                B, H, T, dk, dv, int(window), float(scale or 0.0), _dtype_code(q),
                                _ptr(workspace), workspace.numel(), _stream(stream))
    _raise_on("rod_swska_backward", st)
    return dq, dk_, dv_


def swska_backward_lse(q, k, v, o, lse, dO, window, scale=None, workspace=None, stream=None):
    """swska_backward given the forward's o and lse (from swska_prefill_lse with the same q, k, v,
    window and scale): the tensor-core route reads them instead of recomputing the forward.
    Returns (dq, dk, dv)."""
    _need(q, "q", None, 4)
    _need(k, "k", q.dtype, 3)
    _need(v, "v", q.dtype, 4)
    _need(o, "o", q.dtype, 4)
    _need(lse, "lse", torch.float32, 3)
    _need(dO, "dO", q.dtype, 4)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if (tuple(k.shape) != (B, T, dk) or tuple(v.shape[:3]) != (B, H, T) or tuple(dO.shape) != tuple(v.shape)
            or tuple(o.shape) != tuple(v.shape) or tuple(lse.shape) != (B, H, T)):
        raise ValueError("shape mismatch")
    lib = load_library()
    need = lib.rod_swska_backward_workspace_size(B, H, T)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = lib.rod_swska_backward_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk_),
                                    _ptr(dv_), B, H, T, dk, dv, int(window), float(scale or 0.0), _dtype_code(q),
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    _raise_on("rod_swska_backward_lse", st)
    return dq, dk_, dv_


def _need_codes(t, name, ndim):
    """An FP8 cache: a CUDA tensor of one-byte E4M3 codes (uint8 or float8_e4m3fn), contiguous."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise ValueError(f"{name} must hold E4M3 codes (uint8 or float8_e4m3fn), got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def swska_decode_fp8(q, k_new, v_new, k_cache, v_cache, pos, window, scale=None, k_scale=1.0,
                     v_scale=1.0, o=None, stream=None):
    """Ring-buffer decode over FP8 caches (SALA blog §4.3): k_cache [N,W,dk] and v_cache
    [N,H,W,dv] hold E4M3 codes (value = code * scale) and are updated in place at slot pos mod W
    with the quantized new token. q [N,H,dk], k_new [N,dk], v_new [N,H,dv] bf16, pos [N] int64.
    Returns o [N,H,dv] bf16."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_new, "k_new", torch.bfloat16, 2)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need_codes(k_cache, "k_cache", 3)
    _need_codes(v_cache, "v_cache", 4)
    _need(pos, "pos", torch.int64, 1)
    N, H, dk = q.shape
    dv = v_new.shape[-1]
    W = int(window)
    if (tuple(k_new.shape) != (N, dk) or tuple(k_cache.shape) != (N, W, dk)
            or tuple(v_cache.shape) != (N, H, W, dv) or pos.shape[0] != N):
        raise ValueError("shape mismatch")
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, 3)
    st = load_library().rod_swska_decode_fp8(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                             _ptr(v_cache), _ptr(pos), _ptr(o), N, H, dk, dv, W,
                                             float(scale or 0.0), float(k_scale), float(v_scale),
                                             _stream(stream))
    _raise_on("rod_swska_decode_fp8", st)
    return o


def swska_cache_fill_fp8(k, v, k_cache, v_cache, window, k_scale=1.0, v_scale=1.0, stream=None):
    """Prefill -> decode hand-off into FP8 rings: k [B,T,dk], v [B,H,T,dv] (bf16) quantized into
    k_cache [B,W,dk], v_cache [B,H,W,dv] (E4M3 codes of x / scale at slot p mod W)."""
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 4)
    _need_codes(k_cache, "k_cache", 3)
    _need_codes(v_cache, "v_cache", 4)
    B, T, dk = k.shape
    H, dv = v.shape[1], v.shape[-1]
    W = int(window)
    if (tuple(v.shape) != (B, H, T, dv) or tuple(k_cache.shape) != (B, W, dk)
            or tuple(v_cache.shape) != (B, H, W, dv)):
        raise ValueError("shape mismatch")
    st = load_library().rod_swska_cache_fill_fp8(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), B, H, T,
                                                 dk, dv, W, float(k_scale), float(v_scale), _stream(stream))
    _raise_on("rod_swska_cache_fill_fp8", st)
    return k_cache, v_cache
