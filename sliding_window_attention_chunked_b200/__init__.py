"""Rodimus+ token-mixing hot path on one NVIDIA B200 (sm_100a).

A thin ctypes binding over ``librod.so`` (C ABI in ``include/rod.h``): every call here only
checks and marshals torch CUDA tensors into the library, which runs every step of the path in
its own CUDA kernels. There is no CPU fallback: without the built library (or without a GPU)
the calls raise.

    gla_prefill(q, k, v, g, state, chunk=64)       chunkwise prefill of the gated recurrence
    gla_decode_step(q, k, v, g, state)              one fused recurrent decode step
    gla_backward(q, k, v, g, dO, state0, dstate_final)   gradients of the recurrence
    swska_prefill(q, k, v, window, scale=None)      sliding-window shared-key attention
    swska_backward(q, k, v, dO, window)             gradients of the attention
    swska_prefill_lse(q, k, v, window)              the attention and each row's log-sum-exp
    swska_backward_lse(q, k, v, o, lse, dO, window) gradients from the forward's o and lse
    swska_decode(q, k_new, v_new, k_cache, v_cache, pos, window)   ring-buffer decode
    swska_cache_fill(k, v, k_cache, v_cache, window)   prefill -> decode ring-buffer hand-off
    swska_decode_paged(q, k_new, v_new, k_pool, v_pool, block_table, page_size, pos, window)
                                                    decode over a paged window cache
    swska_decode_fp8(q, k_new, v_new, k_cache, v_cache, pos, window, k_scale=1, v_scale=1)
                                                    decode over an FP8 (E4M3) window cache
    swska_cache_fill_fp8(k, v, k_cache, v_cache, window, k_scale=1, v_scale=1)
                                                    hand-off into FP8 rings
"""
from ._binding import (  # noqa: F401
    ROD_BF16,
    ROD_FP32,
    RodError,
    abi_version,
    check,
    gla_backward,
    gla_decode_step,
    gla_prefill,
    gla_prefill_noalloc,
    gla_prefill_workspace_size,
    launch_count,
    library_path,
    load_library,
    swska_backward,
    swska_backward_lse,
    swska_cache_fill,
    swska_cache_fill_fp8,
    swska_decode,
    swska_decode_fp8,
    swska_decode_paged,
    swska_prefill,
    swska_prefill_lse,
    test_expire_waits,
)
