"""Pins for the fp64 CPU oracle: it is checked against things other than itself.

Each test compares the oracle with an independent statement of what the pages and the
mathematics fix: hand-worked examples (tests/golden), the O(T^2) unrolled form of the
recurrence, closed forms for special gates (g = 1: causal linear attention, SALA blog §2.2
with phi = identity; g = 0: state reset; scalar g: geometric decay, SALA blog §4.3 tip 3),
PyTorch's fp64 CPU softmax attention as a library routine (window >= T is full causal
attention; SKA equals multi-head attention with the shared K replicated per head, CodeFuse
Rodimus* article Fig. 4), window edge cases (W = 1, uniform softmax), and decode/prefill and
split-prefill consistency (SALA blog §3.3 chunked prefill, §3.4 train/infer consistency).
Inputs use dk != dv and per-channel gates so that a transposed operand, a row/column mix-up,
an off-by-one window or a dropped term fails at least one test (tests/test_oracle_mutations.py
plants such mistakes and checks that they are caught).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")
RTOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _gla_case(B=2, H=3, T=23, dk=5, dv=7, seed=0, gate="rand"):
    r = _rng(seed)
    q = r.standard_normal((B, H, T, dk)).astype(np.float32)
    k = r.standard_normal((B, H, T, dk)).astype(np.float32)
    v = r.standard_normal((B, H, T, dv)).astype(np.float32)
    if gate == "rand":
        g = r.uniform(0.05, 1.0, (B, H, T, dk)).astype(np.float32)
    elif gate == "one":
        g = np.ones((B, H, T, dk), np.float32)
    elif gate == "zero":
        g = np.zeros((B, H, T, dk), np.float32)
    else:
        g = np.full((B, H, T, dk), float(gate), np.float32)
    S0 = r.standard_normal((B, H, dk, dv))
    return q, k, v, g, S0


def _close(a, b, tol=RTOL):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"max abs err {err:.3e} > {tol * scale:.3e}"


# ------------------------------------------------------------------------------------------
# gated linear recurrence
# ------------------------------------------------------------------------------------------


def test_gla_hand_worked_example():
    gd = json.load(open(os.path.join(GOLD, "gla_hand_t3.json")))
    f = lambda x: np.asarray(x, np.float32)[None, None]
    o, S = oracle.gla_prefill(f(gd["q"]), f(gd["k"]), f(gd["v"]), f(gd["g"]),
                              np.asarray(gd["state0"], np.float64)[None, None])
    np.testing.assert_array_equal(o[0, 0], np.asarray(gd["o"], np.float64))
    np.testing.assert_array_equal(S[0, 0], np.asarray(gd["state"], np.float64))


def _unrolled(q, k, v, g, S0):
    """o_t = sum_{s<=t} sum_c q_tc k_sc (prod_{r=s+1..t} g_rc) v_s + sum_c q_tc (prod_{r<=t} g_rc) S0[c,:]
    and the final state, written as explicit products of gates (no recurrence)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    q, k, v, g = (x.astype(np.float64) for x in (q, k, v, g))
    o = np.zeros((B, H, T, dv))
    S = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            for t in range(T):
                acc = np.zeros(dv)
                for s in range(t + 1):
                    dec = np.prod(g[b, h, s + 1:t + 1], axis=0)          # [dk]
                    acc += np.sum(q[b, h, t] * k[b, h, s] * dec) * v[b, h, s]
                dec0 = np.prod(g[b, h, :t + 1], axis=0)
                acc += (q[b, h, t] * dec0) @ S0[b, h]
                o[b, h, t] = acc
            for s in range(T):
                dec = np.prod(g[b, h, s + 1:T], axis=0)
                S[b, h] += np.outer(k[b, h, s] * dec, v[b, h, s])
            S[b, h] += np.prod(g[b, h, :T], axis=0)[:, None] * S0[b, h]
    return o, S


@pytest.mark.parametrize("seed", [0, 1])
def test_gla_recurrence_equals_unrolled_masked_form(seed):
    q, k, v, g, S0 = _gla_case(seed=seed)
    o, S = oracle.gla_prefill(q, k, v, g, S0)
    o_ref, S_ref = _unrolled(q, k, v, g, S0)
    _close(o, o_ref)
    _close(S, S_ref)


def test_gla_g1_is_causal_linear_attention():
    q, k, v, g, S0 = _gla_case(gate="one", seed=3)
    o, S = oracle.gla_prefill(q, k, v, g, S0)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    T = q.shape[2]
    mask = np.tril(np.ones((T, T)))
    o_ref = (q64 @ np.swapaxes(k64, -1, -2) * mask) @ v64 + q64 @ S0
    S_ref = S0 + np.swapaxes(k64, -1, -2) @ v64
    _close(o, o_ref)
    _close(S, S_ref)


def test_gla_g0_resets_state():
    q, k, v, g, S0 = _gla_case(gate="zero", seed=4)
    o, S = oracle.gla_prefill(q, k, v, g, S0)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    o_ref = np.sum(q64 * k64, axis=-1, keepdims=True) * v64
    S_ref = k64[:, :, -1, :, None] * v64[:, :, -1, None, :]
    _close(o, o_ref)
    _close(S, S_ref)


def test_gla_scalar_gate_is_geometric_decay():
    gamma = 0.75
    q, k, v, g, S0 = _gla_case(gate=gamma, seed=5, T=17)
    o, S = oracle.gla_prefill(q, k, v, g, S0)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    T = q.shape[2]
    t = np.arange(T)
    D = np.where(t[:, None] >= t[None, :], gamma ** (t[:, None] - t[None, :]), 0.0)
    o_ref = (q64 @ np.swapaxes(k64, -1, -2) * D) @ v64 + (gamma ** (t + 1))[:, None] * (q64 @ S0)
    _close(o, o_ref)


def test_gla_decode_steps_equal_prefill():
    q, k, v, g, S0 = _gla_case(seed=6, T=11)
    o, S = oracle.gla_prefill(q, k, v, g, S0)
    St = S0.copy()
    for t in range(q.shape[2]):
        ot, St = oracle.gla_decode_step(q[:, :, t], k[:, :, t], v[:, :, t], g[:, :, t], St)
        np.testing.assert_array_equal(ot, o[:, :, t])
    np.testing.assert_array_equal(St, S)


@pytest.mark.parametrize("t1", [1, 9, 22])
def test_gla_split_prefill_hands_off_state(t1):
    q, k, v, g, S0 = _gla_case(seed=7)
    o, S = oracle.gla_prefill(q, k, v, g, S0)
    o1, S1 = oracle.gla_prefill(q[:, :, :t1], k[:, :, :t1], v[:, :, :t1], g[:, :, :t1], S0)
    o2, S2 = oracle.gla_prefill(q[:, :, t1:], k[:, :, t1:], v[:, :, t1:], g[:, :, t1:], S1)
    np.testing.assert_array_equal(np.concatenate([o1, o2], axis=2), o)
    np.testing.assert_array_equal(S2, S)


def test_gla_empty_sequence_keeps_state():
    q, k, v, g, S0 = _gla_case(T=0, seed=8)
    o, S = oracle.gla_prefill(q, k, v, g, S0)
    assert o.shape == (2, 3, 0, 7)
    np.testing.assert_array_equal(S, S0)


# ------------------------------------------------------------------------------------------
# sliding-window shared-key attention
# ------------------------------------------------------------------------------------------


def _ska_case(B=2, H=3, T=29, dk=6, dv=5, seed=0):
    r = _rng(100 + seed)
    q = r.standard_normal((B, H, T, dk)).astype(np.float32)
    k = r.standard_normal((B, T, dk)).astype(np.float32)
    v = r.standard_normal((B, H, T, dv)).astype(np.float32)
    return q, k, v


def _sdpa(q, k_rep, v, mask=None, causal=False, scale=None):
    t = lambda x: torch.from_numpy(np.asarray(x, np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k_rep), t(v), attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal, scale=scale).numpy()


def test_swska_hand_worked_example():
    gd = json.load(open(os.path.join(GOLD, "swska_hand_t4.json")))
    q = np.asarray(gd["q"], np.float32)[None, None, :, None]
    k = np.asarray(gd["k"], np.float32)[None, :, None]
    v = np.asarray(gd["v"], np.float32)[None, None, :, None]
    o = oracle.swska_prefill(q, k, v, gd["window"], scale=1.0)
    _close(o[0, 0, :, 0], gd["o"], 1e-15)
    o3 = oracle.swska_prefill(q, k, v, 3, scale=1.0)
    _close(o3[0, 0, :, 0], gd["o_window3"], 1e-15)


def test_swska_two_key_closed_form():
    # one query against two keys: o = (v0 + e^{s1-s0} v1) / (1 + e^{s1-s0})
    q = np.array([0.0, 1.5], np.float32)[None, None, :, None]
    k = np.array([0.5, 2.0], np.float32)[None, :, None]
    v = np.array([2.0, -4.0], np.float32)[None, None, :, None]
    o = oracle.swska_prefill(q, k, v, 2, scale=1.0)
    e = math.exp(1.5 * 2.0 - 1.5 * 0.5)
    _close(o[0, 0, 1, 0], (2.0 - 4.0 * e) / (1.0 + e), 1e-15)


@pytest.mark.parametrize("W", [29, 64])
def test_swska_window_ge_T_is_full_causal_attention(W):
    q, k, v = _ska_case(seed=1)
    H = q.shape[1]
    o = oracle.swska_prefill(q, k, v, W)
    k_rep = np.repeat(k[:, None], H, axis=1)
    _close(o, _sdpa(q, k_rep, v, causal=True), 1e-12)


@pytest.mark.parametrize("W", [1, 2, 5, 17])
def test_swska_shared_key_equals_mha_with_replicated_key(W):
    q, k, v = _ska_case(seed=2)
    B, H, T, _ = q.shape
    o = oracle.swska_prefill(q, k, v, W, scale=0.3)
    k_rep = np.repeat(k[:, None], H, axis=1)
    # boolean "may attend" mask built from the window as a set of positions
    allowed = np.zeros((T, T), bool)
    for t in range(T):
        allowed[t, list(range(max(0, t - W + 1), t + 1))] = True
    _close(o, _sdpa(q, k_rep, v, mask=allowed, scale=0.3), 1e-12)


def test_swska_window_one_is_identity_on_v():
    q, k, v = _ska_case(seed=3)
    o = oracle.swska_prefill(q, k, v, 1)
    np.testing.assert_array_equal(o, v.astype(np.float64))


@pytest.mark.parametrize("W", [3, 8])
def test_swska_zero_query_averages_the_window(W):
    q, k, v = _ska_case(seed=4)
    q[:] = 0
    o = oracle.swska_prefill(q, k, v, W)
    T = q.shape[2]
    ref = np.stack([v[:, :, max(0, t - W + 1):t + 1].astype(np.float64).mean(axis=2)
                    for t in range(T)], axis=2)
    _close(o, ref, 1e-14)


def test_swska_row_sampling_matches_full_output():
    q, k, v = _ska_case(seed=5)
    B, H, T, _ = q.shape
    o = oracle.swska_prefill(q, k, v, 7)
    rows = np.array([0, 5, T - 1, T, 2 * T + 3, B * H * T - 1])
    osub = oracle.swska_prefill(q, k, v, 7, rows=rows)
    np.testing.assert_array_equal(osub, o.reshape(-1, o.shape[-1])[rows])


@pytest.mark.parametrize("W,positions", [(8, [0, 3, 7, 8, 13, 30]), (5, [4, 5, 6, 9, 24])])
def test_swska_ring_buffer_decode_equals_prefill_row(W, positions):
    """Fill a ring buffer from a sequence, then decode position P: the output must equal the
    prefill output row P (SALA blog §3.3 rolling window; §3.4 consistency)."""
    H, dk, dv = 3, 6, 5
    T = max(positions) + 1
    q, k, v = _ska_case(B=1, H=H, T=T, dk=dk, dv=dv, seed=6)
    o_pre = oracle.swska_prefill(q, k, v, W)
    N = len(positions)
    kc = np.zeros((N, W, dk), np.float32)
    vc = np.zeros((N, H, W, dv), np.float32)
    for n, P in enumerate(positions):           # tokens before P sit in slot p mod W
        for p in range(max(0, P - W + 1), P):
            kc[n, p % W] = k[0, p]
            vc[n, :, p % W] = v[0, :, p]
    P = np.asarray(positions)
    o, kc2, vc2 = oracle.swska_decode(q[0][:, P].transpose(1, 0, 2), k[0, P], v[0][:, P].transpose(1, 0, 2),
                                      kc, vc, P, W)
    _close(o, o_pre[0][:, P].transpose(1, 0, 2), 1e-13)
    for n, p in enumerate(positions):
        np.testing.assert_array_equal(kc2[n, p % W], k[0, p])
        np.testing.assert_array_equal(vc2[n, :, p % W], v[0, :, p])


@pytest.mark.parametrize("W,T,steps", [(8, 5, 6), (8, 8, 4), (5, 23, 7), (1, 4, 3)])
def test_swska_cache_fill_then_decode_continues_the_prefill(W, T, steps):
    """Prefill -> decode hand-off (SALA blog §3.3): fill the ring buffers from a T-token prefill,
    then decode positions T .. T+steps-1 one at a time; each decode output equals the prefill
    output row of the whole sequence at that position, and slots the fill does not name keep
    their previous contents."""
    H, dk, dv, B = 3, 6, 5, 2
    total = T + steps
    q, k, v = _ska_case(B=B, H=H, T=total, dk=dk, dv=dv, seed=11)
    o_pre = oracle.swska_prefill(q, k, v, W)
    kc = np.full((B, W, dk), 9.0, np.float32)
    vc = np.full((B, H, W, dv), 9.0, np.float32)
    kc, vc = oracle.swska_cache_fill(k[:, :T], v[:, :, :T], kc, vc, W)
    if T < W:
        assert (kc[:, T:] == 9.0).all() and (vc[:, :, T:] == 9.0).all()
    for P in range(T, total):
        o, kc, vc = oracle.swska_decode(q[:, :, P], k[:, P], v[:, :, P], kc, vc,
                                        np.full(B, P, np.int64), W)
        _close(o, o_pre[:, :, P], 1e-13)


@pytest.mark.parametrize("W,T", [(8, 5), (8, 8), (5, 23), (1, 4), (6, 13)])
def test_swska_cache_fill_equals_decode_writes(W, T):
    """The hand-off fill leaves the caches exactly as T decode steps at positions 0 .. T-1
    would (each writes its token at slot p mod W; the ring rule of the decode is pinned by the
    decode tests above): the last W tokens, each in its slot, other slots untouched."""
    H, dk, dv, B = 2, 4, 3, 2
    q, k, v = _ska_case(B=B, H=H, T=T, dk=dk, dv=dv, seed=12)
    kc0 = np.full((B, W, dk), 9.0, np.float32)
    vc0 = np.full((B, H, W, dv), 9.0, np.float32)
    kf, vf = oracle.swska_cache_fill(k, v, kc0, vc0, W)
    kd, vd = kc0, vc0
    for p in range(T):
        _, kd, vd = oracle.swska_decode(q[:, :, p], k[:, p], v[:, :, p], kd, vd,
                                        np.full(B, p, np.int64), W)
    np.testing.assert_array_equal(kf, kd)
    np.testing.assert_array_equal(vf, vd)


def test_swska_paged_decode_hand_worked_layout():
    """W = 16 slots in pages of 8, table [3, 1] over a pool of 4 pages: position 9 (slot 9,
    logical page 1) lands in physical page 1 at row 1; position 2 (slot 2, logical page 0) in
    physical page 3 at row 2; nothing else in the pools changes."""
    H, dk, dv, W, page = 2, 4, 3, 16, 8
    r = _rng(77)
    kp = np.full((4, page, dk), 5.0, np.float32)
    vp = np.full((4, H, page, dv), 5.0, np.float32)
    table = np.array([3, 1], np.int32)
    for P, (pg, row) in ((9, (1, 1)), (2, (3, 2))):
        q = r.standard_normal((1, H, dk)).astype(np.float32)
        kn = r.standard_normal((1, dk)).astype(np.float32)
        vn = r.standard_normal((1, H, dv)).astype(np.float32)
        before_k, before_v = kp.copy(), vp.copy()
        _, kp, vp = oracle.swska_decode_paged(q, kn, vn, kp, vp, table, page, np.array([P]), W)
        np.testing.assert_array_equal(kp[pg, row], kn[0])
        np.testing.assert_array_equal(vp[pg, :, row], vn[0])
        before_k[pg, row] = kn[0]
        before_v[pg, :, row] = vn[0]
        np.testing.assert_array_equal(kp, before_k)
        np.testing.assert_array_equal(vp, before_v)


@pytest.mark.parametrize("W,page", [(16, 8), (24, 8), (32, 16)])
def test_swska_paged_decode_continues_prefill_and_writes_only_its_pages(W, page):
    """Three sequences share a pool through a shuffled table with spare pages. Decoding every
    position of each sequence from an empty cache (each step writes its token through the table)
    reproduces the prefill rows of that sequence; afterwards exactly the pages the table names
    have been written and the spare pages still hold their fill value."""
    H, dk, dv, N = 2, 5, 4, 3
    pps = W // page
    T = W + 9
    q, k, v = _ska_case(B=N, H=H, T=T, dk=dk, dv=dv, seed=21)
    o_pre = oracle.swska_prefill(q, k, v, W)
    P_pages = N * pps + 3
    perm = _rng(5).permutation(P_pages).astype(np.int32)
    table = perm[:N * pps]
    kp = np.full((P_pages, page, dk), 7.0, np.float32)
    vp = np.full((P_pages, H, page, dv), 7.0, np.float32)
    for t in range(T):
        o, kp, vp = oracle.swska_decode_paged(q[:, :, t], k[:, t], v[:, :, t], kp, vp, table, page,
                                              np.full(N, t, np.int64), W)
        _close(o, o_pre[:, :, t], 1e-13)
    used = set(table.tolist())
    for pg in range(P_pages):
        untouched = bool((kp[pg] == 7.0).all() and (vp[pg] == 7.0).all())
        assert untouched == (pg not in used), pg


# ------------------------------------------------------------------------------------------
# backward of the recurrence
# ------------------------------------------------------------------------------------------


def _gla_loss(q, k, v, g, S0, dO, dSf):
    o, ST = oracle.gla_prefill(q, k, v, g, S0)
    return float(np.sum(o * dO) + np.sum(ST * dSf))


def test_gla_backward_finite_differences():
    """Central differences of L = sum(o . dO) + sum(S_T . dS_final) on a tiny case. Inputs are
    multiples of 2^-8 and the step is 2^-8, so every perturbed input is exact in fp32; L is
    linear in q, k, v, S_0 (central differences exact up to rounding) and a degree-T polynomial
    in the gates (truncation ~h^2)."""
    B, H, T, dk, dv = 1, 1, 7, 3, 2
    r = _rng(31)
    grid = lambda shape, lo, hi: (np.round(r.uniform(lo, hi, shape) * 256) / 256).astype(np.float32)
    q, k = grid((B, H, T, dk), -1, 1), grid((B, H, T, dk), -1, 1)
    v, g = grid((B, H, T, dv), -1, 1), grid((B, H, T, dk), 0.3, 0.95)
    S0 = r.standard_normal((B, H, dk, dv))
    dO = r.standard_normal((B, H, T, dv)).astype(np.float32)
    dSf = r.standard_normal((B, H, dk, dv)).astype(np.float32)
    dq, dk_, dv_, dg, dS0 = oracle.gla_backward(q, k, v, g, dO, S0, dSf)
    h = 2.0 ** -8
    for name, x, grad, tol in (("q", q, dq, 1e-9), ("k", k, dk_, 1e-9), ("v", v, dv_, 1e-9),
                               ("g", g, dg, 2e-4)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v, "g": g}
            fp = _gla_loss(*[xp if n == name else args[n] for n in "qkvg"], S0, dO, dSf)
            fm = _gla_loss(*[xm if n == name else args[n] for n in "qkvg"], S0, dO, dSf)
            fd = (fp - fm) / (2 * h)
            assert abs(fd - grad[idx]) <= tol * max(1.0, abs(fd)), (name, idx, fd, grad[idx])
    for idx in np.ndindex(S0.shape):
        Sp, Sm = S0.copy(), S0.copy()
        Sp[idx] += h
        Sm[idx] -= h
        fd = (_gla_loss(q, k, v, g, Sp, dO, dSf) - _gla_loss(q, k, v, g, Sm, dO, dSf)) / (2 * h)
        assert abs(fd - dS0[idx]) <= 1e-9 * max(1.0, abs(fd))


def test_gla_backward_matches_torch_autograd():
    """The same gradients from PyTorch autograd through a float64 loop of the recurrence."""
    torch = pytest.importorskip("torch")
    B, H, T, dk, dv = 2, 2, 70, 5, 4
    r = _rng(32)
    q, k = [r.standard_normal((B, H, T, dk)).astype(np.float32) for _ in range(2)]
    v = r.standard_normal((B, H, T, dv)).astype(np.float32)
    g = r.uniform(0.2, 1.0, (B, H, T, dk)).astype(np.float32)
    S0 = r.standard_normal((B, H, dk, dv))
    dO = r.standard_normal((B, H, T, dv)).astype(np.float32)
    dSf = r.standard_normal((B, H, dk, dv)).astype(np.float32)
    tq, tk, tv, tg = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v, g)]
    tS0 = torch.tensor(S0, requires_grad=True)
    S, outs = tS0, []
    for t in range(T):
        S = tg[:, :, t, :, None] * S + tk[:, :, t, :, None] * tv[:, :, t, None, :]
        outs.append(torch.einsum("bhc,bhcj->bhj", tq[:, :, t], S))
    o = torch.stack(outs, dim=2)
    loss = (o * torch.tensor(dO, dtype=torch.float64)).sum() + (S * torch.tensor(dSf, dtype=torch.float64)).sum()
    loss.backward()
    got = oracle.gla_backward(q, k, v, g, dO, S0, dSf)
    for name, ref, val in zip(("dq", "dk", "dv", "dg", "dS0"), (tq, tk, tv, tg, tS0), got):
        np.testing.assert_allclose(val, ref.grad.numpy(), rtol=1e-10, atol=1e-10, err_msg=name)


def test_gla_backward_gate_identity():
    """d(log g_r) = g_r dg_r equals the reverse cumulative sum over t >= r of q_t dq_t - k_t dk_t,
    plus the final-state term sum_j dS_final[c, j] S_T[c, j] (pairs s < r <= t of the unrolled
    form), an identity independent of how dg was computed."""
    B, H, T, dk, dv = 2, 3, 130, 6, 5
    r = _rng(33)
    q, k = [r.standard_normal((B, H, T, dk)).astype(np.float32) for _ in range(2)]
    v = r.standard_normal((B, H, T, dv)).astype(np.float32)
    g = r.uniform(0.5, 1.0, (B, H, T, dk)).astype(np.float32)
    S0 = r.standard_normal((B, H, dk, dv))
    dO = r.standard_normal((B, H, T, dv)).astype(np.float32)
    dSf = r.standard_normal((B, H, dk, dv)).astype(np.float32)
    dq, dk_, _, dg, _ = oracle.gla_backward(q, k, v, g, dO, S0, dSf)
    _, ST = oracle.gla_prefill(q, k, v, g, S0)
    F = np.sum(dSf.astype(np.float64) * ST, axis=-1)              # [B,H,dk]
    terms = q.astype(np.float64) * dq - k.astype(np.float64) * dk_  # [B,H,T,dk]
    rev = np.flip(np.cumsum(np.flip(terms, axis=2), axis=2), axis=2) + F[:, :, None, :]
    _close(g.astype(np.float64) * dg, rev, 1e-10)


# ------------------------------------------------------------------------------------------
# backward of SW-SKA
# ------------------------------------------------------------------------------------------


def test_swska_backward_finite_differences():
    """Central differences of L = sum(o . dO) on a tiny case (step 2^-8 on inputs that are
    multiples of 2^-8, so perturbed inputs are exact in fp32)."""
    B, H, T, dk, dv, W = 1, 2, 6, 3, 2, 4
    r = _rng(41)
    grid = lambda shape: (np.round(r.uniform(-1, 1, shape) * 256) / 256).astype(np.float32)
    q, k, v = grid((B, H, T, dk)), grid((B, T, dk)), grid((B, H, T, dv))
    dO = r.standard_normal((B, H, T, dv)).astype(np.float32)
    dq, dk_, dv_ = oracle.swska_backward(q, k, v, dO, W)
    loss = lambda q_, k_, v_: float(np.sum(oracle.swska_prefill(q_, k_, v_, W) * dO))
    h = 2.0 ** -8
    for name, x, grad in (("q", q, dq), ("k", k, dk_), ("v", v, dv_)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = lambda xx: [xx if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            fd = (loss(*args(xp)) - loss(*args(xm))) / (2 * h)
            assert abs(fd - grad[idx]) <= 2e-5 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


@pytest.mark.parametrize("W", [1, 5, 40])
def test_swska_backward_matches_torch_autograd(W):
    """The same gradients from PyTorch autograd through float64 attention with the key
    replicated over heads (its gradient is the sum of the replicas') and an explicit window
    mask."""
    torch = pytest.importorskip("torch")
    B, H, T, dk, dv = 2, 3, 33, 6, 5
    q, k, v = _ska_case(B=B, H=H, T=T, dk=dk, dv=dv, seed=42)
    dO = _rng(43).standard_normal((B, H, T, dv)).astype(np.float32)
    tq, tk, tv = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v)]
    t = torch.arange(T)
    mask = (t[None, :] <= t[:, None]) & (t[None, :] > t[:, None] - W)
    s = torch.einsum("bhtc,bjc->bhtj", tq, tk) / np.sqrt(dk)
    s = s.masked_fill(~mask, float("-inf"))
    o = torch.einsum("bhtj,bhjd->bhtd", torch.softmax(s, dim=-1), tv)
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    dq, dk_, dv_ = oracle.swska_backward(q, k, v, dO, W)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk_, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv_, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


# ------------------------------------------------------------------------------------------
# FP8 (E4M3) window cache (SALA blog §4.3: the KV cache stored in FP8)
# ------------------------------------------------------------------------------------------


def test_e4m3_codebook_closed_forms():
    """Values fixed by the E4M3 definition (1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
    exponent field 0 subnormal, S.1111.111 NaN): zero, the subnormal step 2^-9, the smallest
    normal 2^-6, one, the largest finite 448, the sign bit."""
    d = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert d[0x00] == 0.0 and math.copysign(1.0, d[0x80]) == -1.0
    assert d[0x01] == 2.0 ** -9 and d[0x07] == 7 * 2.0 ** -9
    assert d[0x08] == 2.0 ** -6 and d[0x38] == 1.0 and d[0x39] == 1.125
    assert d[0x77] == 1.875 * 2 ** 7 and d[0x7E] == 448.0 and d[0xFE] == -448.0
    assert np.isnan(d[0x7F]) and np.isnan(d[0xFF])
    finite = d[np.isfinite(d)]
    assert finite.size == 254  # every code but the two NaNs
    pos = d[:0x7F]
    assert (np.diff(pos) > 0).all()  # non-negative codes in increasing order


def test_e4m3_encode_round_trip_ties_and_saturation():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals), codes)  # exact values round-trip
    # midpoints between neighbouring codes go to the even code
    lo = oracle.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8))
    hi = oracle.e4m3_decode(np.arange(1, 0x7F, dtype=np.uint8))
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)  # the midpoints are exact in fp32
    enc = oracle.e4m3_encode(mid).astype(int)
    expect = np.where(np.arange(0, 0x7E) % 2 == 0, np.arange(0, 0x7E), np.arange(1, 0x7F))
    np.testing.assert_array_equal(enc, expect)
    # saturation at +-448, NaN stays NaN
    np.testing.assert_array_equal(oracle.e4m3_encode(np.array([449, 464, 1e9, np.inf, -500, -np.inf], np.float32)),
                                  np.array([0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE], np.uint8))
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F
    # the scale divides in fp32 before rounding
    np.testing.assert_array_equal(oracle.e4m3_encode(np.array([3.0], np.float32), scale=2.0),
                                  oracle.e4m3_encode(np.array([1.5], np.float32)))


def test_e4m3_encode_matches_torch_float8_in_range():
    """PyTorch's float8_e4m3fn conversion (a library routine, round to nearest even) agrees code
    for code on values inside the finite range (PyTorch does not saturate beyond it)."""
    r = _rng(7).normal(0, 40, 200000).astype(np.float32)
    r = np.concatenate([r[np.abs(r) <= 448], _rng(8).uniform(-2 ** -5, 2 ** -5, 20000).astype(np.float32)])
    t = torch.from_numpy(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(r), t)


@pytest.mark.parametrize("W,T,steps,ks,vs", [(8, 5, 6, 1.0, 1.0), (5, 23, 7, 0.25, 2.0), (1, 4, 3, 1.0, 0.5)])
def test_swska_fp8_cache_fill_then_decode_equals_prefill_of_dequantized_kv(W, T, steps, ks, vs):
    """With FP8 rings, decode reads value(code) * scale: filling the rings from a T-token prefill
    and decoding positions T .. T+steps-1 reproduces the (pinned) fp64 prefill of the whole
    sequence run on the dequantized keys and values, e4m3(x / scale) * scale."""
    H, dk, dv, B = 3, 6, 5, 2
    total = T + steps
    q, k, v = _ska_case(B=B, H=H, T=total, dk=dk, dv=dv, seed=21)
    kq = (oracle.e4m3_decode(oracle.e4m3_encode(k, ks)) * np.float32(ks)).astype(np.float32)
    vq = (oracle.e4m3_decode(oracle.e4m3_encode(v, vs)) * np.float32(vs)).astype(np.float32)
    o_pre = oracle.swska_prefill(q, kq, vq, W)
    kc = np.full((B, W, dk), 0x55, np.uint8)
    vc = np.full((B, H, W, dv), 0x55, np.uint8)
    kc, vc = oracle.swska_cache_fill_fp8(k[:, :T], v[:, :, :T], kc, vc, W, ks, vs)
    if T < W:
        assert (kc[:, T:] == 0x55).all() and (vc[:, :, T:] == 0x55).all()
    for P in range(T, total):
        o, kc, vc = oracle.swska_decode_fp8(q[:, :, P], k[:, P], v[:, :, P], kc, vc,
                                            np.full(B, P, np.int64), W, k_scale=ks, v_scale=vs)
        _close(o, o_pre[:, :, P], 1e-13)


def test_swska_fp8_decode_writes_codes_and_rejects_negative_position():
    H, dk, dv, N, W = 2, 4, 3, 3, 6
    r = _rng(23)
    q = r.standard_normal((N, H, dk)).astype(np.float32)
    kn = r.standard_normal((N, dk)).astype(np.float32)
    vn = r.standard_normal((N, H, dv)).astype(np.float32)
    kc = oracle.e4m3_encode(r.standard_normal((N, W, dk)).astype(np.float32))
    vc = oracle.e4m3_encode(r.standard_normal((N, H, W, dv)).astype(np.float32))
    pos = np.array([9, 2, -1], np.int64)
    o, kc2, vc2 = oracle.swska_decode_fp8(q, kn, vn, kc, vc, pos, W, k_scale=0.5, v_scale=0.5)
    np.testing.assert_array_equal(kc2[0, 9 % W], oracle.e4m3_encode(kn[0], 0.5))
    np.testing.assert_array_equal(vc2[1, :, 2], oracle.e4m3_encode(vn[1], 0.5))
    np.testing.assert_array_equal(kc2[2], kc[2])  # the rejected sequence's cache is untouched
    np.testing.assert_array_equal(vc2[2], vc[2])
    assert np.isnan(o[2]).all() and np.isfinite(o[:2]).all()
    # only the new slot changed for the accepted sequences
    changed = (kc2 != kc).any(axis=-1)
    assert not changed[0, [s for s in range(W) if s != 9 % W]].any()
