"""The oracle's row log-sum-exp of SW-SKA (rodref_swska_prefill_lse), pinned on the CPU.

lse[b,h,t] = log sum over the window of t of exp(scale q[b,h,t] . k[b,j]) is checked against
what the mathematics fixes, not against the oracle's own formula:
- brute force: scipy's logsumexp of numpy-computed scores on small random cases;
- window 1: the single score scale * q_t . k_t;
- equal keys in a window of n: score + log n;
- large logits (scores near 800, where exp overflows without the maximum shift): finite and
  equal to the brute force;
- the output rows: exactly those of rodref_swska_prefill.
"""
import numpy as np
from scipy.special import logsumexp

import oracle


def _inputs(B, H, T, d, seed, mag=1.0):
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal((B, H, T, d)) * mag).astype(np.float32)
    k = (rng.standard_normal((B, T, d)) * mag).astype(np.float32)
    v = rng.standard_normal((B, H, T, d)).astype(np.float32)
    return q, k, v


def _brute(q, k, W, scale):
    B, H, T, d = q.shape
    out = np.empty((B, H, T))
    for b in range(B):
        for h in range(H):
            for t in range(T):
                j0 = max(0, t - W + 1)
                s = scale * (k[b, j0:t + 1].astype(np.float64) @ q[b, h, t].astype(np.float64))
                out[b, h, t] = logsumexp(s)
    return out


def test_lse_matches_brute_force():
    for (B, H, T, d, W, seed) in [(1, 2, 9, 8, 4, 0), (2, 3, 40, 16, 7, 1), (1, 1, 33, 32, 100, 2)]:
        q, k, v = _inputs(B, H, T, d, seed)
        o, lse = oracle.swska_prefill_lse(q, k, v, W)
        np.testing.assert_allclose(lse, _brute(q, k, W, 1 / np.sqrt(d)), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(o, oracle.swska_prefill(q, k, v, W))


def test_lse_window_one_is_the_score():
    q, k, v = _inputs(1, 2, 12, 8, 3)
    _, lse = oracle.swska_prefill_lse(q, k, v, 1, scale=0.25)
    s = 0.25 * np.einsum("bhtc,btc->bht", q.astype(np.float64), k.astype(np.float64))
    np.testing.assert_allclose(lse, s, rtol=0, atol=1e-12)


def test_lse_equal_keys_add_log_count():
    q, k, v = _inputs(1, 1, 10, 4, 4)
    k[0, :] = k[0, 0]  # every key the same: every score in a row equal
    W = 4
    _, lse = oracle.swska_prefill_lse(q, k, v, W, scale=1.0)
    s = np.einsum("bhtc,c->bht", q.astype(np.float64), k[0, 0].astype(np.float64))
    n = np.minimum(np.arange(10) + 1, W)
    np.testing.assert_allclose(lse[0, 0], s[0, 0] + np.log(n), rtol=0, atol=1e-12)


def test_lse_large_logits_stay_finite():
    q, k, v = _inputs(1, 2, 20, 16, 5, mag=7.0)  # scores of several hundred
    _, lse = oracle.swska_prefill_lse(q, k, v, 6, scale=1.0)
    assert np.all(np.isfinite(lse)) and np.max(np.abs(lse)) > 200
    np.testing.assert_allclose(lse, _brute(q, k, 6, 1.0), rtol=1e-15, atol=1e-10)


def test_lse_rows_subset():
    q, k, v = _inputs(2, 2, 15, 8, 6)
    o, lse = oracle.swska_prefill_lse(q, k, v, 5)
    rows = np.array([0, 7, 14, 31, 59])
    o_r, lse_r = oracle.swska_prefill_lse(q, k, v, 5, rows=rows)
    np.testing.assert_array_equal(lse_r, lse.reshape(-1)[rows])
    np.testing.assert_array_equal(o_r, o.reshape(-1, 8)[rows])
