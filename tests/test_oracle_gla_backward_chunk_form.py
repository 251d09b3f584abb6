"""The oracle's recurrence backward pinned to an independent derivation: the chunk form.

The recurrence S_t = diag(g_t) S_{t-1} + k_t^T v_t, o_t = q_t S_t (CodeFuse Rodimus* article,
Rodimus block) is differentiated here chunk by chunk, as a tensor-core backward would do it,
instead of step by step as the oracle does. Within a chunk with incoming state S_in and
gradient dS_out reaching its last state from later chunks, let P(a, b) = prod_{a<=u<=b} g_u per
key channel (1 when a > b). Then, with the future gradient of S_t written out,
    D_t = sum_{r>=t} P(t+1, r) q_r^T dO_r + P(t+1, C-1) dS_out,
one has:
    dq_t   = (dO_t S_in^T) . P(0, t) + sum_{s<=t} (dO_t . v_s) k_s . P(s+1, t)
    dk_s   = sum_{t>=s} (dO_t . v_s) q_t . P(s+1, t) + (v_s dS_out^T) . P(s+1, C-1)
    dv_s   = sum_{t>=s} ((q_t . P(s+1, t)) . k_s) dO_t + (k_s . P(s+1, C-1)) dS_out
    dS_in  = sum_t P(0, t) q_t^T dO_t + diag(P(0, C-1)) dS_out       (handed to the chunk before)
    dg_t   = sum_j D_t[:, j] S_{t-1}[:, j]
with dg in four terms: the pairing of the two parts of D_t with the two parts of S_{t-1} (the
incoming state, and the chunk's own earlier keys and values). Products over ranges are formed
directly, with no division by prefix products, so gates equal to 0 need no special case.
"""
import numpy as np
import pytest

import oracle


def range_products(g):
    """P[a, b, c] = prod_{a<=u<=b} g[u, c] (1 for a > b); P has shape (C+1, C+1, dk) so that
    the index C-1+1 = C is valid as an empty-range start."""
    C, dk = g.shape
    P = np.ones((C + 1, C + 1, dk))
    for a in range(C):
        acc = np.ones(dk)
        for b in range(a, C):
            acc = acc * g[b]
            P[a, b] = acc
    return P


def chunk_backward(q, k, v, g, dO, S0, dSf, C):
    """One (batch, head): returns dq, dk, dv, dg, dstate0 by the chunk form."""
    T, dk = q.shape
    dv = v.shape[1]
    bounds = [(c0, min(c0 + C, T)) for c0 in range(0, T, C)]
    # forward over chunks: incoming state of each chunk
    S_in = []
    S = S0.copy()
    for c0, c1 in bounds:
        S_in.append(S)
        n = c1 - c0
        P = range_products(g[c0:c1])
        S = P[0, n - 1][:, None] * S
        for s in range(n):
            S = S + np.outer(k[c0 + s] * P[s + 1, n - 1], v[c0 + s])
    dq, dkk, dvv, dg = (np.zeros((T, dk)), np.zeros((T, dk)), np.zeros((T, dv)), np.zeros((T, dk)))
    dS_out = np.zeros((dk, dv)) if dSf is None else dSf.copy()
    for ci in range(len(bounds) - 1, -1, -1):
        c0, c1 = bounds[ci]
        n = c1 - c0
        P = range_products(g[c0:c1])
        Sin = S_in[ci]
        qc, kc, vc, oc = q[c0:c1], k[c0:c1], v[c0:c1], dO[c0:c1]
        for t in range(n):
            acc = (Sin @ oc[t]) * P[0, t]
            for s in range(t + 1):
                acc = acc + (oc[t] @ vc[s]) * kc[s] * P[s + 1, t]
            dq[c0 + t] = acc
        for s in range(n):
            ak = (dS_out @ vc[s]) * P[s + 1, n - 1]
            av = (kc[s] * P[s + 1, n - 1]) @ dS_out
            for t in range(s, n):
                ak = ak + (oc[t] @ vc[s]) * qc[t] * P[s + 1, t]
                av = av + ((qc[t] * P[s + 1, t]) @ kc[s]) * oc[t]
            dkk[c0 + s], dvv[c0 + s] = ak, av
        for t in range(n):
            # D_t . S_{t-1}, term by term
            term_BE = P[t + 1, n - 1] * P[0, t - 1] * np.sum(dS_out * Sin, axis=1) if t > 0 else \
                P[t + 1, n - 1] * np.sum(dS_out * Sin, axis=1)
            term_BF = np.zeros(dk)
            for s in range(t):
                term_BF = term_BF + P[t + 1, n - 1] * P[s + 1, t - 1] * kc[s] * (dS_out @ vc[s])
            term_AE = np.zeros(dk)
            term_AF = np.zeros(dk)
            for r in range(t, n):
                pre = P[0, t - 1] if t > 0 else np.ones(dk)
                term_AE = term_AE + pre * P[t + 1, r] * qc[r] * (Sin @ oc[r])
                for s in range(t):
                    term_AF = term_AF + P[t + 1, r] * P[s + 1, t - 1] * qc[r] * kc[s] * (oc[r] @ vc[s])
            dg[c0 + t] = term_BE + term_BF + term_AE + term_AF
        dS_in = P[0, n - 1][:, None] * dS_out
        for r in range(n):
            dS_in = dS_in + np.outer(qc[r] * P[0, r], oc[r])
        dS_out = dS_in
    return dq, dkk, dvv, dg, dS_out


def _inputs(seed, B, H, T, dk, dv):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, dk)).astype(np.float32)
    k = rng.standard_normal((B, H, T, dk)).astype(np.float32)
    v = rng.standard_normal((B, H, T, dv)).astype(np.float32)
    g = rng.uniform(0.3, 1.0, (B, H, T, dk)).astype(np.float32)
    g[rng.random((B, H, T, dk)) < 0.05] = 0.0   # state resets on some channels
    g[rng.random((B, H, T, dk)) < 0.05] = 1.0   # no decay on others
    dO = rng.standard_normal((B, H, T, dv)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dk, dv))
    dSf = rng.standard_normal((B, H, dk, dv)).astype(np.float32)
    return q, k, v, g, dO, S0, dSf


@pytest.mark.parametrize("T,C,final", [(37, 8, True), (16, 16, False), (5, 8, True), (24, 1, True)])
def test_oracle_backward_equals_chunk_form(T, C, final):
    B, H, dk, dv = 1, 2, 5, 3
    q, k, v, g, dO, S0, dSf = _inputs(T + C, B, H, T, dk, dv)
    ref = oracle.gla_backward(q, k, v, g, dO, state0=S0, dS_final=dSf if final else None)
    for b in range(B):
        for h in range(H):
            got = chunk_backward(q[b, h].astype(np.float64), k[b, h].astype(np.float64),
                                 v[b, h].astype(np.float64), g[b, h].astype(np.float64),
                                 dO[b, h].astype(np.float64), S0[b, h],
                                 dSf[b, h].astype(np.float64) if final else None, C)
            for name, a, r in zip(("dq", "dk", "dv", "dg", "dstate0"), got, ref):
                np.testing.assert_allclose(a, r[b, h], rtol=1e-9, atol=1e-9, err_msg=name)


def test_query_key_term_of_the_gate_gradient_by_recurrence():
    """The fourth term of dg_t, sum over s < t <= r of P(t+1, r) P(s+1, t-1) q_r k_s (dO_r . v_s),
    computed as a kernel would: K_{t+1}[r] = g_t K_t[r] + (dO_r . v_t) k_t over the chunk, then
    sum_{r>=t} P(t+1, r) q_r K_t[r]. It equals the direct double sum, gates of 0 included."""
    rng = np.random.default_rng(7)
    C, dk, dv = 12, 4, 3
    q, k = rng.standard_normal((C, dk)), rng.standard_normal((C, dk))
    v, dO = rng.standard_normal((C, dv)), rng.standard_normal((C, dv))
    g = rng.uniform(0.2, 1.0, (C, dk))
    g[3, 1] = g[7, 2] = 0.0
    P = range_products(g)
    A2 = dO @ v.T  # A2[r, s] = dO_r . v_s
    direct = np.zeros((C, dk))
    for t in range(C):
        for r in range(t, C):
            for s in range(t):
                direct[t] += P[t + 1, r] * P[s + 1, t - 1] * q[r] * k[s] * A2[r, s]
    K = np.zeros((C, dk))  # K_t[r], t = 0: empty sum
    rec = np.zeros((C, dk))
    for t in range(C):
        for r in range(t, C):
            rec[t] += P[t + 1, r] * q[r] * K[r]
        K = g[t] * K + A2[:, t:t + 1] * k[t]
    np.testing.assert_allclose(rec, direct, rtol=1e-12, atol=1e-12)
