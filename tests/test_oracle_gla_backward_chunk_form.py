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


def chunk_backward_products(q, k, v, g, dO, S0, dSf, C, fast_min=2.0 ** -60):
    """The chunk backward in the shape a tensor-core kernel computes it, for one (batch, head):
    per chunk, matrix products with the prefix products G (fast route: q~ = q.G, k~ = k/G,
    k^ = k.(a/G)) when every channel's chunk decay a is at least fast_min, else range products
    (exact route); the gate gradient from two decayed scans and the query-key recurrence.
    Returns dq, dk, dv, dg, dstate0 and the number of chunks that took the exact route."""
    T, dk = q.shape
    bounds = [(c0, min(c0 + C, T)) for c0 in range(0, T, C)]
    S_in, S = [], S0.copy()
    for c0, c1 in bounds:  # forward: incoming states
        S_in.append(S)
        G = np.cumprod(g[c0:c1], axis=0)
        P = range_products(g[c0:c1])
        n = c1 - c0
        S = G[-1][:, None] * S + (k[c0:c1] * P[1:n + 1, n - 1]).T @ v[c0:c1]
    out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(q)]
    dq, dkk, dvv, dg = out
    dS_out = np.zeros((dk, v.shape[1])) if dSf is None else dSf.copy()
    exact_chunks = 0
    for ci in range(len(bounds) - 1, -1, -1):
        c0, c1 = bounds[ci]
        n = c1 - c0
        qc, kc, vc, oc, gc = q[c0:c1], k[c0:c1], v[c0:c1], dO[c0:c1], g[c0:c1]
        Sin = S_in[ci]
        G = np.cumprod(gc, axis=0)
        a = G[-1]
        A2 = oc @ vc.T                                   # A2[t, s] = dO_t . v_s
        M = np.tril(np.ones((n, n)))
        if a.min() >= fast_min:
            qt, kt, kh = qc * G, kc / G, kc * (a / G)
            dq[c0:c1] = (oc @ Sin.T + (M * A2) @ kt) * G
            dkk[c0:c1] = ((M * A2).T @ qt) / G + (vc @ dS_out.T) * (a / G)
            dvv[c0:c1] = (M * (qt @ kt.T)).T @ oc + kh @ dS_out
            F = a / G                                    # P(t+1, n-1)
        else:
            exact_chunks += 1
            P = range_products(gc)
            for t in range(n):
                dq[c0 + t] = (Sin @ oc[t]) * P[0, t] + sum(A2[t, s] * kc[s] * P[s + 1, t] for s in range(t + 1))
            for s in range(n):
                dkk[c0 + s] = (dS_out @ vc[s]) * P[s + 1, n - 1] + sum(
                    A2[t, s] * qc[t] * P[s + 1, t] for t in range(s, n))
                dvv[c0 + s] = (kc[s] * P[s + 1, n - 1]) @ dS_out + sum(
                    ((qc[t] * P[s + 1, t]) @ kc[s]) * oc[t] for t in range(s, n))
            F = P[1:n + 1, n - 1]
        Gprev = np.vstack([np.ones((1, dk)), G[:-1]])    # P(0, t-1)
        # the four terms of dg_t = sum_j D_t[:, j] S_{t-1}[:, j]
        BE = F * Gprev * np.sum(dS_out * Sin, axis=1)
        Y, X = kc * (vc @ dS_out.T), qc * (oc @ Sin.T)
        Z, BF = np.zeros(dk), np.zeros((n, dk))
        for t in range(n):                               # Z_t = sum_{s<t} P(s+1, t-1) Y_s
            BF[t] = F[t] * Z
            Z = gc[t] * Z + Y[t]
        W, AE = np.zeros(dk), np.zeros((n, dk))
        for t in range(n - 1, -1, -1):                   # W_t = sum_{r>=t} P(t+1, r) X_r
            W = X[t] + (gc[t + 1] * W if t + 1 < n else 0.0)
            AE[t] = Gprev[t] * W
        K, AF = np.zeros((n, dk)), np.zeros((n, dk))
        for t in range(n):                               # K_t[r] = sum_{s<t} P(s+1, t-1) A2[r, s] k_s
            acc, dec = np.zeros(dk), np.ones(dk)
            for r in range(t, n):                        # sum_{r>=t} P(t+1, r) q_r K_t[r]
                if r > t:
                    dec = dec * gc[r]
                acc = acc + dec * qc[r] * K[r]
            AF[t] = acc
            K = gc[t] * K + A2[:, t:t + 1] * kc[t]
        dg[c0:c1] = BE + BF + AE + AF
        dS_out = a[:, None] * dS_out + (qc * G).T @ oc
    return dq, dkk, dvv, dg, dS_out, exact_chunks


@pytest.mark.parametrize("gates,T,C", [("slow", 70, 16), ("resets", 70, 16), ("slow", 9, 16)])
def test_product_shaped_chunk_backward_equals_oracle(gates, T, C):
    """Both routes of the product-shaped chunk backward against the oracle: gates in [0.9, 1]
    keep every chunk on the fast route, gates with zeros send chunks to the exact route."""
    rng = np.random.default_rng(11 + T)
    B, H, dk, dv = 1, 1, 6, 4
    q = rng.standard_normal((B, H, T, dk)).astype(np.float32)
    k = rng.standard_normal((B, H, T, dk)).astype(np.float32)
    v = rng.standard_normal((B, H, T, dv)).astype(np.float32)
    g = rng.uniform(0.9, 1.0, (B, H, T, dk)).astype(np.float32)
    if gates == "resets":
        g[0, 0, 5, 2] = g[0, 0, 40, 0] = 0.0
    dO = rng.standard_normal((B, H, T, dv)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dk, dv))
    dSf = rng.standard_normal((B, H, dk, dv)).astype(np.float32)
    ref = oracle.gla_backward(q, k, v, g, dO, state0=S0, dS_final=dSf)
    *got, exact = chunk_backward_products(*(x[0, 0].astype(np.float64) for x in (q, k, v, g, dO)),
                                         S0[0, 0], dSf[0, 0].astype(np.float64), C)
    assert (exact > 0) == (gates == "resets")
    for name, a, r in zip(("dq", "dk", "dv", "dg", "dstate0"), got, ref):
        np.testing.assert_allclose(a, r[0, 0], rtol=1e-8, atol=1e-8, err_msg=name)
