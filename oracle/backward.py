"""CPU oracle of the read path's backward (the gradient that reaches the slow weights).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  Plain fp64 numpy, loops over
tokens and ranks in the order below.

What it computes ("Fast-weight Product Key Memory" (paperlayer summary) §2 / Figure 1: slow
weights learn during training, the fast key/value parameters online; §3.1, §3.2: the
slow-weight projections supply q, v and g, and the read is
    D_j[a] = ||q_j - K_j[a]||^2,  sigma_j[a] = -log(eps + D_j[a]),
    S_i = sigma_1[a] + sigma_2[b]  (slot i = a n + b),  s' = softmax(S over I_t),
    vhat_t = sum_i s'_i V_i,  o_t = g_t vhat_t + (1 - g_t) v_t):
the gradient of a loss L with dL/do_t given, with respect to q_t, v_t and g_t.

Readings (the pages describe no backward of the memory into the slow weights):
  * the fast weights V, K1, K2 as they were at the chunk's read are constants of this
    backward: they learn only from their own chunk-local losses (§3.1), and no gradient is
    passed through their updates into earlier tokens;
  * the discrete selection I_t passes no gradient: q reaches L through the selected slots'
    scores and the softmax only.

Then, per token t with slots I_t (rank order) and a_r = I_t[r] // n, b_r = I_t[r] % n:
    dg_t  = <dL/do_t, vhat_t - v_t>
    dv_t  = (1 - g_t) dL/do_t
    ds_r  = <g_t dL/do_t, V_{I_t[r]}>
    dS_r  = s'_r (ds_r - sum_r' s'_r' ds_r')
    dq_1  = sum_r dS_r * (-1 / (eps + D_1[a_r])) * 2 (q_1 - K_1[a_r])
    dq_2  = sum_r dS_r * (-1 / (eps + D_2[b_r])) * 2 (q_2 - K_2[b_r])
(dq of half 1 is the first h entries of dq_t.)
"""
from __future__ import annotations

import numpy as np


def read_backward(n: int, eps_idw: float, q, v, g, K1, K2, V, I, d_o):
    """q [len][d], v [len][d_v], g [len], K1, K2 [n][h], V [n*n][d_v], I [len][k] int slots in
    rank order, d_o [len][d_v]  ->  (dq [len][d], dv [len][d_v], dg [len]), all fp64."""
    q = np.asarray(q, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    K1 = np.asarray(K1, dtype=np.float64)
    K2 = np.asarray(K2, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    d_o = np.asarray(d_o, dtype=np.float64)
    I = np.asarray(I, dtype=np.int64)
    L, d = q.shape
    h = d // 2
    k = I.shape[1]
    dq = np.zeros((L, d))
    dv = np.zeros_like(v)
    dg = np.zeros(L)
    for t in range(L):
        q1, q2 = q[t, :h], q[t, h:]
        a = I[t] // n
        b = I[t] % n
        D1 = np.array([np.sum((q1 - K1[a[r]]) ** 2) for r in range(k)])
        D2 = np.array([np.sum((q2 - K2[b[r]]) ** 2) for r in range(k)])
        S = -np.log(eps_idw + D1) - np.log(eps_idw + D2)
        e = np.exp(S - S.max())
        s = e / e.sum()
        rows = V[I[t]]                      # [k][d_v]
        vhat = s @ rows
        dg[t] = float(np.dot(d_o[t], vhat - v[t]))
        dv[t] = (1.0 - g[t]) * d_o[t]
        dvhat = g[t] * d_o[t]
        ds = rows @ dvhat                   # [k]
        dS = s * (ds - np.dot(s, ds))
        for r in range(k):
            dq[t, :h] += dS[r] * (-1.0 / (eps_idw + D1[r])) * 2.0 * (q1 - K1[a[r]])
            dq[t, h:] += dS[r] * (-1.0 / (eps_idw + D2[r])) * 2.0 * (q2 - K2[b[r]])
    return dq, dv, dg
