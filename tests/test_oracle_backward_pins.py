"""Pins of the read-path backward oracle (oracle/backward.py) against things it does not
compute itself:

  * central finite differences of L = sum_t <dL/do_t, o_t>, where o_t comes from the
    pinned forward oracle (oracle.chunk) with the slot lists held fixed (forced mode), with
    respect to every entry of q, g and v on tiny memories;
  * special cases: g = 0 (no gradient to q; dv = dL/do; dg = <dL/do, vhat - v>), k = 1 (the
    single weight is 1 whatever q is, so dq = 0), dL/do = 0 (all gradients 0).
"""
import numpy as np
import pytest

import oracle
from oracle.backward import read_backward


def _case(seed, n=6, h=3, dv=4, k=3, L=4):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(L, 2 * h))
    v = rng.normal(size=(L, dv))
    g = rng.uniform(0.1, 0.9, size=L)
    K1 = rng.normal(size=(n, h))
    K2 = rng.normal(size=(n, h))
    V = rng.normal(size=(n * n, dv))
    d_o = rng.normal(size=(L, dv))
    return q, v, g, K1, K2, V, d_o


def _slots(cfg, q, K1, K2):
    """The forward oracle's own selection (so the forced slots are the top-k ones)."""
    h = cfg.h
    I = []
    for t in range(q.shape[0]):
        D1 = oracle.subkey_dist(cfg, q[t, :h], K1.astype(np.float32))
        D2 = oracle.subkey_dist(cfg, q[t, h:], K2.astype(np.float32))
        I_t, _, _ = oracle.select(cfg, D1, D2)
        I.append(I_t)
    return np.array(I, dtype=np.int32)


def _loss(cfg, q, v, g, K1, K2, V, I, d_o):
    """sum_t <d_o_t, o_t> with o from the forward oracle, slots fixed to I (the write that
    follows the read inside the call does not change o)."""
    L = q.shape[0]
    o, _, _ = oracle.chunk(cfg, q, v, g, None, K1.astype(np.float32).copy(), K2.astype(np.float32).copy(),
                           V.astype(np.float32).copy(), forced=I, force_mask=np.ones(L, np.int32))
    return float(np.sum(d_o * o))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_finite_differences(seed):
    q, v, g, K1, K2, V, d_o = _case(seed)
    n, h, dv, k, L = 6, 3, 4, 3, q.shape[0]
    # the forward oracle stores K and V as fp32: give the backward the same values
    K1, K2, V = (x.astype(np.float32).astype(np.float64) for x in (K1, K2, V))
    cfg = oracle.make_cfg(n, 2 * h, dv, k, L)
    I = _slots(cfg, q, K1, K2)
    dq, dv_, dg = read_backward(n, cfg.eps_idw, q, v, g, K1, K2, V, I, d_o)
    eps = 1e-6

    def fd(arr, idx):
        x0 = arr[idx]
        arr[idx] = x0 + eps
        lp = _loss(cfg, q, v, g, K1, K2, V, I, d_o)
        arr[idx] = x0 - eps
        lm = _loss(cfg, q, v, g, K1, K2, V, I, d_o)
        arr[idx] = x0
        return (lp - lm) / (2 * eps)

    for idx in np.ndindex(q.shape):
        num = fd(q, idx)
        assert abs(num - dq[idx]) <= 1e-6 * max(1.0, abs(num)), f"dq{idx}: {dq[idx]} vs {num}"
    for t in range(L):
        num = fd(g, t)
        assert abs(num - dg[t]) <= 1e-6 * max(1.0, abs(num)), f"dg[{t}]: {dg[t]} vs {num}"
    for idx in np.ndindex(v.shape):
        num = fd(v, idx)
        assert abs(num - dv_[idx]) <= 1e-6 * max(1.0, abs(num)), f"dv{idx}: {dv_[idx]} vs {num}"


def test_gate_zero_passes_nothing_to_the_query():
    q, v, g, K1, K2, V, d_o = _case(3)
    g[:] = 0.0
    cfg = oracle.make_cfg(6, 6, 4, 3, 4)
    I = _slots(cfg, q, K1, K2)
    dq, dv_, dg = read_backward(6, cfg.eps_idw, q, v, g, K1, K2, V, I, d_o)
    assert np.all(dq == 0.0)
    assert np.array_equal(dv_, d_o)
    o_read = np.array([np.dot(_weights(cfg, q[t], K1, K2, I[t]), V[I[t]]) for t in range(q.shape[0])])
    assert np.allclose(dg, np.sum(d_o * (o_read - v), axis=1), rtol=1e-12, atol=1e-12)


def _weights(cfg, qt, K1, K2, It):
    h, n = cfg.h, cfg.n
    S = np.array([-np.log(cfg.eps_idw + np.sum((qt[:h] - K1[i // n]) ** 2))
                  - np.log(cfg.eps_idw + np.sum((qt[h:] - K2[i % n]) ** 2)) for i in It])
    e = np.exp(S - S.max())
    return e / e.sum()


def test_single_slot_has_no_query_gradient():
    q, v, g, K1, K2, V, d_o = _case(4)
    cfg = oracle.make_cfg(6, 6, 4, 1, 4)
    I = _slots(cfg, q, K1, K2)
    dq, dv_, dg = read_backward(6, cfg.eps_idw, q, v, g, K1, K2, V, I, d_o)
    assert np.all(np.abs(dq) <= 1e-15)
    assert np.allclose(dg, np.sum(d_o * (V[I[:, 0]] - v), axis=1), rtol=1e-12, atol=1e-12)


def test_zero_upstream_gradient():
    q, v, g, K1, K2, V, d_o = _case(5)
    cfg = oracle.make_cfg(6, 6, 4, 3, 4)
    I = _slots(cfg, q, K1, K2)
    dq, dv_, dg = read_backward(6, cfg.eps_idw, q, v, g, K1, K2, V, I, np.zeros_like(d_o))
    assert not dq.any() and not dv_.any() and not dg.any()
