"""Pins of the oracle of heads that share one value table (oracle.chunk_heads).

Readings (fwpkm_oracle.c, orc_chunk_heads; "Fast-weight Product Key Memory"
(paperlayer summary) §D.1, §D.3): each head has its own codebooks and query and selects
its own slots; the read is the mean of the heads' reads; the write is the gradient of
1/2 sum_t g_t ||tau_t - vhat_t||^2 on the shared rows, averaged over the tokens that read
a row; each head's codebooks take their own addressing step.  Pinned against: the
one-head oracle (H = 1, and H identical heads), finite differences of the loss, the
one-head key step of every head, and two hand-worked examples (tests/golden).
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(seed, H, n=8, h=4, dv=6, k=3, C=5, T=5):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(H, T, 2 * h))
    v = rng.normal(size=(T, dv))
    g = rng.uniform(0.1, 1.0, size=T)
    K1 = rng.normal(size=(H, n, h)).astype(np.float32)
    K2 = rng.normal(size=(H, n, h)).astype(np.float32)
    V = (0.3 * rng.normal(size=(n * n, dv))).astype(np.float32)
    return q, v, g, K1, K2, V


@pytest.mark.parametrize("key_update", [False, True])
def test_one_head_is_the_single_memory_chunk(key_update):
    q, v, g, K1, K2, V = _case(1, 1)
    vn = np.ones(6)
    cfg = oracle.make_cfg(8, 8, 6, 3, 5, key_update=key_update, lr_key=10.0)
    a1, a2, av = K1.copy(), K2.copy(), V.copy()
    o_h, I_h, w_h = oracle.chunk_heads(cfg, q, v, g, vn, a1, a2, av)
    b1, b2, bv = K1[0].copy(), K2[0].copy(), V.copy()
    o_s, I_s, w_s = oracle.chunk(cfg, q[0], v, g, vn, b1, b2, bv)
    assert np.array_equal(o_h, o_s) and np.array_equal(I_h[0], I_s) and np.array_equal(w_h[0], w_s)
    assert np.array_equal(av, bv)
    assert np.array_equal(a1[0], b1) and np.array_equal(a2[0], b2)


@pytest.mark.parametrize("key_update", [False, True])
def test_identical_heads_are_one_head(key_update):
    """H copies of one head (same query, same codebooks) read, write and step like that
    head alone: the mean of equal reads is the read, the H halves of each weight add up
    to it, and a token that reads a row through every head counts once."""
    q, v, g, K1, K2, V = _case(2, 1)
    H = 3
    qH = np.repeat(q, H, axis=0)
    K1H, K2H = np.repeat(K1, H, axis=0), np.repeat(K2, H, axis=0)
    cfg = oracle.make_cfg(8, 8, 6, 3, 5, key_update=key_update, lr_key=10.0)
    vn = np.full(6, 0.5)
    VH = V.copy()
    o_h, I_h, _ = oracle.chunk_heads(cfg, qH, v, g, vn, K1H, K2H, VH)
    b1, b2, bv = K1[0].copy(), K2[0].copy(), V.copy()
    o_s, I_s, _ = oracle.chunk(cfg, q[0], v, g, vn, b1, b2, bv)
    assert all(np.array_equal(I_h[i], I_s) for i in range(H))
    np.testing.assert_allclose(o_h, o_s, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(VH, bv, rtol=1e-6, atol=1e-7)  # fp32 storage of fp64 results
    for i in range(H):
        assert np.array_equal(K1H[i], b1) and np.array_equal(K2H[i], b2)


def test_each_head_takes_its_own_key_step():
    q, v, g, K1, K2, V = _case(3, 2)
    cfg = oracle.make_cfg(8, 8, 6, 3, 5, key_update=True, lr_key=10.0)
    a1, a2 = K1.copy(), K2.copy()
    oracle.chunk_heads(cfg, q, v, g, None, a1, a2, V.copy())
    for hd in range(2):
        b1, b2 = K1[hd].copy(), K2[hd].copy()
        oracle.chunk(cfg, q[hd], v, g, None, b1, b2, V.copy())
        assert np.array_equal(a1[hd], b1) and np.array_equal(a2[hd], b2), f"head {hd}"


def _loss(Vf, I, w, g, tau, pair, H):
    """1/2 sum_t g_t ||tau_t - vhat_t||^2, vhat_t = (1/H) sum_h sum_r w V[I] (fp64)."""
    L = 0.0
    for t in range(len(g)):
        if not pair[t]:
            continue
        vh = sum(w[hd, t, r] * Vf[I[hd, t, r]] for hd in range(H) for r in range(I.shape[2])) / H
        L += 0.5 * g[t] * np.sum((tau[t] - vh) ** 2)
    return L


@pytest.mark.parametrize("seed", [4, 5])
def test_value_step_is_the_token_averaged_gradient(seed):
    """V_i moves by -G_i / N_i with G_i = dL_mem/dV_i (central differences with the slot
    lists and weights held fixed: they do not depend on V) and N_i the number of pair
    tokens that read row i through any head."""
    H, n, dv = 2, 4, 3
    q, v, g, K1, K2, V = _case(seed, H, n=n, h=2, dv=dv, k=3, C=6, T=6)
    cfg = oracle.make_cfg(n, 4, dv, 3, 6, target_norm=False)
    V0 = V.astype(np.float64)
    V1 = V.copy()
    o, I, w = oracle.chunk_heads(cfg, q, v, g, None, K1.copy(), K2.copy(), V1)
    T = len(g)
    pair = np.array([t + 1 < T for t in range(T)])
    tau = np.zeros_like(v)
    tau[:-1] = v[1:]
    eps = 1e-6
    for i in range(n * n):
        toks = {t for t in range(T) if pair[t] and any(i in I[hd, t] for hd in range(H))}
        if not toks:
            assert np.array_equal(V1[i], V[i])
            continue
        grad = np.zeros(dv)
        for e in range(dv):
            Vp, Vm = V0.copy(), V0.copy()
            Vp[i, e] += eps
            Vm[i, e] -= eps
            grad[e] = (_loss(Vp, I, w, g, tau, pair, H) - _loss(Vm, I, w, g, tau, pair, H)) / (2 * eps)
        step = V0[i] - V1[i].astype(np.float64)
        np.testing.assert_allclose(step, grad / len(toks), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("case", ["two_slots", "same_slot"])
def test_golden_heads_shared_v(case):
    with open(os.path.join(GOLDEN, "heads_shared_v.json")) as f:
        j = json.load(f)
    c = j["cfg"]
    cfg = oracle.make_cfg(c["n"], c["d"], c["d_v"], c["k"], c["chunk"], target_norm=c["target_norm"],
                          lookahead=c["lookahead"], gate_weight=c["gate_weight"])
    cs = j["cases"][case]
    K1 = np.array(j["K1"], np.float32)
    K2 = np.array(j["K2"], np.float32)
    V = np.array(j["V"], np.float32)
    o, I, w = oracle.chunk_heads(cfg, np.array(cs["q"]), np.array(j["v"]), np.array(j["g"]), None, K1, K2, V)
    np.testing.assert_array_equal(o[0], cs["o0"])
    np.testing.assert_array_equal(V, np.array(cs["V_after"], np.float32))


def test_sequence_of_heads_is_chunk_after_chunk():
    q, v, g, K1, K2, V = _case(6, 2, T=13, C=5)
    cfg = oracle.make_cfg(8, 8, 6, 3, 5, key_update=True, lr_key=5.0)
    a1, a2, av = K1.copy(), K2.copy(), V.copy()
    o_s, _, _ = oracle.run_sequence_heads(cfg, q, v, g, a1, a2, av, n_iter=1)
    b1, b2, bv = K1.copy(), K2.copy(), V.copy()
    for t0 in range(0, 13, 5):
        t1 = min(13, t0 + 5)
        o_c, _, _ = oracle.chunk_heads(cfg, q[:, t0:t1], v[t0:t1], g[t0:t1], v[t1] if t1 < 13 else None, b1, b2, bv)
        assert np.array_equal(o_c, o_s[t0:t1])
    assert np.array_equal(av, bv) and np.array_equal(a1, b1)
