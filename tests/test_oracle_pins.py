"""Pins of the CPU oracle against facts the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a library routine
(scipy distances / softmax / entropy), exhaustive search, finite differences of the
losses the pages define, hand-worked examples (tests/golden), or invariants
(causality, pass composition, z-score moments, gate limits).
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.spatial.distance import cdist
from scipy.special import softmax
from scipy.stats import entropy

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _cfg_from(j, **over):
    c = dict(j["cfg"])
    c.update(over)
    return oracle.make_cfg(n=c["n"], d=c["d"], d_v=c["d_v"], k=c["k"], chunk=c.get("chunk", 64),
                           eps_idw=c.get("eps_idw", 1e-3), eps_norm=c.get("eps_norm", 1e-5),
                           lr_key=c.get("lr_key", 1.0), key_update=c.get("key_update", False),
                           target_norm=c.get("target_norm", True), lookahead=c.get("lookahead", True),
                           gate_weight=c.get("gate_weight", True))


# --------------------------------------------------------------------------- step 1
def test_distance_matches_scipy_sqeuclidean():
    rng = np.random.default_rng(1)
    cfg = oracle.make_cfg(n=37, d=10, d_v=4, k=3, chunk=8)
    K = rng.standard_normal((37, 5)).astype(np.float32)
    q = rng.standard_normal(5)
    D = oracle.subkey_dist(cfg, q, K)
    ref = cdist(q[None, :], K.astype(np.float64), "sqeuclidean")[0]
    np.testing.assert_allclose(D, ref, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------- steps 2-4
def _exhaustive_topk(D1, D2, k, eps):
    """Top-k over ALL n*n slots of sigma1[a] + sigma2[b], ordered (score desc, slot asc)."""
    n = D1.shape[0]
    libm_log = np.vectorize(math.log)  # same libm as the C oracle, so scores agree to the bit
    s1 = -libm_log(eps + D1)
    s2 = -libm_log(eps + D2)
    S = (s1[:, None] + s2[None, :]).reshape(-1)
    slots = np.arange(n * n)
    order = np.lexsort((slots, -S))
    return order[:k].astype(np.int32), S[order[:k]]


@pytest.mark.parametrize("n", [4, 8, 16])
@pytest.mark.parametrize("k", [1, 2, 4, 8])
def test_product_key_topk_equals_exhaustive(n, k):
    if k > n:
        pytest.skip("k > n")
    rng = np.random.default_rng(100 * n + k)
    h = 3
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=2, k=k, chunk=4)
    for trial in range(40):
        K1 = rng.standard_normal((n, h)).astype(np.float32)
        K2 = rng.standard_normal((n, h)).astype(np.float32)
        if trial % 4 == 3:  # exact ties: duplicated sub-keys
            K1[n // 2] = K1[0]
            K2[n - 1] = K2[1]
        q = rng.standard_normal(2 * h)
        if trial % 8 == 7:  # a query exactly between two keys
            q[:h] = 0.5 * (K1[0].astype(np.float64) + K1[1].astype(np.float64))
        D1 = cdist(q[None, :h], K1.astype(np.float64), "sqeuclidean")[0]
        D2 = cdist(q[None, h:], K2.astype(np.float64), "sqeuclidean")[0]
        I, S, w = oracle.select(cfg, D1, D2)
        I_ref, S_ref = _exhaustive_topk(D1, D2, k, cfg.eps_idw)
        np.testing.assert_array_equal(I, I_ref)
        np.testing.assert_array_equal(S, S_ref)
        if k == 1:
            assert I[0] == np.argmin(D1) * n + np.argmin(D2)


def test_softmax_weights_closed_form():
    """s'_i = prod_j (eps + D_j)^-1 / sum over the selected slots (IDW with power 2)."""
    rng = np.random.default_rng(7)
    n, h, k = 16, 4, 8
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=2, k=k, chunk=4)
    K1 = rng.standard_normal((n, h)).astype(np.float32)
    K2 = rng.standard_normal((n, h)).astype(np.float32)
    q = rng.standard_normal(2 * h)
    D1 = oracle.subkey_dist(cfg, q[:h], K1)
    D2 = oracle.subkey_dist(cfg, q[h:], K2)
    I, S, w = oracle.select(cfg, D1, D2)
    a, b = I // n, I % n
    inv = 1.0 / ((cfg.eps_idw + D1[a]) * (cfg.eps_idw + D2[b]))
    np.testing.assert_allclose(w, inv / inv.sum(), rtol=1e-13)
    assert abs(w.sum() - 1.0) < 1e-14
    assert np.all(np.diff(w) <= 1e-15)  # rank order = descending weight


def test_forced_selection_uses_given_slots():
    rng = np.random.default_rng(9)
    n, h, k = 8, 2, 3
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=2, k=k, chunk=4)
    D1 = rng.uniform(0.5, 3, n)
    D2 = rng.uniform(0.5, 3, n)
    forced = np.array([5, 17, 60], np.int32)
    I, S, w = oracle.select(cfg, D1, D2, forced=forced)
    np.testing.assert_array_equal(I, forced)
    ref = -np.log(cfg.eps_idw + D1[forced // n]) - np.log(cfg.eps_idw + D2[forced % n])
    np.testing.assert_allclose(w, softmax(ref), rtol=1e-13)


# --------------------------------------------------------------------------- golden examples
def test_golden_k2_shared_slot():
    j = _load("write_k2_shared_slot.json")
    cfg = _cfg_from(j)
    K1 = np.array(j["K1"], np.float32); K2 = np.array(j["K2"], np.float32)
    V = np.array(j["V"], np.float32)
    o, I, w = oracle.chunk(cfg, np.array(j["q"]), np.array(j["v"]), np.array(j["g"]), None, K1, K2, V)
    np.testing.assert_array_equal(I, np.array(j["expect_I"]))
    np.testing.assert_allclose(w, np.array(j["expect_w"]), rtol=1e-14)
    np.testing.assert_allclose(o, np.array(j["expect_o"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(V, np.array(j["expect_V"]), rtol=1e-7)


@pytest.mark.parametrize("case", ["rewrite", "collide2", "collide3"])
def test_golden_collisions_k1(case):
    j = _load("write_collisions_k1.json")
    c = j["cases"][case]
    cfg = _cfg_from(j, chunk=len(c["g"]))
    K1 = np.array(j["K1"], np.float32); K2 = np.array(j["K2"], np.float32)
    V = np.zeros((4, 4), np.float32)
    V[0] = c["V0"]
    V[3] = [7, 7, 7, 7]
    T = len(c["g"])
    q = np.tile(np.array(j["q_all"]), (T, 1))
    o, I, w = oracle.chunk(cfg, q, np.array(c["v"], float), np.array(c["g"]), None, K1, K2, V)
    assert np.all(I == 0) and np.all(w == 1.0)
    np.testing.assert_allclose(V[0], c["expect_V0"], rtol=1e-7, atol=1e-7)
    np.testing.assert_array_equal(V[3], [7, 7, 7, 7])
    np.testing.assert_array_equal(V[1:3], 0)


def test_golden_address_n2():
    j = _load("address_n2.json")
    cfg = _cfg_from(j)
    K1 = np.array(j["K1"], np.float32); K2 = np.array(j["K2"], np.float32)
    V = np.full((4, 2), 3.0, np.float32)
    oracle.chunk(cfg, np.array(j["q"]), np.zeros((1, 2)), np.ones(1), None, K1, K2, V)
    np.testing.assert_allclose(K1, np.array(j["expect_K1"]), rtol=1e-7)
    np.testing.assert_array_equal(K2, np.array(j["expect_K2"], np.float32))
    np.testing.assert_array_equal(V, 3.0)


# --------------------------------------------------------------------------- finite differences
def _mem_loss(V, I, w, g, targets, pair):
    """1/2 sum_t g_t ||target_t - sum_r w_tr V[I_tr]||^2 over pair tokens (the pages' L_mem)."""
    L = 0.0
    for t in range(I.shape[0]):
        if not pair[t]:
            continue
        vhat = (w[t][:, None] * V[I[t]]).sum(0)
        L += 0.5 * g[t] * np.sum((targets[t] - vhat) ** 2)
    return L


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_value_step_is_read_count_averaged_gradient(seed):
    """-dV_i * N_read,i equals dL_mem/dV_i by central differences (L_mem is quadratic in V)."""
    rng = np.random.default_rng(seed)
    n, h, dv, k, T = 4, 2, 3, 3, 6
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=dv, k=k, chunk=T, target_norm=False)
    K1 = rng.standard_normal((n, h)).astype(np.float32)
    K2 = rng.standard_normal((n, h)).astype(np.float32)
    V0 = rng.standard_normal((n * n, dv)).astype(np.float32)
    q = rng.standard_normal((T, 2 * h)); v = rng.standard_normal((T, dv)); g = rng.uniform(0.1, 1, T)
    V1 = V0.copy()
    o, I, w = oracle.chunk(cfg, q, v, g, None, K1.copy(), K2.copy(), V1)
    pair = np.arange(T) < T - 1
    targets = np.zeros((T, dv)); targets[:-1] = v[1:]
    counts = np.zeros(n * n, int)
    for t in range(T - 1):
        counts[I[t]] += 1
    assert counts.max() >= 2, "seed must produce a collision"
    Vd = V0.astype(np.float64)
    step = 1e-4
    for i in np.nonzero(counts)[0]:
        for e in range(dv):
            Vp = Vd.copy(); Vp[i, e] += step
            Vm = Vd.copy(); Vm[i, e] -= step
            fd = (_mem_loss(Vp, I, w, g, targets, pair) - _mem_loss(Vm, I, w, g, targets, pair)) / (2 * step)
            got = -(float(V1[i, e]) - float(V0[i, e])) * counts[i]
            assert abs(got - fd) <= 1e-6 + 1e-5 * abs(fd), (i, e, got, fd)
    untouched = counts == 0
    np.testing.assert_array_equal(V1[untouched], V0[untouched])


def _addr_loss(q, K1, K2, eps):
    """sum_j -H(pbar_j), pbar_j = mean_t softmax(-log(eps + ||q_j - K_j||^2))."""
    h = K1.shape[1]
    L = 0.0
    for j, K in enumerate((K1, K2)):
        D = cdist(q[:, j * h:(j + 1) * h], K, "sqeuclidean")
        P = softmax(-np.log(eps + D), axis=1)
        L -= entropy(P.mean(0))
    return L


@pytest.mark.parametrize("seed", [0, 3])
def test_key_step_is_entropy_gradient(seed):
    rng = np.random.default_rng(seed)
    n, h, T = 6, 3, 5
    q = rng.standard_normal((T, 2 * h))
    K1 = rng.standard_normal((n, h)).astype(np.float32)
    K2 = rng.standard_normal((n, h)).astype(np.float32)
    eps = 1e-3
    step = 1e-5
    fd = []
    for K in (K1, K2):
        G = np.zeros((n, h))
        for b in range(n):
            for e in range(h):
                Kp = [K1.astype(np.float64), K2.astype(np.float64)]
                Km = [K1.astype(np.float64), K2.astype(np.float64)]
                idx = 0 if K is K1 else 1
                Kp[idx][b, e] += step; Km[idx][b, e] -= step
                G[b, e] = (_addr_loss(q, *Kp, eps) - _addr_loss(q, *Km, eps)) / (2 * step)
        fd.append(G)
    lr = 1.0 / max(np.abs(fd[0]).max(), np.abs(fd[1]).max())
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=2, k=2, chunk=T, eps_idw=eps, lr_key=lr, key_update=True)
    K1n, K2n = K1.copy(), K2.copy()
    oracle.chunk(cfg, q, rng.standard_normal((T, 2)), np.ones(T), None, K1n, K2n,
                 np.zeros((n * n, 2), np.float32))
    for K0, K1_, G in ((K1, K1n, fd[0]), (K2, K2n, fd[1])):
        got = -(K1_.astype(np.float64) - K0.astype(np.float64)) / lr
        np.testing.assert_allclose(got, G, rtol=2e-5, atol=2e-6 * np.abs(G).max())


@pytest.mark.parametrize("seed", [4, 5])
def test_key_step_factors_through_inverse_square_distances(seed):
    """The key gradient rebuilt from u = (eps + D)^-2, which does not depend on the usage
    marginals, and the small per-token factors 1/Z_t and L_t/Z_t:
    dL/dK[b] = (2/C) (lp[b] sum_t u q_t / Z_t - sum_t u L_t q_t / Z_t
                      - (lp[b] sum_t u / Z_t - sum_t u L_t / Z_t) K[b]),
    at a size the finite-difference check cannot afford (n = 64, C = 40)."""
    rng = np.random.default_rng(seed)
    n, h, C, eps, lr = 64, 16, 40, 1e-3, 3.0
    q = rng.standard_normal((C, 2 * h))
    K1 = rng.standard_normal((n, h)).astype(np.float32)
    K2 = rng.standard_normal((n, h)).astype(np.float32)
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=2, k=4, chunk=C, eps_idw=eps, lr_key=lr, key_update=True)
    K1n, K2n = K1.copy(), K2.copy()
    oracle.chunk(cfg, q, rng.standard_normal((C, 2)), np.ones(C), None, K1n, K2n,
                 np.zeros((n * n, 2), np.float32))
    for j, (K0, Kn) in enumerate(((K1, K1n), (K2, K2n))):
        K = K0.astype(np.float64)
        qj = q[:, j * h:(j + 1) * h]
        D = cdist(qj, K, "sqeuclidean")
        Z = (1.0 / (eps + D)).sum(axis=1)
        P = (1.0 / (eps + D)) / Z[:, None]
        lp = np.log(P.mean(axis=0))
        L = P @ lp
        u = (eps + D) ** -2
        A1 = u.T @ (qj / Z[:, None])
        A2 = u.T @ (qj * (L / Z)[:, None])
        s1 = u.T @ (1.0 / Z)
        s2 = u.T @ (L / Z)
        grad = (2.0 / C) * (lp[:, None] * A1 - A2 - (lp * s1 - s2)[:, None] * K)
        step = Kn.astype(np.float64) - K  # the oracle's update, stored in fp32
        ulp = np.spacing(np.abs(Kn)).astype(np.float64)
        assert np.abs(lr * grad).max() > 1e3 * ulp.max()  # a step far above the storage rounding
        assert np.all(np.abs(step + lr * grad) <= ulp)


def test_uniform_usage_gives_zero_key_step():
    """Two tokens mirrored about symmetric keys: pbar is uniform, so the entropy is maximal."""
    cfg = oracle.make_cfg(n=2, d=2, d_v=2, k=1, chunk=2, key_update=True, lr_key=10.0)
    K1 = np.array([[1.0], [-1.0]], np.float32)
    K2 = np.array([[2.0], [-2.0]], np.float32)
    q = np.array([[0.5, 0.25], [-0.5, -0.25]])
    K1n, K2n = K1.copy(), K2.copy()
    oracle.chunk(cfg, q, np.zeros((2, 2)), np.ones(2), None, K1n, K2n, np.zeros((4, 2), np.float32))
    np.testing.assert_allclose(K1n, K1, atol=1e-7)
    np.testing.assert_allclose(K2n, K2, atol=1e-7)


# --------------------------------------------------------------------------- invariants
def _rand_seq(rng, n, h, dv, T):
    q = rng.standard_normal((T, 2 * h)); v = rng.standard_normal((T, dv)); g = rng.uniform(0, 1, T)
    K1 = rng.standard_normal((n, h)).astype(np.float32)
    K2 = rng.standard_normal((n, h)).astype(np.float32)
    V = (0.1 * rng.standard_normal((n * n, dv))).astype(np.float32)
    return q, v, g, K1, K2, V


@pytest.mark.parametrize("key_update", [False, True])
def test_causality(key_update):
    rng = np.random.default_rng(11)
    n, h, dv, k, C, T = 8, 3, 5, 4, 4, 16
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=dv, k=k, chunk=C, key_update=key_update, lr_key=50.0)
    q, v, g, K1, K2, V = _rand_seq(rng, n, h, dv, T)
    base = oracle.run_sequence(cfg, q, v, g, K1.copy(), K2.copy(), V.copy())[0]
    # everything from token 2C on changes: outputs of chunks 0 and 1 must not move
    q2, v2, g2 = q.copy(), v.copy(), g.copy()
    q2[2 * C:] += 1.0; v2[2 * C:] -= 2.0; g2[2 * C:] = 1 - g2[2 * C:]
    pert = oracle.run_sequence(cfg, q2, v2, g2, K1.copy(), K2.copy(), V.copy())[0]
    np.testing.assert_array_equal(pert[:2 * C], base[:2 * C])
    assert np.abs(pert[2 * C:] - base[2 * C:]).max() > 0
    # only v_{2C} changes: it is the lookahead target of token 2C-1, so chunk 2 reads differ
    v3 = v.copy(); v3[2 * C] += np.linspace(-3.0, 2.0, dv)  # not a constant: z-scoring removes those
    pert = oracle.run_sequence(cfg, q, v3, g, K1.copy(), K2.copy(), V.copy())[0]
    np.testing.assert_array_equal(pert[:2 * C], base[:2 * C])
    sa = [K1.copy(), K2.copy(), V.copy()]
    sb = [K1.copy(), K2.copy(), V.copy()]
    oracle.run_sequence(cfg, q[:2 * C + 1], v[:2 * C + 1], g[:2 * C + 1], *sa)
    oracle.run_sequence(cfg, q[:2 * C + 1], v3[:2 * C + 1], g[:2 * C + 1], *sb)
    assert np.abs(sa[2] - sb[2]).max() > 0  # the state after chunk 1 saw v_{2C}
    np.testing.assert_array_equal(sa[0], sb[0])  # keys never see values
    # a target inside chunk 1 does not reach that chunk's own outputs except its own residual
    v4 = v.copy(); v4[C + 2] += np.linspace(-3.0, 2.0, dv)
    pert = oracle.run_sequence(cfg, q, v4, g, K1.copy(), K2.copy(), V.copy())[0]
    np.testing.assert_array_equal(np.delete(pert[:2 * C], C + 2, axis=0), np.delete(base[:2 * C], C + 2, axis=0))


@pytest.mark.parametrize("key_update", [False, True])
def test_passes_compose(key_update):
    """n_iter = 2 equals two n_iter = 1 runs on the carried state, bit for bit."""
    rng = np.random.default_rng(12)
    n, h, dv, k, C, T = 8, 2, 4, 3, 5, 13  # ragged last chunk
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=dv, k=k, chunk=C, key_update=key_update, lr_key=20.0)
    q, v, g, K1, K2, V = _rand_seq(rng, n, h, dv, T)
    a = [K1.copy(), K2.copy(), V.copy()]
    o2 = oracle.run_sequence(cfg, q, v, g, *a, n_iter=2)[0]
    b = [K1.copy(), K2.copy(), V.copy()]
    oracle.run_sequence(cfg, q, v, g, *b, n_iter=1)
    o1 = oracle.run_sequence(cfg, q, v, g, *b, n_iter=1)[0]
    np.testing.assert_array_equal(o2, o1)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    assert np.abs(a[2] - V).max() > 0


def test_sequence_equals_chunk_calls_with_boundary_lookahead():
    rng = np.random.default_rng(13)
    n, h, dv, k, C, T = 8, 2, 4, 3, 4, 10
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=dv, k=k, chunk=C, key_update=True, lr_key=5.0)
    q, v, g, K1, K2, V = _rand_seq(rng, n, h, dv, T)
    s = [K1.copy(), K2.copy(), V.copy()]
    o_seq = oracle.run_sequence(cfg, q, v, g, *s)[0]
    c = [K1.copy(), K2.copy(), V.copy()]
    outs = []
    for t0 in range(0, T, C):
        t1 = min(T, t0 + C)
        vn = v[t1] if t1 < T else None
        outs.append(oracle.chunk(cfg, q[t0:t1], v[t0:t1], g[t0:t1], vn, *c)[0])
    np.testing.assert_array_equal(np.concatenate(outs), o_seq)
    for x, y in zip(s, c):
        np.testing.assert_array_equal(x, y)


def test_boundary_token_rewrites_to_next_chunk_value():
    """k = 1, g = 1: a slot read only by the last token of chunk 0 becomes z(v_C)."""
    C = 3
    cfg = oracle.make_cfg(n=2, d=2, d_v=4, k=1, chunk=C, eps_norm=0.0)
    K1 = np.array([[0.0], [10.0]], np.float32); K2 = K1.copy()
    V = np.zeros((4, 4), np.float32)
    q = np.array([[10.0, 10.0], [10.0, 0.0], [0.0, 0.0], [0.0, 10.0], [10.0, 10.0]])  # token 2 -> slot 0
    v = np.zeros((5, 4)); v[3] = [4, -4, -4, 4]
    g = np.ones(5)
    oracle.chunk(cfg, q[:C], v[:C], g[:C], v[C], K1, K2, V)
    np.testing.assert_array_equal(V[0], [1, -1, -1, 1])


def test_zscore_moments():
    rng = np.random.default_rng(14)
    cfg = oracle.make_cfg(n=2, d=2, d_v=64, k=1, chunk=2, eps_norm=1e-5)
    for scale in (1e-3, 1.0, 50.0):
        u = scale * rng.standard_normal(64) + 3.0
        tau = oracle.target(cfg, u)
        var = u.var()
        assert abs(tau.mean()) < 1e-12
        assert abs(tau.var() - var / (var + 1e-5)) < 1e-12
        assert np.all(np.sign(tau) == np.sign(u - u.mean()))


def test_gate_limits():
    rng = np.random.default_rng(15)
    n, h, dv, k, T = 8, 2, 4, 1, 6
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=dv, k=k, chunk=T)
    q, v, g, K1, K2, V = _rand_seq(rng, n, h, dv, T)
    # g = 0: output is the token's own value and the memory is not written
    V0 = V.copy()
    o, I, w = oracle.chunk(cfg, q, v, np.zeros(T), None, K1, K2, V)
    np.testing.assert_array_equal(o, v)
    np.testing.assert_array_equal(V, V0)
    # g = 1, k = 1: output is exactly the selected row
    o, I, w = oracle.chunk(cfg, q, v, np.ones(T), None, K1, K2, V)
    np.testing.assert_array_equal(o, V0[I[:, 0]].astype(np.float64))


def test_single_token_and_lookahead_off():
    rng = np.random.default_rng(16)
    n, h, dv, k = 4, 2, 3, 2
    q, v, g, K1, K2, V = _rand_seq(rng, n, h, dv, 1)
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=dv, k=k, chunk=4)
    V0 = V.copy()
    oracle.run_sequence(cfg, q, v, g, K1, K2, V)
    np.testing.assert_array_equal(V, V0)  # one token: no lookahead target, nothing written
    # lookahead off: the target is the token's own value, so the lone token writes
    cfg2 = oracle.make_cfg(n=n, d=2 * h, d_v=dv, k=1, chunk=4, lookahead=False, target_norm=False)
    o, I, w = oracle.run_sequence(cfg2, q, v, np.ones(1), K1, K2, V)
    np.testing.assert_allclose(V[I[0, 0]], v[0], rtol=1e-7)


@pytest.mark.parametrize("nthreads", [1, 2, 3, 7])
def test_independent_memories_in_threads_equal_one_call_per_memory(nthreads):
    """orc_run_sequence_multi (the CPU baseline's entry point: memories spread over
    threads, each memory's inputs and state at its own stride; with more threads than
    memories each chunk's read phase is split over token ranges) gives, bit for bit, the
    outputs, slots and states of one orc_run_sequence per memory -- the memories share
    nothing and the tokens of a chunk's read phase are independent."""
    rng = np.random.default_rng(7)
    n, h, dv, k, C, T, M = 16, 8, 8, 4, 5, 13, 3
    cfg = oracle.make_cfg(n, 2 * h, dv, k, C, key_update=True, lr_key=10.0)
    q = rng.normal(size=(M, T, 2 * h))
    v = rng.normal(size=(M, T, dv))
    g = rng.uniform(size=(M, T))
    K1 = rng.normal(size=(M, n, h)).astype(np.float32)
    K2 = rng.normal(size=(M, n, h)).astype(np.float32)
    V = (0.02 * rng.normal(size=(M, n * n, dv))).astype(np.float32)
    k1, k2, vv = K1.copy(), K2.copy(), V.copy()
    o_multi, used, I_multi = oracle.run_sequence_multi(cfg, q, v, g, k1, k2, vv, n_iter=2, nthreads=nthreads,
                                                       with_slots=True)
    assert used == (nthreads if nthreads <= M else M * (nthreads // M))
    for m in range(M):
        a1, a2, av = K1[m].copy(), K2[m].copy(), V[m].copy()
        o_m, I_m, _ = oracle.run_sequence(cfg, q[m], v[m], g[m], a1, a2, av, n_iter=2)
        assert np.array_equal(o_multi[m], o_m), f"memory {m}: o"
        assert np.array_equal(I_multi[m], I_m), f"memory {m}: slots"
        assert np.array_equal(k1[m], a1) and np.array_equal(k2[m], a2), f"memory {m}: keys"
        assert np.array_equal(vv[m], av), f"memory {m}: values"
