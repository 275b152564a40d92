"""Pins of the slow-weight projection oracle (oracle/layer.py) to things other than itself:
a hand-worked example (tests/golden), the library's own RMSNorm and Linear in fp64, and
invariants a dropped term, a wrong gamma or a variance-for-mean-square slip would break.
"""
import json
import os

import numpy as np
import pytest

from oracle import layer

torch = pytest.importorskip("torch")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_hand_worked():
    f = json.load(open(os.path.join(GOLDEN, "layer_rmsnorm_linear.json")))
    h = np.array(f["h"])
    q, v, g = layer.project_in(h, f["gamma_q"], f["W_q"], f["b_q"], f["gamma_v"], f["W_v"], f["b_v"],
                               f["gamma_g"], f["w_g"], f["b_g"], eps=0.0)
    np.testing.assert_allclose(q, f["expect_q"], rtol=0, atol=1e-9)
    np.testing.assert_allclose(v, f["expect_v"], rtol=0, atol=1e-9)
    np.testing.assert_allclose(g, f["expect_g"], rtol=0, atol=1e-9)
    oo = layer.project_out(np.array(f["o"]), f["gamma_o"], f["W_o"], f["b_o"], eps=0.0)
    np.testing.assert_allclose(oo, f["expect_o_out"], rtol=0, atol=1e-12)


def test_matches_library_rmsnorm_and_linear():
    rng = np.random.default_rng(5)
    R, D, N = 7, 48, 20
    x = rng.normal(size=(R, D)) + 0.7  # non-zero mean: a variance-based norm would differ
    gamma = rng.uniform(0.5, 1.5, size=D)
    W = rng.normal(size=(N, D)) / np.sqrt(D)
    b = rng.normal(size=N)
    ref = torch.nn.functional.linear(
        torch.nn.functional.rms_norm(torch.from_numpy(x), (D,), torch.from_numpy(gamma), eps=1e-6),
        torch.from_numpy(W), torch.from_numpy(b)).numpy()
    np.testing.assert_allclose(layer.linear(layer.rmsnorm(x, gamma, 1e-6), W, b), ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(layer.project_out(x, gamma, W, b), ref, rtol=1e-12, atol=1e-12)


def test_unit_mean_square_and_scale_invariance():
    rng = np.random.default_rng(6)
    x = rng.normal(size=(5, 32)) * rng.uniform(0.1, 10, size=(5, 1)) + 3.0
    y = layer.rmsnorm(x, np.ones(32), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-13)
    W = rng.normal(size=(8, 32))
    wg = rng.normal(size=32)
    a = layer.project_in(x, np.ones(32), W, None, np.ones(32), W, None, np.ones(32), wg, 0.0, eps=0.0)
    bb = layer.project_in(37.5 * x, np.ones(32), W, None, np.ones(32), W, None, np.ones(32), wg, 0.0, eps=0.0)
    for u, w in zip(a, bb):
        np.testing.assert_allclose(u, w, rtol=1e-12, atol=1e-14)


def test_each_projection_uses_its_own_norm_weight_and_gate_limits():
    rng = np.random.default_rng(7)
    D = 16
    h = rng.normal(size=(4, D))
    W = rng.normal(size=(6, D))
    ones = np.ones(D)
    q1, v1, g1 = layer.project_in(h, ones, W, None, ones, W, None, ones, np.zeros(D), 0.0)
    q2, v2, g2 = layer.project_in(h, ones, W, None, 2 * ones, W, None, ones, np.zeros(D), 0.0)
    np.testing.assert_array_equal(q1, q2)          # gamma_v does not reach q
    np.testing.assert_allclose(v2, 2 * v1, rtol=1e-14)  # gamma scales the normalised input
    np.testing.assert_array_equal(g1, 0.5)         # zero gate weights and bias: sigmoid(0)
    _, _, g3 = layer.project_in(h, ones, W, None, ones, W, None, ones, np.zeros(D), 40.0)
    assert np.all(g3 >= 1 - 1e-15)
    _, _, g4 = layer.project_in(h, ones, W, None, ones, W, None, ones, np.zeros(D), -40.0)
    assert np.all(g4 < 1e-15)
