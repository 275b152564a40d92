"""Plain fp64 oracle of the slow-weight projections around the fast-weight memory.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline
leg may import this module; the CUDA library shares no code with it and never calls it.

Source: "快速权重积键值记忆 Fast-weight Product Key Memory" (structured summary), method
steps 1 and 3: the memory's inputs are built by the slow-weight network as
q_t = Linear_q(RMSNorm_q(h_t)), v_t = Linear_v(RMSNorm_v(h_t)),
g_t = sigmoid(Linear_g(RMSNorm_g(h_t))), and the output is o'_t = Linear_o(RMSNorm_o(o_t)).

Readings where the pages are silent:
  * RMSNorm(x) = x / sqrt(mean_e x_e^2 + eps) * gamma (elementwise weight gamma, no
    mean subtraction, eps = 1e-6).
  * Linear(x) = x W^T + b with W stored [out][in] (bias b; zero in the workloads).
  * Every projection has its own RMSNorm weight, as the pages' notation gives each one.

Everything is evaluated in fp64 from the stored (bf16 or fp32) values, in the order of
the definition: the norm, then the weight, then the product, then the bias.
"""
from __future__ import annotations

import numpy as np


def rmsnorm(x, gamma, eps):
    """RMSNorm of every row of x ([R][D]) with weight gamma ([D]), fp64."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)[None, :]


def linear(x, W, b):
    """x W^T + b with W [out][in], fp64 (the matrix product is numpy's)."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :]
    return y


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))


def project_in(h, gq, Wq, bq, gv, Wv, bv, gg, wg, bg, eps=1e-6):
    """Method step 1: h [R][D] -> q [R][d], v [R][d_v], g [R] (all fp64)."""
    q = linear(rmsnorm(h, gq, eps), Wq, bq)
    v = linear(rmsnorm(h, gv, eps), Wv, bv)
    zg = linear(rmsnorm(h, gg, eps), np.asarray(wg, dtype=np.float64)[None, :],
                None if bg is None else np.array([bg], dtype=np.float64))
    return q, v, sigmoid(zg[:, 0])


def project_out(o, go, Wo, bo, eps=1e-6):
    """Method step 3 (second half): o [R][d_v] -> o' [R][D] (fp64)."""
    return linear(rmsnorm(o, go, eps), Wo, bo)
