"""The seeded synthetic inputs follow their recipe (CPU only).

The generators hold none of the method's arithmetic; these checks pin the recipe the
workloads state: RMS-normalised q and v, gates in (0, 1) (uniform or sigmoid of a
normal), N(0, 1) sub-keys, V zero or N(0, 0.02^2), the needle planting structure, the
layer's clustered hidden states and N(0, 1/fan_in) weights, and determinism.
"""
import numpy as np
import pytest

from sparse_weight_memory_chunk_b200.inputs import (WORKLOADS, bf16_to_f32, f32_to_bf16, gen_keys, gen_layer,
                                                    gen_needles, gen_qvg, gen_values)


def test_bf16_round_trip_and_rounding():
    # bf16 keeps 8 significant bits: the spacing just above 1 is 2^-7
    exact = np.array([1.0, 1.0 + 2.0 ** -7, -3.140625, 0.0, 2.0 ** -20], dtype=np.float32)
    assert np.array_equal(bf16_to_f32(f32_to_bf16(exact)), exact)
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 3 * 2.0 ** -9], dtype=np.float32)
    # halfway cases go to the even neighbour; others to the nearest
    want = np.array([1.0, 1.0 + 2.0 ** -6, 1.0 + 2.0 ** -7], dtype=np.float32)
    assert np.array_equal(bf16_to_f32(f32_to_bf16(ties)), want)
    r = np.random.default_rng(0).normal(size=4096).astype(np.float32)
    rel = np.abs(bf16_to_f32(f32_to_bf16(r)) - r) / np.abs(r)
    assert rel.max() <= 2.0 ** -8


@pytest.mark.parametrize("wid", [1, 2])
def test_qvg_recipe(wid):
    w = WORKLOADS[wid]
    M = min(2, w.M)
    q, v, g = gen_qvg(w, M=M, T=64)
    assert q.shape == (M, 64, w.d) and v.shape == (M, 64, w.d_v) and g.shape == (M, 64)
    qf = bf16_to_f32(q) if w.qv == "bf16" else q
    vf = bf16_to_f32(v) if w.qv == "bf16" else v
    tol = 2e-2 if w.qv == "bf16" else 1e-5
    np.testing.assert_allclose(np.mean(qf.astype(np.float64) ** 2, axis=-1), 1.0, atol=tol)
    np.testing.assert_allclose(np.mean(vf.astype(np.float64) ** 2, axis=-1), 1.0, atol=tol)
    assert g.dtype == np.float32 and (g > 0).all() and (g < 1).all()
    # deterministic, and the first tokens do not depend on how many are asked for
    q2, v2, g2 = gen_qvg(w, M=M, T=32)
    assert np.array_equal(q2, q[:, :32]) and np.array_equal(v2, v[:, :32]) and np.array_equal(g2, g[:, :32])


def test_gate_distributions():
    _, _, gu = gen_qvg(WORKLOADS[1])          # uniform gates
    _, _, gs = gen_qvg(WORKLOADS[2], M=4)     # sigmoid of N(0, 1)
    assert abs(gu.mean() - 0.5) < 0.05 and abs(gu.std() - np.sqrt(1 / 12)) < 0.03
    z = np.log(gs / (1 - gs))
    assert abs(z.mean()) < 0.05 and abs(z.std() - 1.0) < 0.05


def test_keys_and_values():
    w = WORKLOADS[2]
    K1, K2 = gen_keys(w, M=2)
    assert K1.shape == (2, w.n, w.h) and K1.dtype == np.float32
    assert not np.array_equal(K1, K2)
    assert abs(K1.std() - 1.0) < 0.02 and abs(K1.mean()) < 0.02
    V = gen_values(w, 0)
    assert V.shape == (w.N, w.d_v) and V.dtype == np.float32
    assert abs(V.std() - 0.02) < 1e-3
    assert not np.array_equal(V[:64], gen_values(w, 1)[:64])
    assert not gen_values(WORKLOADS[1], 0).any()  # the tiny workload starts from V = 0


def test_needle_structure():
    from dataclasses import replace
    w = replace(WORKLOADS[4], T=4096, needles=16)
    q, v, g = gen_qvg(w)
    pos, qpos, qs, vs = gen_needles(w, q, v)
    T = q.shape[1]
    assert pos.shape == (16, 3) and qpos.shape == (16,)
    assert (pos % 2 == 0).all() and (pos + 1 < int(0.9 * T)).all()
    assert len(np.unique(pos)) == 48                       # distinct planting positions
    assert (qpos >= int(0.9 * T)).all() and len(np.unique(qpos)) == 16
    for i in range(16):
        for p in pos[i]:
            assert np.array_equal(q[0, p], qs[i]) and np.array_equal(v[0, p + 1], vs[i])
        assert np.array_equal(q[0, qpos[i]], qs[i])


def test_layer_recipe():
    w = WORKLOADS[5]
    L = gen_layer(w, B=2, T=256)
    h = bf16_to_f32(L["h"]).astype(np.float64)
    assert h.shape == (2, 256, w.d_model)
    # clustered: each token is a centre plus 0.1 N(0, I) noise, so two tokens of one cluster
    # differ by ~0.1 sqrt(2) per coordinate while centres differ by ~sqrt(2)
    x = h.reshape(-1, w.d_model)
    d = np.sqrt(np.mean((x[:, None, :64] - x[None, :, :64]) ** 2, axis=-1))
    near = d < 0.5
    assert near.sum() > x.shape[0]  # some pairs share a cluster (the Zipf head is heavy)
    assert np.all((d[near] < 0.3) | np.eye(len(x), dtype=bool)[near])
    for name, fan_in in (("Wq", w.d_model), ("Wv", w.d_model), ("Wo", w.d_v)):
        W = bf16_to_f32(L[name]).astype(np.float64)
        assert abs(W.std() * np.sqrt(fan_in) - 1.0) < 0.05, name
    assert L["Wq"].shape == (w.d, w.d_model) and L["Wo"].shape == (w.d_model, w.d_v)
