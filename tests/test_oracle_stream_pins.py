"""Pins of the token-at-a-time oracle (oracle/stream.py) to what the method fixes.

§A.1 (Lookahead Value Targets) of the method's description says that the fast weights
change only after a full chunk and that inference accumulates pairs until a chunk's worth
is ready, so feeding a sequence one token (or any group) at a time must give exactly the
chunk-sequential result; and the lookahead target of a chunk's last token (the next
chunk's first value) must not reach the outputs of that chunk.
"""
import numpy as np
import pytest

import oracle
from oracle.stream import read_token, stream_sequence


def case(seed, n=16, h=4, dv=8, k=4, C=5, T=23, key_update=True):
    rng = np.random.default_rng(seed)
    cfg = oracle.make_cfg(n=n, d=2 * h, d_v=dv, k=k, chunk=C, key_update=key_update, lr_key=30.0)
    q = rng.normal(size=(T, 2 * h))
    v = rng.normal(size=(T, dv))
    g = rng.uniform(0.1, 0.9, size=T)
    K1 = rng.normal(size=(n, h)).astype(np.float32)
    K2 = rng.normal(size=(n, h)).astype(np.float32)
    V = (0.3 * rng.normal(size=(n * n, dv))).astype(np.float32)
    return cfg, q, v, g, K1, K2, V


@pytest.mark.parametrize("groups", [[1] * 23, [5] * 4 + [3], [2, 7, 1, 13], [23], [4, 1, 6, 5, 5, 2]])
@pytest.mark.parametrize("key_update", [False, True])
def test_any_grouping_equals_the_chunked_loop(groups, key_update):
    cfg, q, v, g, K1, K2, V = case(1, key_update=key_update)
    a = [x.copy() for x in (K1, K2, V)]
    o_ref, _, _ = oracle.run_sequence(cfg, q, v, g, *a)
    b = [x.copy() for x in (K1, K2, V)]
    o = stream_sequence(cfg, q, v, g, *b, groups)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)  # the same write steps on the same inputs
    np.testing.assert_allclose(o, o_ref, rtol=1e-14, atol=1e-15)
    assert not np.array_equal(b[2], V), "the memory was not written"


def test_lookahead_reaches_only_the_state():
    cfg, q, v, g, K1, K2, V = case(2, n=8, C=5, T=15, key_update=False)
    q[6] = q[4]  # token 6 reads the rows that chunk 0's last token wrote
    base = [x.copy() for x in (K1, K2, V)]
    o0 = stream_sequence(cfg, q, v, g, *base, [1] * 15)
    v2 = v.copy()
    # first value of chunk 1 = the lookahead target of chunk 0's last token (a change
    # that survives the z-score: not a constant shift or a scale)
    v2[5] += 3.0 * np.random.default_rng(5).normal(size=v.shape[1])
    pert = [x.copy() for x in (K1, K2, V)]
    o1 = stream_sequence(cfg, q, v2, g, *pert, [1] * 15)
    np.testing.assert_array_equal(o0[:5], o1[:5])     # chunk 0's outputs unchanged
    assert not np.array_equal(base[2], pert[2])       # the state is
    assert not np.array_equal(o0[6], o1[6])           # and chunk 1 reads that state


def test_read_token_matches_the_chunk_read():
    cfg, q, v, g, K1, K2, V = case(3, C=6, T=6, key_update=False)
    o_chunk, I_chunk, w_chunk = oracle.chunk(cfg, q, v, g, None, K1.copy(), K2.copy(), V.copy())
    for t in range(6):
        o_t, I_t, w_t = read_token(cfg, q[t], v[t], g[t], K1, K2, V)
        np.testing.assert_array_equal(I_t, I_chunk[t])
        np.testing.assert_allclose(w_t, w_chunk[t], rtol=1e-15, atol=0)
        np.testing.assert_allclose(o_t, o_chunk[t], rtol=1e-14, atol=1e-15)
