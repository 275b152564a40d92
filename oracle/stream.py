"""Token-at-a-time inference in the oracle: the memory read one token at a time and
written once a chunk of (q_t, v_{t+1}) pairs is ready.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline
leg may import this module; the CUDA library shares no code with it and never calls it.

Source: "Fast-weight Product Key Memory" (paperlayer summary of arXiv 2601.00671v2),
§A.1 Lookahead Value Targets: the target of q_t is the next token's value v_{t+1}; the
fast weights change only after a full chunk, so the lookahead does not alter the outputs
inside the chunk; at inference the memory accumulates pairs until a chunk's worth is
ready.  Steps, per arriving token t of one memory:
  1. if C tokens are held, the held chunk is written now, the arriving token's v being
     the target of the chunk's last token (the write of the method: the gated
     reconstruction step on V and, when enabled, the entropy step on the keys);
  2. token t is read against the current state (sub-key distances, per-half top-k,
     Cartesian top-k of the inverse-distance scores, softmax weights, weighted value
     sum, gated output) and held.
At the end of the sequence the held tokens are written with no target for the last one.
The read and write steps are the oracle's own (oracle/__init__.py and fwpkm_oracle.c).
"""
from __future__ import annotations

import numpy as np

from . import chunk, read_values, select, subkey_dist


def read_token(cfg, q_t, v_t, g_t, K1, K2, V):
    """The read of one token against the state (K1, K2, V) -- method steps 2-3 of the
    rainbus summary, the scores of paperlayer §A.2: returns (o_t, I_t, s'_t)."""
    q_t = np.asarray(q_t, dtype=np.float64)
    D1 = subkey_dist(cfg, q_t[:cfg.h], K1)
    D2 = subkey_dist(cfg, q_t[cfg.h:], K2)
    I, _, w = select(cfg, D1, D2)
    vhat = read_values(cfg, I, w, V)
    return g_t * vhat + (1.0 - g_t) * np.asarray(v_t, dtype=np.float64), I, w


def stream_sequence(cfg, q, v, g, K1, K2, V, groups):
    """Feed the tokens of one memory in arrival groups of the given sizes (summing to T),
    then end the sequence (paperlayer §A.1: pairs accumulate until a chunk is ready).
    K1, K2, V (fp32) are updated in place.  Returns o [T][d_v]."""
    q = np.asarray(q, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    T = q.shape[0]
    assert sum(groups) == T
    o = np.empty((T, cfg.d_v))
    held0, held = 0, 0  # held tokens are [held0, held0 + held)
    t = 0
    for n in groups:
        for _ in range(n):
            if held == cfg.chunk:
                chunk(cfg, q[held0:t], v[held0:t], g[held0:t], v[t], K1, K2, V)
                held0, held = t, 0
            o[t], _, _ = read_token(cfg, q[t], v[t], g[t], K1, K2, V)
            held += 1
            t += 1
    if held:
        chunk(cfg, q[held0:t], v[held0:t], g[held0:t], None, K1, K2, V)
    return o
