"""Plain oracle of the addressing metrics (slot-use balance of the memory reads).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline
leg may import this module; the CUDA library shares no code with it and never calls it.

Source: "Fast-weight Product Key Memory" (paperlayer summary of arXiv 2601.00671v2),
§D.3 Addressing Metrics: the row contribution of a value row is how many accesses it
received; from it come the coverage rate (share of the slots that were accessed), the
collision rate (share of competitive accesses) and the KL divergence of slot use from
the uniform distribution, each measured over fixed windows of tokens (32K tokens there,
chosen so that a perfectly balanced top-8 selection would touch every one of the 256K
slots exactly once).

Readings where the section is silent:
  * An access is one (token, selected slot) pair of the read: a token of a memory with
    top-k selection makes k accesses, one to each of its k distinct slots.
  * Windows are consecutive blocks of `window` tokens of one memory's sequence; the last
    window holds the remaining tokens (it may be shorter).  Memories are measured apart.
  * Collision rate = (accesses whose row received at least two accesses in the window)
    / (all accesses of the window): an access is competitive when another access of the
    same window lands on its row.
  * KLD = sum_i p_i log(p_i N) with p_i = c_i / sum c (natural log, 0 log 0 = 0), the
    divergence KL(p || uniform over all N slots).
  * Entries outside [0, N) are not accesses; they are counted apart (`invalid`).
  * A window with no access has coverage, collision and KLD 0.

The definition is written out directly: a per-window histogram (numpy bincount) and the
three ratios evaluated from it in fp64.
"""
from __future__ import annotations

import numpy as np


def window_count(T: int, window: int) -> int:
    """Windows of `window` tokens covering T tokens (the last one may be shorter; §D.3
    measures every 32K tokens)."""
    return (T + window - 1) // window


def addressing_metrics(idx, N: int, window: int):
    """Metrics of every (memory, window), paperlayer §D.3: row contributions c_i per window,
    then coverage, collision rate and KL divergence from uniform slot use.

    idx: int array [M][T][k] of selected slots.  Returns (metrics, counts):
      metrics fp64 [M][W][3]: coverage, collision rate, KLD;
      counts  int64 [M][W][4]: rows accessed, accesses, competitive accesses, invalid entries.
    """
    idx = np.asarray(idx)
    M, T, _ = idx.shape
    W = window_count(T, window)
    metrics = np.zeros((M, W, 3), dtype=np.float64)
    counts = np.zeros((M, W, 4), dtype=np.int64)
    for m in range(M):
        for w in range(W):
            sel = idx[m, w * window:min(T, (w + 1) * window)].reshape(-1).astype(np.int64)
            ok = (sel >= 0) & (sel < N)
            c = np.bincount(sel[ok], minlength=N).astype(np.int64)  # row contributions
            S = int(c.sum())
            U = int((c > 0).sum())
            comp = int(c[c >= 2].sum())
            counts[m, w] = (U, S, comp, int((~ok).sum()))
            if S == 0:
                continue
            p = c[c > 0].astype(np.float64) / S
            metrics[m, w, 0] = U / N
            metrics[m, w, 1] = comp / S
            metrics[m, w, 2] = float(np.sum(p * np.log(p * N)))
    return metrics, counts
