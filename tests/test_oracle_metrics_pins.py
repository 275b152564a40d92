"""Pins of the addressing-metrics oracle (oracle/metrics.py) to things other than itself.

* The design point the section states for its window size: a perfectly balanced
  selection whose window makes exactly N accesses touches every slot once (coverage 1,
  no collision, zero divergence).
* Closed forms of degenerate histograms: one hot slot, all-distinct accesses, every
  accessed row hit exactly r times.
* KLD against scipy's relative entropy on arbitrary histograms (a library routine).
* Brute force with plain Python counting on tiny inputs with ragged windows and invalid
  entries, and invariants (slot relabelling, token order inside a window).
A dropped term, a wrong window boundary, a base-2 log or a collision count over rows
instead of accesses fails one of them.
"""
import math
from collections import Counter

import numpy as np
import pytest

from oracle.metrics import addressing_metrics, window_count

scipy_stats = pytest.importorskip("scipy.stats")


def test_balanced_window_covers_every_slot_once():
    # 32K tokens x top-8 = 256K slots in the section; here 64 tokens x top-4 = 256 slots
    N, k, W = 256, 4, 64
    rng = np.random.default_rng(0)
    perm = rng.permutation(N).reshape(1, W, k).astype(np.int32)
    met, cnt = addressing_metrics(perm, N, W)
    assert met.shape == (1, 1, 3)
    assert tuple(cnt[0, 0]) == (N, N, 0, 0)
    assert met[0, 0, 0] == 1.0 and met[0, 0, 1] == 0.0 and abs(met[0, 0, 2]) < 1e-15


def test_one_hot_slot():
    N, T = 1000, 50
    idx = np.full((1, T, 1), 7, dtype=np.int32)
    met, cnt = addressing_metrics(idx, N, T)
    assert tuple(cnt[0, 0]) == (1, T, T, 0)
    assert met[0, 0, 0] == 1 / N and met[0, 0, 1] == 1.0
    assert math.isclose(met[0, 0, 2], math.log(N), rel_tol=1e-15)
    # a single access has no competitor
    met1, cnt1 = addressing_metrics(idx[:, :1], N, T)
    assert tuple(cnt1[0, 0]) == (1, 1, 0, 0) and met1[0, 0, 1] == 0.0


def test_all_distinct_and_equal_multiplicity():
    N, k = 4096, 8
    rng = np.random.default_rng(1)
    slots = rng.permutation(N)[:40 * k].reshape(1, 40, k).astype(np.int32)
    met, cnt = addressing_metrics(slots, N, 40)
    S = 40 * k
    assert tuple(cnt[0, 0]) == (S, S, 0, 0)
    assert met[0, 0, 0] == S / N and met[0, 0, 1] == 0.0
    assert math.isclose(met[0, 0, 2], math.log(N / S), rel_tol=1e-14)
    # the same U rows each read r = 3 times (three copies of the token block)
    rep = np.concatenate([slots, slots, slots], axis=1)
    met3, cnt3 = addressing_metrics(rep, N, 120)
    assert tuple(cnt3[0, 0]) == (S, 3 * S, 3 * S, 0)
    assert met3[0, 0, 0] == S / N and met3[0, 0, 1] == 1.0
    assert math.isclose(met3[0, 0, 2], math.log(N / S), rel_tol=1e-14)


@pytest.mark.parametrize("seed", [2, 3, 4])
def test_kld_matches_scipy_relative_entropy(seed):
    rng = np.random.default_rng(seed)
    N, T, k = 300, 97, 5
    # skewed use: Zipf-like slot popularity, distinct slots per token
    pop = 1.0 / np.arange(1, N + 1) ** 1.1
    pop /= pop.sum()
    idx = np.stack([rng.choice(N, size=k, replace=False, p=pop) for _ in range(T)])[None].astype(np.int32)
    met, cnt = addressing_metrics(idx, N, T)
    c = np.bincount(idx.reshape(-1), minlength=N)
    want = scipy_stats.entropy(c / c.sum(), np.full(N, 1.0 / N))  # natural log
    assert math.isclose(met[0, 0, 2], want, rel_tol=1e-12)
    assert met[0, 0, 2] > 0


def _brute(idx, N, window):
    M, T, _ = idx.shape
    out = []
    for m in range(M):
        row = []
        for w0 in range(0, T, window):
            c = Counter()
            bad = 0
            for t in range(w0, min(T, w0 + window)):
                for s in idx[m, t]:
                    if 0 <= s < N:
                        c[int(s)] += 1
                    else:
                        bad += 1
            S = sum(c.values())
            comp = sum(v for v in c.values() if v > 1)
            kl = sum((v / S) * math.log(v / S * N) for v in c.values()) if S else 0.0
            row.append(((len(c), S, comp, bad), (len(c) / N if S else 0.0, comp / S if S else 0.0, kl)))
        out.append(row)
    return out


@pytest.mark.parametrize("T,window", [(23, 5), (20, 5), (1, 4), (9, 100)])
def test_brute_force_ragged_windows_and_invalid_entries(T, window):
    rng = np.random.default_rng(T * 31 + window)
    M, N, k = 3, 12, 3
    idx = np.stack([np.stack([rng.choice(N, size=k, replace=False) for _ in range(T)]) for _ in range(M)])
    idx = idx.astype(np.int32)
    idx[0, 0, 0] = -1
    idx[2, T - 1, k - 1] = N  # out of range: not an access
    met, cnt = addressing_metrics(idx, N, window)
    ref = _brute(idx, N, window)
    assert met.shape[1] == window_count(T, window) == len(ref[0])
    for m in range(M):
        for w, (c, mm) in enumerate(ref[m]):
            assert tuple(cnt[m, w]) == c
            np.testing.assert_allclose(met[m, w], mm, rtol=1e-13, atol=1e-15)
    assert cnt[0, 0, 3] == 1 and cnt[2, -1, 3] == 1


def test_window_boundaries_and_invariants():
    N, k, window = 50, 2, 4
    idx = np.zeros((1, 8, k), dtype=np.int32)
    idx[0, :4] = [0, 1]
    idx[0, 4:] = [2, 3]  # token 4 opens the second window
    met, cnt = addressing_metrics(idx, N, window)
    assert tuple(cnt[0, 0]) == (2, 8, 8, 0) and tuple(cnt[0, 1]) == (2, 8, 8, 0)
    assert met[0, 0, 0] == met[0, 1, 0] == 2 / N
    # relabelling the slots and reordering tokens inside a window change nothing
    rng = np.random.default_rng(9)
    idx = np.stack([rng.choice(N, size=k, replace=False) for _ in range(40)])[None].astype(np.int32)
    perm = rng.permutation(N).astype(np.int32)
    a = addressing_metrics(idx, N, 10)
    b = addressing_metrics(perm[idx], N, 10)
    order = np.concatenate([rng.permutation(10) + 10 * w for w in range(4)])
    c = addressing_metrics(idx[:, order], N, 10)
    for x in (b, c):
        np.testing.assert_array_equal(a[1], x[1])
        np.testing.assert_allclose(a[0], x[0], rtol=1e-14, atol=0)
    # competitive accesses plus rows read once make up all accesses
    cc = np.bincount(idx[0, :10].reshape(-1), minlength=N)
    assert a[1][0, 0, 2] + int((cc == 1).sum()) == a[1][0, 0, 1]


def test_empty_sequence():
    met, cnt = addressing_metrics(np.zeros((2, 0, 4), dtype=np.int32), 16, 8)
    assert met.shape == (2, 0, 3) and cnt.shape == (2, 0, 4)
