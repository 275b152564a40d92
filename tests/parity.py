"""Shared helpers of the GPU-vs-oracle parity tests (imported by tests only).

Tolerances (fp32 GPU arithmetic against the fp64 oracle):
  * slot indices: bit-exact, except documented near-ties: at every rank r the GPU's
    slot scores (in fp64) within 1e-6 * max(1, |S_r|) of the oracle's r-th score.
    Near-ties are counted; the oracle then adopts the GPU's slots for that token
    (forced mode) so o / V / K comparisons do not cascade.
  * o, V, K1, K2 and the weights: |gpu - oracle| <= 1e-5 + 1e-4 * |oracle|.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from sparse_weight_memory_chunk_b200.inputs import bf16_to_f32

RTOL, ATOL = 1e-4, 1e-5
TIE_REL = 1e-6


def as_f64(x, qv):
    return bf16_to_f32(x).astype(np.float64) if qv == "bf16" else np.asarray(x, np.float64)


def to_device(x, qv, torch, device="cuda"):
    """numpy input (fp32 or bf16 bits) -> torch tensor on the device."""
    if qv == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)


def assert_close(got, ref, what, rtol=RTOL, atol=ATOL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bad = np.abs(got - ref) > atol + rtol * np.abs(ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"gpu={got[tuple(i)]!r} oracle={ref[tuple(i)]!r}")


_libm_log = np.vectorize(math.log)


def classify_selection(ocfg, q_tok, K1, K2, I_gpu):
    """'exact', 'near_tie' or a failure string for one token's GPU slot list."""
    h, n, k = ocfg.h, ocfg.n, ocfg.k
    D1 = oracle.subkey_dist(ocfg, q_tok[:h], K1)
    D2 = oracle.subkey_dist(ocfg, q_tok[h:], K2)
    I_o, S_o, _ = oracle.select(ocfg, D1, D2)
    if np.array_equal(I_o, I_gpu):
        return "exact"
    if len(set(I_gpu.tolist())) != k or I_gpu.min() < 0 or I_gpu.max() >= n * n:
        return f"invalid slot list {I_gpu}"
    a, b = I_gpu // n, I_gpu % n
    S_g = -_libm_log(ocfg.eps_idw + D1[a]) - _libm_log(ocfg.eps_idw + D2[b])
    tol = TIE_REL * np.maximum(1.0, np.abs(S_o))
    if np.all(np.abs(S_g - S_o) <= tol):
        return "near_tie"
    return f"selection mismatch: gpu {I_gpu} (S {S_g}) vs oracle {I_o} (S {S_o})"


def oracle_chunk_against_gpu(ocfg, q, v, g, v_next, K1, K2, V, idx_gpu):
    """Run the oracle on one chunk of one memory from the given (GPU) pre-chunk state.

    q, v, g: fp64 chunk inputs; K1, K2, V: fp32 copies (updated in place).
    Returns (o, I, w, near_ties)."""
    length = q.shape[0]
    force = np.zeros(length, np.int32)
    ties = 0
    for t in range(length):
        verdict = classify_selection(ocfg, q[t], K1, K2, idx_gpu[t])
        if verdict == "near_tie":
            force[t] = 1
            ties += 1
        elif verdict != "exact":
            raise AssertionError(f"token {t}: {verdict}")
    o, I, w = oracle.chunk(ocfg, q, v, g, v_next, K1, K2, V, forced=idx_gpu, force_mask=force)
    return o, I, w, ties
