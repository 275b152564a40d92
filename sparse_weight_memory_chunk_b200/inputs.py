"""Seeded synthetic workloads for the FwPKM retrieve + chunk-write loop.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can be fed from it.
Every tensor comes from its own numpy ``PCG64`` sub-stream (``SeedSequence.spawn``)
in a fixed order, so a tensor's bits never depend on which other tensors were
generated.  Large per-memory tensors (V) get one sub-stream per memory, so one
memory's V can be regenerated alone.

Workload shapes follow the five workloads of the measurement plan:
  1 tiny    n=64 (N=4096), d=d_v=64, k=8, T=256, C=64, fp32 q/v, 1 memory
  2 mid     n=256 (N=65,536), d=d_v=128, k=16, T=4096, C=128, bf16 q/v, B4 x H4
  3 paper   n=1024 (N=1,048,576), d=d_v=256, k=32, T=4096, C=256, bf16, B4 x H2,
            entropy key update on
  4 needle  N=1,048,576, d=d_v=256, k=32, T=131,072, C=512, 1 memory, 64 planted
            needle pairs, n_iter in {1, 2, 4}
  5 layer   d_model=2048 clustered bf16 hidden states, N=262,144 (n=512), k=32,
            B16 x H1, T=4096, C=256, key update on
bf16 tensors are carried as ``uint16`` bit patterns (round-to-nearest-even from
fp32); ``bf16_to_f32`` widens them exactly.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n: int
    d: int
    d_v: int
    k: int
    T: int
    C: int
    B: int
    H: int
    qv: str            # "f32" or "bf16"
    key_update: bool
    seed: int
    gate: str          # "uniform" (U(0,1)) or "sigmoid" (sigmoid(N(0,1)))
    v_init: str        # "zero" or "normal002" (N(0, 0.02^2))
    n_iter: int = 1
    d_model: int = 0   # > 0: hidden states + slow-weight projections (layer workload)
    needles: int = 0   # > 0: planted needle pairs (needle workload)

    @property
    def M(self) -> int:
        return self.B * self.H

    @property
    def N(self) -> int:
        return self.n * self.n

    @property
    def h(self) -> int:
        return self.d // 2


WORKLOADS = {
    1: Workload("tiny", 64, 64, 64, 8, 256, 64, 1, 1, "f32", False, 0, "uniform", "zero"),
    2: Workload("mid", 256, 128, 128, 16, 4096, 128, 4, 4, "bf16", False, 1, "sigmoid", "normal002"),
    3: Workload("paper", 1024, 256, 256, 32, 4096, 256, 4, 2, "bf16", True, 2, "sigmoid", "normal002"),
    4: Workload("needle", 1024, 256, 256, 32, 131072, 512, 1, 1, "bf16", False, 3, "sigmoid",
                "normal002", needles=64),
    5: Workload("layer", 512, 256, 256, 32, 4096, 256, 16, 1, "bf16", True, 4, "sigmoid",
                "normal002", d_model=2048),
}


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit pattern."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = u + (((u >> 16) & 1) + 0x7FFF)
    return (u >> 16).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rms_rows(x: np.ndarray) -> np.ndarray:
    """x / sqrt(mean(x^2)) along the last axis, in fp64 (input recipe, not the method)."""
    x = x.astype(np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True))


def _cast(x64: np.ndarray, qv: str) -> np.ndarray:
    x32 = x64.astype(np.float32)
    return f32_to_bf16(x32) if qv == "bf16" else x32


def _streams(seed: int):
    names = ["q", "v", "g", "K1", "K2", "V", "needle", "layer"]
    kids = np.random.SeedSequence(seed).spawn(len(names))
    return dict(zip(names, kids))


def gen_qvg(w: Workload, M: int | None = None, T: int | None = None):
    """q [M][T][d], v [M][T][d_v] (fp32 or bf16 bits), g [M][T] fp32 for memories 0..M-1.

    The first ``T`` tokens of each memory do not depend on the total ``T`` asked for
    because every memory's row block is drawn in one call of fixed shape."""
    M = w.M if M is None else M
    T = w.T if T is None else T
    ss = _streams(w.seed)
    gq = np.random.Generator(np.random.PCG64(ss["q"]))
    gv = np.random.Generator(np.random.PCG64(ss["v"]))
    gg = np.random.Generator(np.random.PCG64(ss["g"]))
    q = _cast(_rms_rows(gq.standard_normal((w.M, w.T, w.d))[:M, :T]), w.qv)
    v = _cast(_rms_rows(gv.standard_normal((w.M, w.T, w.d_v))[:M, :T]), w.qv)
    if w.gate == "uniform":
        g = gg.uniform(0.0, 1.0, (w.M, w.T))[:M, :T].astype(np.float32)
    else:
        z = gg.standard_normal((w.M, w.T))[:M, :T]
        g = (1.0 / (1.0 + np.exp(-z))).astype(np.float32)
    return np.ascontiguousarray(q), np.ascontiguousarray(v), np.ascontiguousarray(g)


def gen_keys(w: Workload, M: int | None = None):
    """K1, K2 [M][n][h] fp32, N(0, 1)."""
    M = w.M if M is None else M
    ss = _streams(w.seed)
    out = []
    for name in ("K1", "K2"):
        kids = ss[name].spawn(w.M)
        out.append(np.stack([np.random.Generator(np.random.PCG64(kids[m]))
                             .standard_normal((w.n, w.h), dtype=np.float32) for m in range(M)]))
    return out[0], out[1]


def gen_values(w: Workload, m: int) -> np.ndarray:
    """Initial V of memory m: [N][d_v] fp32 (zeros, or N(0, 0.02^2))."""
    if w.v_init == "zero":
        return np.zeros((w.N, w.d_v), np.float32)
    kid = _streams(w.seed)["V"].spawn(w.M)[m]
    x = np.random.Generator(np.random.PCG64(kid)).standard_normal((w.N, w.d_v), dtype=np.float32)
    x *= np.float32(0.02)
    return x


def gen_needles(w: Workload, q: np.ndarray, v: np.ndarray):
    """Plant ``w.needles`` (q*, v*) pairs into memory 0's stream (in place).

    Each needle is written at 3 distinct even positions p in the first 90% of the
    stream as q_p = q*, v_{p+1} = v* (so the lookahead target of q* is v*), and
    queried once at a distinct position r in the last 10% (q_r = q*).  Even p keeps
    the (p, p+1) pairs of different needles disjoint.  Returns (positions [nd][3],
    query positions [nd], q* [nd][d], v* [nd][d_v]) with q*, v* in the stream's dtype."""
    ss = _streams(w.seed)
    gn = np.random.Generator(np.random.PCG64(ss["needle"]))
    nd = w.needles
    T = q.shape[1]
    qs = _cast(_rms_rows(gn.standard_normal((nd, w.d))), w.qv)
    vs = _cast(_rms_rows(gn.standard_normal((nd, w.d_v))), w.qv)
    lim = int(0.9 * T)
    evens = np.arange(0, lim - 1, 2)
    pos = gn.choice(evens, size=3 * nd, replace=False).reshape(nd, 3)
    qpos = gn.choice(np.arange(lim, T), size=nd, replace=False)
    for i in range(nd):
        for p in pos[i]:
            q[0, p] = qs[i]
            v[0, p + 1] = vs[i]
        q[0, qpos[i]] = qs[i]
    return pos, qpos, qs, vs


def gen_layer(w: Workload, B: int | None = None, T: int | None = None, clusters: int = 64, zipf: float = 1.1):
    """Hidden states and slow weights of the layer workload.

    h [B][T][d_model] bf16 bits from `clusters` Gaussian clusters (centres N(0, I),
    cluster weights proportional to j^-zipf, x = centre + 0.1 N(0, I)); RMSNorm gains = 1;
    W_q [d][d_model], W_v [d_v][d_model], w_g [d_model] and W_o [d_model][d_v]
    ([out][in]) as bf16 bits drawn N(0, 1/fan_in); gate bias 0.  The workload itself is
    64 clusters with s = 1.1; fewer clusters or a larger exponent give the hotter
    variants that the skew tests use (same weights, same streams)."""
    B = w.B if B is None else B
    T = w.T if T is None else T
    ss = _streams(w.seed)
    kids = ss["layer"].spawn(6)
    gc = np.random.Generator(np.random.PCG64(kids[0]))
    centres = gc.standard_normal((clusters, w.d_model), dtype=np.float32)
    pz = np.arange(1, clusters + 1, dtype=np.float64) ** -zipf
    pz /= pz.sum()
    ga = np.random.Generator(np.random.PCG64(kids[1]))
    assign = ga.choice(clusters, size=(w.B, w.T), p=pz)[:B, :T]
    gx = np.random.Generator(np.random.PCG64(kids[2]))
    noise = gx.standard_normal((w.B, w.T, w.d_model), dtype=np.float32)[:B, :T]
    hid = f32_to_bf16(centres[assign] + np.float32(0.1) * noise)

    def lin(kid, shape, fan_in):
        x = np.random.Generator(np.random.PCG64(kid)).standard_normal(shape, dtype=np.float32)
        return f32_to_bf16(x * np.float32(1.0 / np.sqrt(fan_in)))

    Wq = lin(kids[3], (w.d, w.d_model), w.d_model)
    Wv = lin(kids[4], (w.d_v, w.d_model), w.d_model)
    kg, ko = kids[5].spawn(2)
    wg = lin(kg, (w.d_model,), w.d_model)
    Wo = lin(ko, (w.d_model, w.d_v), w.d_v)
    return dict(h=np.ascontiguousarray(hid), Wq=Wq, Wv=Wv, wg=wg, Wo=Wo, assign=assign)
