"""CPU oracle for the FwPKM retrieve + chunk-write loop.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``sparse_weight_memory_chunk_b200``) never imports it and shares no code with it.

The arithmetic lives in ``fwpkm_oracle.c`` (plain C, fp64, fp32 state storage);
this module compiles it with gcc and marshals numpy arrays through ctypes.
Function-level citations are in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fwpkm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

KEY_UPDATE = 1
TARGET_NORM = 2
LOOKAHEAD = 4
GATE_WEIGHT = 8
DEFAULT_FLAGS = TARGET_NORM | LOOKAHEAD | GATE_WEIGHT


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.check_call(cmd)
    return _LIB


class Cfg(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int), ("h", ctypes.c_int), ("d_v", ctypes.c_int), ("k", ctypes.c_int),
                ("chunk", ctypes.c_int), ("eps_idw", ctypes.c_double), ("eps_norm", ctypes.c_double),
                ("lr_key", ctypes.c_double), ("flags", ctypes.c_uint)]


def make_cfg(n, d, d_v, k, chunk, eps_idw=1e-3, eps_norm=1e-5, lr_key=1.0, key_update=False,
             target_norm=True, lookahead=True, gate_weight=True) -> Cfg:
    flags = ((KEY_UPDATE if key_update else 0) | (TARGET_NORM if target_norm else 0)
             | (LOOKAHEAD if lookahead else 0) | (GATE_WEIGHT if gate_weight else 0))
    assert d % 2 == 0
    return Cfg(int(n), int(d // 2), int(d_v), int(k), int(chunk), float(eps_idw), float(eps_norm),
               float(lr_key), flags)


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        _lib.orc_subkey_dist.argtypes = [ctypes.POINTER(Cfg), P, P, P]
        _lib.orc_topk_half.argtypes = [ctypes.POINTER(Cfg), P, P]
        _lib.orc_select.argtypes = [ctypes.POINTER(Cfg), P, P, P, P, P, P]
        _lib.orc_read_values.argtypes = [ctypes.POINTER(Cfg), P, P, P, P]
        _lib.orc_target.argtypes = [ctypes.POINTER(Cfg), P, P]
        _lib.orc_chunk.argtypes = [ctypes.POINTER(Cfg), ctypes.c_int] + [P] * 12
        _lib.orc_run_sequence.argtypes = [ctypes.POINTER(Cfg), ctypes.c_int, ctypes.c_int] + [P] * 9
        _lib.orc_chunk_heads.argtypes = [ctypes.POINTER(Cfg), ctypes.c_int, ctypes.c_int] + [P] * 12
        _lib.orc_run_sequence_multi.argtypes = ([ctypes.POINTER(Cfg), ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int] + [P] * 8 + [ctypes.c_int])
        _lib.orc_run_sequence_multi.restype = ctypes.c_int
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a):
    assert a.dtype == np.float32 and a.flags.c_contiguous
    return a


def subkey_dist(cfg: Cfg, qh, K):
    qh = _f64(qh); K = _f32(K)
    D = np.empty(cfg.n, np.float64)
    _load().orc_subkey_dist(ctypes.byref(cfg), _p(qh), _p(K), _p(D))
    return D


def topk_half(cfg: Cfg, D):
    D = _f64(D)
    A = np.empty(cfg.k, np.int32)
    _load().orc_topk_half(ctypes.byref(cfg), _p(D), _p(A))
    return A


def select(cfg: Cfg, D1, D2, forced=None):
    D1 = _f64(D1); D2 = _f64(D2)
    f = None if forced is None else np.ascontiguousarray(forced, dtype=np.int32)
    I = np.empty(cfg.k, np.int32); S = np.empty(cfg.k); w = np.empty(cfg.k)
    _load().orc_select(ctypes.byref(cfg), _p(D1), _p(D2), _p(f), _p(I), _p(S), _p(w))
    return I, S, w


def read_values(cfg: Cfg, I, w, V):
    I = np.ascontiguousarray(I, dtype=np.int32); w = _f64(w); V = _f32(V)
    vhat = np.empty(cfg.d_v)
    _load().orc_read_values(ctypes.byref(cfg), _p(I), _p(w), _p(V), _p(vhat))
    return vhat


def target(cfg: Cfg, u):
    u = _f64(u)
    tau = np.empty(cfg.d_v)
    _load().orc_target(ctypes.byref(cfg), _p(u), _p(tau))
    return tau


def chunk(cfg: Cfg, q, v, g, v_next, K1, K2, V, forced=None, force_mask=None):
    """One chunk of one memory; K1, K2, V (fp32) are updated in place.

    Returns (o [len][d_v] fp64, I [len][k] int32, w [len][k] fp64)."""
    q = _f64(q); v = _f64(v); g = _f64(g)
    vn = None if v_next is None else _f64(v_next)
    length = q.shape[0]
    o = np.empty((length, cfg.d_v)); I = np.empty((length, cfg.k), np.int32)
    w = np.empty((length, cfg.k))
    f = None if forced is None else np.ascontiguousarray(forced, dtype=np.int32)
    fm = None if force_mask is None else np.ascontiguousarray(force_mask, dtype=np.int32)
    _load().orc_chunk(ctypes.byref(cfg), length, _p(q), _p(v), _p(g), _p(vn), _p(_f32(K1)),
                      _p(_f32(K2)), _p(_f32(V)), _p(o), _p(I), _p(w), _p(f), _p(fm))
    return o, I, w


def chunk_heads(cfg: Cfg, q, v, g, v_next, K1, K2, V, forced=None, force_mask=None):
    """One chunk of H heads sharing one value table (fwpkm_oracle.c, orc_chunk_heads).

    q [H][len][d]; v [len][d_v], g [len], v_next [d_v] or None (the sequence's);
    K1, K2 [H][n][h] and V [N][d_v] fp32, updated in place; forced [H][len][k] and
    force_mask [H][len] optional.  Returns (o [len][d_v], I [H][len][k], w [H][len][k])."""
    q = _f64(q); v = _f64(v); g = _f64(g)
    vn = None if v_next is None else _f64(v_next)
    H, length = q.shape[0], q.shape[1]
    o = np.empty((length, cfg.d_v)); I = np.empty((H, length, cfg.k), np.int32)
    w = np.empty((H, length, cfg.k))
    f = None if forced is None else np.ascontiguousarray(forced, dtype=np.int32)
    fm = None if force_mask is None else np.ascontiguousarray(force_mask, dtype=np.int32)
    _load().orc_chunk_heads(ctypes.byref(cfg), H, length, _p(q), _p(v), _p(g), _p(vn), _p(_f32(K1)), _p(_f32(K2)),
                            _p(_f32(V)), _p(o), _p(I), _p(w), _p(f), _p(fm))
    return o, I, w


def run_sequence_heads(cfg: Cfg, q, v, g, K1, K2, V, n_iter=1):
    """A whole sequence of H heads sharing V: chunk after chunk (lookahead v_next = the next
    chunk's first value), n_iter passes.  Returns the final pass's (o, I, w)."""
    q = _f64(q); v = _f64(v); g = _f64(g)
    H, T = q.shape[0], q.shape[1]
    o = np.empty((T, cfg.d_v)); I = np.empty((H, T, cfg.k), np.int32); w = np.empty((H, T, cfg.k))
    for _ in range(n_iter):
        for t0 in range(0, T, cfg.chunk):
            t1 = min(T, t0 + cfg.chunk)
            vn = v[t1] if t1 < T else None
            o[t0:t1], I[:, t0:t1], w[:, t0:t1] = chunk_heads(cfg, q[:, t0:t1], v[t0:t1], g[t0:t1], vn, K1, K2, V)
    return o, I, w


def run_sequence(cfg: Cfg, q, v, g, K1, K2, V, n_iter=1):
    """Whole sequence of one memory; state updated in place.  Returns final-pass (o, I, w)."""
    q = _f64(q); v = _f64(v); g = _f64(g)
    T = q.shape[0]
    o = np.empty((T, cfg.d_v)); I = np.empty((T, cfg.k), np.int32); w = np.empty((T, cfg.k))
    _load().orc_run_sequence(ctypes.byref(cfg), T, n_iter, _p(q), _p(v), _p(g), _p(_f32(K1)),
                             _p(_f32(K2)), _p(_f32(V)), _p(o), _p(I), _p(w))
    return o, I, w


def run_sequence_multi(cfg: Cfg, q, v, g, K1, K2, V, n_iter=1, nthreads=1, with_slots=False):
    """M independent memories ([M][T][..] inputs, [M][..] state) on ``nthreads`` threads
    (with more threads than memories, each memory splits its chunks' read phase over
    nthreads // M threads).

    Returns (o [M][T][d_v], threads used), plus the final pass's slots I [M][T][k] when
    ``with_slots``."""
    q = _f64(q); v = _f64(v); g = _f64(g)
    M, T = q.shape[0], q.shape[1]
    o = np.empty((M, T, cfg.d_v))
    I = np.empty((M, T, cfg.k), np.int32) if with_slots else None
    used = _load().orc_run_sequence_multi(ctypes.byref(cfg), M, T, n_iter, _p(q), _p(v), _p(g),
                                          _p(_f32(K1)), _p(_f32(K2)), _p(_f32(V)), _p(o), _p(I), nthreads)
    return (o, used, I) if with_slots else (o, used)
