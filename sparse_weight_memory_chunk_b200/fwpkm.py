"""Thin ctypes binding of ``libfwpkm.so`` (declared in ``include/fwpkm.h``).

Argument marshalling only: every step of the FwPKM hot path runs in the library's
CUDA kernels.  Functions keep the C names without the ``fwpkm_`` prefix; device
buffers are passed as torch tensors (their ``data_ptr``) and streams as
``torch.cuda.Stream`` (default: the current stream).  A non-OK status raises
``FwpkmError``.  If the library is missing, loading raises instead of falling back
to anything else.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfwpkm.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_STATE, ERR_BAD_SLOT = \
    0, -1, -2, -3, -4, -5, -6, -7
F32, BF16 = 0, 1
KEY_UPDATE, TARGET_NORM, LOOKAHEAD, GATE_WEIGHT = 1, 2, 4, 8
DEFAULT_FLAGS = TARGET_NORM | LOOKAHEAD | GATE_WEIGHT
KIND = {"gather": 1, "write": 2, "score": 3, "cartesian": 4, "sort": 5, "address": 6, "other": 7, "topk": 8,
        "prep": 9, "pbar": 10, "wbuild": 11, "fused": 12, "value_loop": 13, "all": 100}
KIND_NAME = {v: k for k, v in KIND.items()}


class FwpkmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class Config(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int), ("d", ctypes.c_int), ("d_v", ctypes.c_int), ("k", ctypes.c_int),
                ("chunk", ctypes.c_int), ("num_mem", ctypes.c_int), ("qv_dtype", ctypes.c_int),
                ("eps_idw", ctypes.c_float), ("eps_norm", ctypes.c_float), ("lr_key", ctypes.c_float),
                ("flags", ctypes.c_uint), ("v_heads", ctypes.c_int)]


def make_config(n, d, d_v, k, chunk, num_mem, bf16, eps_idw=1e-3, eps_norm=1e-5, lr_key=1.0,
                key_update=False, target_norm=True, lookahead=True, gate_weight=True, v_heads=1) -> Config:
    flags = ((KEY_UPDATE if key_update else 0) | (TARGET_NORM if target_norm else 0)
             | (LOOKAHEAD if lookahead else 0) | (GATE_WEIGHT if gate_weight else 0))
    return Config(n, d, d_v, k, chunk, num_mem, BF16 if bf16 else F32, eps_idw, eps_norm, lr_key, flags, v_heads)


_lib = None
_P = ctypes.c_void_p


class LayerConfig(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("d", ctypes.c_int), ("d_v", ctypes.c_int), ("max_rows", ctypes.c_int),
                ("eps_rms", ctypes.c_float), ("qv_dtype", ctypes.c_int)]


class LayerParams(ctypes.Structure):
    _fields_ = [("W_q", _P), ("gamma_q", _P), ("b_q", _P),
                ("W_v", _P), ("gamma_v", _P), ("b_v", _P),
                ("w_g", _P), ("gamma_g", _P), ("b_g", ctypes.c_float),
                ("W_o", _P), ("gamma_o", _P), ("b_o", _P)]


def lib():
    """Load libfwpkm.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python sparse_weight_memory_chunk_b200/build.py`")
        L = ctypes.CDLL(LIB_PATH)
        C = ctypes.POINTER(Config)
        sig = {
            "fwpkm_workspace_size": ([C, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "fwpkm_init_state": ([C, _P, _P, _P, ctypes.c_int, _P, ctypes.c_size_t, ctypes.POINTER(_P)],
                                 ctypes.c_int),
            "fwpkm_forward_chunk": ([_P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P], ctypes.c_int),
            "fwpkm_write_chunk": ([_P, _P, _P], ctypes.c_int),
            "fwpkm_run_sequence": ([_P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P], ctypes.c_int),
            "fwpkm_read_backward": ([C, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P],
                                    ctypes.c_int),
            "fwpkm_run_sequence_host_scratch_size": ([C, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)],
                                                     ctypes.c_int),
            "fwpkm_run_sequence_host": ([_P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P, ctypes.c_size_t, _P],
                                        ctypes.c_int),
            "fwpkm_last_addressing": ([_P, ctypes.c_int, _P, _P, _P], ctypes.c_int),
            "fwpkm_chunk_step_noalloc": ([C, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P],
                                         ctypes.c_int),
            "fwpkm_stream_tokens": ([_P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P], ctypes.c_int),
            "fwpkm_stream_flush": ([_P, _P], ctypes.c_int),
            "fwpkm_stream_pending": ([_P, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
            "fwpkm_sync": ([_P, _P], ctypes.c_int),
            "fwpkm_destroy_state": ([_P], None),
            "fwpkm_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "fwpkm_launch_count": ([], ctypes.c_uint64),
            "fwpkm_profile_kernel": ([_P, ctypes.c_int], ctypes.c_int),
            "fwpkm_kernel_time": ([_P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)],
                                  ctypes.c_int),
            "fwpkm_kernel_timeline": ([_P, ctypes.c_int, _P, _P, _P, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
            "fwpkm_layer_workspace_size": ([ctypes.POINTER(LayerConfig), ctypes.POINTER(ctypes.c_size_t)],
                                           ctypes.c_int),
            "fwpkm_layer_init": ([ctypes.POINTER(LayerConfig), _P, ctypes.c_size_t, ctypes.POINTER(_P)],
                                 ctypes.c_int),
            "fwpkm_layer_set_params": ([_P, ctypes.POINTER(LayerParams), _P], ctypes.c_int),
            "fwpkm_layer_in": ([_P, _P, ctypes.c_int, _P, _P, _P, _P], ctypes.c_int),
            "fwpkm_layer_out": ([_P, _P, ctypes.c_int, _P, _P], ctypes.c_int),
            "fwpkm_layer_sync": ([_P, _P], ctypes.c_int),
            "fwpkm_layer_destroy": ([_P], None),
            "fwpkm_run_layer_scratch_size": ([C, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "fwpkm_run_layer": ([_P, _P, _P, ctypes.c_int, ctypes.c_int, _P, ctypes.c_size_t, _P, _P], ctypes.c_int),
            "fwpkm_test_stall_waits": ([ctypes.c_int], None),
            "fwpkm_metrics_workspace_size": ([ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "fwpkm_addressing_metrics": ([_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          _P, ctypes.c_size_t, _P, _P, _P], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != OK:
        raise FwpkmError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def status_string(status: int) -> str:
    return lib().fwpkm_status_string(status).decode()


def launch_count() -> int:
    return int(lib().fwpkm_launch_count())


def test_stall_waits(n_launches: int):
    """Test hook: the next n tensor-core launches wait once on a barrier that nothing
    completes, so their bounded wait runs out (no fault; see include/fwpkm.h)."""
    lib().fwpkm_test_stall_waits(int(n_launches))


def run_layer_scratch_size(cfg: Config, T: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().fwpkm_run_layer_scratch_size(ctypes.byref(cfg), T, ctypes.byref(out)), "run_layer_scratch_size")
    return out.value


def read_backward(cfg: Config, K1, K2, V, q, v, g, idx, d_o, dq, dv, dg, len_=None, seq_stride=None, stream=None):
    """fwpkm_read_backward: dq, dv, dg (fp32, the q, v, g layouts) from d_o for the tokens
    whose slots `idx` ([M][len][k]) the forward read with the state K1, K2, V."""
    len_ = idx.shape[1] if len_ is None else len_
    seq_stride = q.shape[1] if seq_stride is None else seq_stride
    _check(lib().fwpkm_read_backward(ctypes.byref(cfg), _ptr(K1), _ptr(K2), _ptr(V), _ptr(q), _ptr(v), _ptr(g),
                                     _ptr(idx), _ptr(d_o), len_, seq_stride, _ptr(dq), _ptr(dv), _ptr(dg),
                                     _stream(stream)), "read_backward")


def run_sequence_host_scratch_size(cfg: Config, T: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().fwpkm_run_sequence_host_scratch_size(ctypes.byref(cfg), T, ctypes.byref(out)),
           "run_sequence_host_scratch_size")
    return out.value


def run_layer_parts(cfg: Config, T: int, scratch):
    """Views of the q, v, g, o that fwpkm_run_layer leaves in `scratch` (a uint8 tensor)."""
    import torch
    M, d, dv = cfg.num_mem, cfg.d, cfg.d_v
    es = 2 if cfg.qv_dtype == BF16 else 4
    qdt = torch.bfloat16 if cfg.qv_dtype == BF16 else torch.float32
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    sizes = [es * M * T * d, es * M * T * dv, 4 * M * T, 4 * M * T * dv]
    offs, o = [], 0
    for b in sizes:
        offs.append(o)
        o = al(o + b)
    q = scratch[offs[0]:offs[0] + sizes[0]].view(qdt).view(M, T, d)
    v = scratch[offs[1]:offs[1] + sizes[1]].view(qdt).view(M, T, dv)
    g = scratch[offs[2]:offs[2] + sizes[2]].view(torch.float32).view(M, T)
    ob = scratch[offs[3]:offs[3] + sizes[3]].view(torch.float32).view(M, T, dv)
    return q, v, g, ob


def workspace_size(cfg: Config, max_T: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().fwpkm_workspace_size(ctypes.byref(cfg), max_T, ctypes.byref(out)), "workspace_size")
    return out.value


def chunk_step_noalloc(cfg: Config, K1, K2, V, q, v, g, o, c_len, seq_stride=None, v_next=None,
                       stream=None):
    """One chunk step (read + write + key step) with no workspace and no allocation."""
    seq_stride = c_len if seq_stride is None else seq_stride
    _check(lib().fwpkm_chunk_step_noalloc(ctypes.byref(cfg), _ptr(K1), _ptr(K2), _ptr(V), _ptr(q), _ptr(v),
                                          _ptr(g), _ptr(v_next), c_len, seq_stride, _ptr(o), _stream(stream)),
           "chunk_step_noalloc")


def metrics_workspace_size(num_mem: int, T: int, N: int, window: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().fwpkm_metrics_workspace_size(num_mem, T, N, window, ctypes.byref(out)), "metrics_workspace_size")
    return out.value


def addressing_metrics(idx, N: int, window: int = 32768, workspace=None, stream=None, out=None):
    """Addressing metrics of selections idx (int32 CUDA tensor [M][T][k]) per window of tokens.

    Returns (metrics fp64 [M][W][3]: coverage, collision rate, KLD; counts int64 [M][W][4]:
    rows accessed, accesses, competitive accesses, invalid entries), W = ceil(T / window);
    `out` = (metrics, counts) tensors of those shapes to fill instead of new ones.
    """
    import torch
    M, T, k = idx.shape
    W = (T + window - 1) // window
    if out is None:
        met = torch.zeros(M, W, 3, dtype=torch.float64, device=idx.device)
        cnt = torch.zeros(M, W, 4, dtype=torch.int64, device=idx.device)
    else:
        met, cnt = out
        if tuple(met.shape) != (M, W, 3) or tuple(cnt.shape) != (M, W, 4) or met.dtype != torch.float64 \
                or cnt.dtype != torch.int64 or not (met.is_contiguous() and cnt.is_contiguous()):
            raise ValueError("out must be contiguous fp64 [M][W][3] and int64 [M][W][4] tensors")
    if workspace is None:
        workspace = torch.empty(metrics_workspace_size(M, T, N, window), dtype=torch.uint8, device=idx.device)
    _check(lib().fwpkm_addressing_metrics(_ptr(idx), M, T, k, N, window, _ptr(workspace), workspace.numel(),
                                          _ptr(met), _ptr(cnt), _stream(stream)), "addressing_metrics")
    return met, cnt


class State:
    """A handle from ``fwpkm_init_state``; keeps the caller's tensors alive."""

    def __init__(self, cfg: Config, K1, K2, V, max_T: int, workspace=None):
        import torch
        self.cfg = cfg
        self.max_T = max_T
        nbytes = workspace_size(cfg, max_T)
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=V.device)
        for t in (K1, K2, V):
            assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
        self.K1, self.K2, self.V, self.workspace = K1, K2, V, workspace
        h = _P()
        _check(lib().fwpkm_init_state(ctypes.byref(cfg), _ptr(K1), _ptr(K2), _ptr(V), max_T,
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      ctypes.byref(h)), "init_state")
        self.handle = h
        self._pending = None

    def forward_chunk(self, q, v, g, o, c_len, seq_stride=None, idx_out=None, w_out=None, stream=None):
        seq_stride = c_len if seq_stride is None else seq_stride
        self._pending = (q, v, g)
        _check(lib().fwpkm_forward_chunk(self.handle, _ptr(q), _ptr(v), _ptr(g), c_len, seq_stride, _ptr(o),
                                         _ptr(idx_out), _ptr(w_out), _stream(stream)), "forward_chunk")

    def write_chunk(self, v_next=None, stream=None):
        _check(lib().fwpkm_write_chunk(self.handle, _ptr(v_next), _stream(stream)), "write_chunk")
        self._pending = None

    def run_sequence(self, q, v, g, o, T=None, n_iter=1, stream=None):
        T = q.shape[1] if T is None else T
        _check(lib().fwpkm_run_sequence(self.handle, _ptr(q), _ptr(v), _ptr(g), T, n_iter, _ptr(o),
                                        _stream(stream)), "run_sequence")

    def run_sequence_host(self, q, v, g, o, T=None, n_iter=1, scratch=None, stream=None):
        """run_sequence on page-locked HOST tensors q, v, g, o (copies overlap the compute);
        `scratch`: a device uint8 tensor of run_sequence_host_scratch_size bytes (made here if
        None).  Returns the scratch so that repeated calls can reuse it."""
        import torch
        T = q.shape[1] if T is None else T
        if scratch is None:
            scratch = torch.empty(run_sequence_host_scratch_size(self.cfg, T), dtype=torch.uint8, device="cuda")
        _check(lib().fwpkm_run_sequence_host(self.handle, _ptr(q), _ptr(v), _ptr(g), T, n_iter, _ptr(o),
                                             _ptr(scratch), scratch.numel(), _stream(stream)), "run_sequence_host")
        return scratch

    def stream_tokens(self, q, v, g, o, n_tok=None, seq_stride=None, stream=None):
        """Read n_tok new tokens of every memory ([M][seq_stride][..] rows); writes o for them."""
        n_tok = q.shape[1] if n_tok is None else n_tok
        seq_stride = q.shape[1] if seq_stride is None else seq_stride
        _check(lib().fwpkm_stream_tokens(self.handle, _ptr(q), _ptr(v), _ptr(g), n_tok, seq_stride, _ptr(o),
                                         _stream(stream)), "stream_tokens")

    def stream_flush(self, stream=None):
        """Write the pending tokens of a token-at-a-time sequence (no lookahead for the last)."""
        _check(lib().fwpkm_stream_flush(self.handle, _stream(stream)), "stream_flush")

    def stream_pending(self) -> int:
        """Tokens read by stream_tokens and not yet written (host-side count)."""
        n = ctypes.c_int(0)
        _check(lib().fwpkm_stream_pending(self.handle, ctypes.byref(n)), "stream_pending")
        return n.value

    def last_addressing(self, T, idx_out=None, w_out=None, stream=None):
        _check(lib().fwpkm_last_addressing(self.handle, T, _ptr(idx_out), _ptr(w_out), _stream(stream)),
               "last_addressing")

    def sync(self, stream=None):
        _check(lib().fwpkm_sync(self.handle, _stream(stream)), "sync")

    def profile_kernel(self, kind):
        kind = KIND.get(kind, kind) if isinstance(kind, str) else kind
        _check(lib().fwpkm_profile_kernel(self.handle, int(kind)), "profile_kernel")

    def kernel_timeline(self, max_launches=4096):
        """[(kind name, start ms, end ms)] of the launches timed in the last call."""
        import numpy as np
        kinds = np.zeros(max_launches, dtype=np.int32)
        t0 = np.zeros(max_launches, dtype=np.float32)
        t1 = np.zeros(max_launches, dtype=np.float32)
        n = ctypes.c_int(0)
        _check(lib().fwpkm_kernel_timeline(self.handle, max_launches, kinds.ctypes.data_as(_P), t0.ctypes.data_as(_P),
                                           t1.ctypes.data_as(_P), ctypes.byref(n)), "kernel_timeline")
        m = min(n.value, max_launches)
        return [(KIND_NAME.get(int(kinds[i]), str(int(kinds[i]))), float(t0[i]), float(t1[i])) for i in range(m)]

    def kernel_time(self):
        ms = ctypes.c_double(0.0)
        n = ctypes.c_int(0)
        _check(lib().fwpkm_kernel_time(self.handle, ctypes.byref(ms), ctypes.byref(n)), "kernel_time")
        return ms.value, n.value

    def destroy(self):
        if getattr(self, "handle", None):
            lib().fwpkm_destroy_state(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


class Layer:
    """A handle from ``fwpkm_layer_init``: the slow-weight projections (method steps 1
    and 3).  Weights are bf16 tensors [out][in]; norm weights and biases fp32 (None:
    ones / zeros)."""

    def __init__(self, d_model, d, d_v, max_rows, eps_rms=1e-6, qv_bf16=False, device="cuda"):
        import torch
        self.cfg = LayerConfig(d_model, d, d_v, max_rows, eps_rms, BF16 if qv_bf16 else F32)
        out = ctypes.c_size_t(0)
        _check(lib().fwpkm_layer_workspace_size(ctypes.byref(self.cfg), ctypes.byref(out)), "layer_workspace_size")
        self.workspace = torch.empty(out.value, dtype=torch.uint8, device=device)
        h = _P()
        _check(lib().fwpkm_layer_init(ctypes.byref(self.cfg), _ptr(self.workspace), out.value, ctypes.byref(h)),
               "layer_init")
        self.handle = h

    def set_params(self, W_q, W_v, w_g, W_o, gamma_q=None, gamma_v=None, gamma_g=None, gamma_o=None,
                   b_q=None, b_v=None, b_g=0.0, b_o=None, stream=None):
        p = LayerParams(_ptr(W_q), _ptr(gamma_q), _ptr(b_q), _ptr(W_v), _ptr(gamma_v), _ptr(b_v),
                        _ptr(w_g), _ptr(gamma_g), float(b_g), _ptr(W_o), _ptr(gamma_o), _ptr(b_o))
        _check(lib().fwpkm_layer_set_params(self.handle, ctypes.byref(p), _stream(stream)), "layer_set_params")

    def project_in(self, h, q, v, g, rows=None, stream=None):
        rows = h.shape[0] if rows is None else rows
        _check(lib().fwpkm_layer_in(self.handle, _ptr(h), rows, _ptr(q), _ptr(v), _ptr(g), _stream(stream)),
               "layer_in")

    def project_out(self, o, o_out, rows=None, stream=None):
        rows = o.shape[0] if rows is None else rows
        _check(lib().fwpkm_layer_out(self.handle, _ptr(o), rows, _ptr(o_out), _stream(stream)), "layer_out")

    def sync(self, stream=None):
        _check(lib().fwpkm_layer_sync(self.handle, _stream(stream)), "layer_sync")

    def run_layer(self, state, h, o_out, T=None, n_iter=1, scratch=None, stream=None):
        """fwpkm_run_layer: h [M][T][d_model] bf16 -> o_out [M][T][d_model] bf16 through the
        projections and the memory `state`.  Returns the scratch tensor (see run_layer_parts)."""
        import torch
        T = h.shape[1] if T is None else T
        if scratch is None:
            scratch = torch.empty(run_layer_scratch_size(state.cfg, T), dtype=torch.uint8, device=h.device)
        _check(lib().fwpkm_run_layer(self.handle, state.handle, _ptr(h), T, n_iter, _ptr(scratch), scratch.numel(),
                                     _ptr(o_out), _stream(stream)), "run_layer")
        return scratch

    def destroy(self):
        if getattr(self, "handle", None):
            lib().fwpkm_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass
