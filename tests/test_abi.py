"""The C ABI library builds for sm_100a, loads without a GPU and exports every entry
point that include/fwpkm.h declares.  Only host-side calls are made (no kernels)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sparse_weight_memory_chunk_b200 import build, fwpkm
    build.build()
    return fwpkm


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(fwpkm_\w+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    so = ctypes.CDLL(lib.LIB_PATH)
    missing = [n for n in names if not hasattr(so, n)]
    assert not missing, missing


def test_library_is_built_for_sm100a(lib):
    data = open(lib.LIB_PATH, "rb").read()
    assert b"sm_100a" in data


def test_status_strings(lib):
    assert lib.status_string(0) == "ok"
    assert lib.status_string(-3) == "workspace too small"
    assert lib.status_string(-5) == "device wait timed out"
    assert lib.status_string(lib.ERR_BAD_SLOT) == "slot index out of range in the write"


def test_run_layer_scratch_and_checks(lib):
    import ctypes as C
    cfg = lib.make_config(n=512, d=256, d_v=256, k=32, chunk=256, num_mem=16, bf16=True, key_update=True)
    rows = 16 * 4096
    # q, v (bf16), g, o (fp32), each part on a 256-byte boundary
    assert lib.run_layer_scratch_size(cfg, 4096) == 2 * rows * 256 * 2 + rows * 4 + rows * 256 * 4
    so = lib.lib()
    fake = C.c_void_p(1 << 20)
    assert so.fwpkm_run_layer(None, None, fake, 16, 1, fake, 1 << 30, fake, None) == lib.ERR_INVALID_ARG
    with pytest.raises(lib.FwpkmError):
        lib.run_layer_scratch_size(cfg, -1)
    lib.test_stall_waits(0)  # the timeout test hook is host-side state only


def test_workspace_size_and_validation(lib):
    cfg = lib.make_config(n=1024, d=256, d_v=256, k=32, chunk=256, num_mem=8, bf16=True, key_update=True)
    ws = lib.workspace_size(cfg, 4096)
    # idx + w + per-half survivors + pair lists dominate: O(M T k) + the chunk distance rows
    assert 8 * 4096 * 32 * 4 * 6 < ws < 128 << 20
    bad = [dict(k=33), dict(k=0), dict(n=16, k=32), dict(d=7), dict(d_v=6), dict(chunk=2048),
           dict(num_mem=0), dict(n=8192)]
    for over in bad:
        c = dict(n=1024, d=256, d_v=256, k=32, chunk=256, num_mem=8, bf16=True)
        c.update(over)
        with pytest.raises(lib.FwpkmError) as e:
            lib.workspace_size(lib.make_config(**c), 4096)
        assert e.value.status in (lib.ERR_INVALID_ARG, lib.ERR_UNSUPPORTED)
    with pytest.raises(lib.FwpkmError):
        lib.workspace_size(cfg, 0)


def test_launch_counter_starts_at_zero(lib):
    assert lib.launch_count() == 0


def test_layer_workspace_size_and_validation(lib):
    import ctypes as C
    so = lib.lib()
    out = C.c_size_t(0)
    cfg = lib.LayerConfig(2048, 256, 256, 65536, 1e-6, 0)
    assert so.fwpkm_layer_workspace_size(C.byref(cfg), C.byref(out)) == lib.OK
    # three bf16 pieces of both weight matrices + the per-row scratch of the output call
    pieces = 2 * 3 * (512 * 2048 + 2048 * 256)
    scratch = 4 * 65536 + 2 * 2 * 65536 * 256
    assert pieces + scratch <= out.value < pieces + scratch + (1 << 20)
    for bad, want in [((2048, 256, 256, 0, 1e-6), lib.ERR_INVALID_ARG), ((2000, 256, 256, 16, 1e-6), lib.ERR_UNSUPPORTED),
                      ((2048, 48, 256, 16, 1e-6), lib.ERR_UNSUPPORTED), ((2048, 256, 96, 16, 1e-6), lib.ERR_UNSUPPORTED),
                      ((2048, 256, 256, 16, -1.0), lib.ERR_INVALID_ARG)]:
        c = lib.LayerConfig(*bad, 0)
        assert so.fwpkm_layer_workspace_size(C.byref(c), C.byref(out)) == want, bad
    assert so.fwpkm_layer_workspace_size(C.byref(cfg), None) == lib.ERR_INVALID_ARG
    c = lib.LayerConfig(2048, 256, 256, 16, 1e-6, 7)
    assert so.fwpkm_layer_workspace_size(C.byref(c), C.byref(out)) == lib.ERR_INVALID_ARG


def test_metrics_workspace_size_and_validation(lib):
    import ctypes as C
    so = lib.lib()
    N = 1024 * 1024
    # one window per memory: 8 windows of N 32-bit counters, plus 8 KiB of partials per window
    ws = lib.metrics_workspace_size(8, 4096, N, 32768)
    assert 8 * N * 4 <= ws < 8 * N * 4 + (1 << 17)
    # at most 32 windows at once, however long the sequence
    assert lib.metrics_workspace_size(8, 1 << 22, N, 32768) < 33 * N * 4
    out = C.c_size_t(0)
    for args in [(0, 16, 64, 8), (1, -1, 64, 8), (1, 16, 0, 8), (1, 16, 64, 0)]:
        assert so.fwpkm_metrics_workspace_size(*args, C.byref(out)) == lib.ERR_INVALID_ARG
    fake = C.c_void_p(1 << 20)  # aligned, never dereferenced: every call below returns before any launch
    assert so.fwpkm_addressing_metrics(fake, 1, 0, 4, 64, 8, fake, 0, fake, None, None) == lib.OK  # T = 0
    assert so.fwpkm_addressing_metrics(None, 1, 16, 4, 64, 8, fake, 1 << 20, fake, None, None) == lib.ERR_INVALID_ARG
    assert so.fwpkm_addressing_metrics(fake, 1, 16, 0, 64, 8, fake, 1 << 20, fake, None, None) == lib.ERR_INVALID_ARG
    assert so.fwpkm_addressing_metrics(fake, 1, 16, 4, 64, 8, C.c_void_p((1 << 20) + 16), 1 << 20, fake, None,
                                       None) == lib.ERR_INVALID_ARG  # workspace not 256-byte aligned
    assert so.fwpkm_addressing_metrics(fake, 1, 16, 4, 64, 8, fake, 64, fake, None, None) == lib.ERR_WORKSPACE


def test_metrics_binding_checks_given_outputs(lib):
    import torch
    idx = torch.zeros(2, 10, 4, dtype=torch.int32)
    bad = (torch.zeros(2, 1, 3, dtype=torch.float32), torch.zeros(2, 1, 4, dtype=torch.int64))
    with pytest.raises(ValueError):
        lib.addressing_metrics(idx, 64, 16, workspace=torch.zeros(1), out=bad)
    bad = (torch.zeros(2, 2, 3, dtype=torch.float64), torch.zeros(2, 2, 4, dtype=torch.int64))  # W = 1
    with pytest.raises(ValueError):
        lib.addressing_metrics(idx, 64, 16, workspace=torch.zeros(1), out=bad)
