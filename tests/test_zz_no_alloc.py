"""The allocation-free chunk step gives the same results as the workspace entry points.

fwpkm_chunk_step_noalloc exists for callers that cannot allocate device memory; it
keeps its scratch in a fixed array inside the library.  Two chunk steps in a row
through it must match fwpkm_forward_chunk + fwpkm_write_chunk on the same inputs
(outputs, values and keys), within the parity tolerance.  This file is collected
last on purpose, and must pass both alone and after every other test.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import Workload, gen_keys, gen_qvg, gen_values  # noqa: E402

RTOL, ATOL = 1e-4, 1e-5


def close(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return bool(((a - b).abs() <= ATOL + RTOL * b.abs()).all())


@pytest.mark.parametrize("qv,key_update,shape", [("f32", True, (64, 64, 64, 8, 64, 2)),
                                                  ("bf16", False, (256, 128, 128, 16, 128, 2)),
                                                  ("bf16", True, (64, 128, 64, 8, 32, 2))])
def test_noalloc_chunk_steps_match_workspace_entry_points(qv, key_update, shape):
    # the last case: bf16 queries with the key step, which this entry point runs on the
    # CUDA-core kernels while the workspace entry points take the tensor-core path
    n, d, dv, k, C, M = shape
    T = 2 * C
    w = Workload("noalloc", n, d, dv, k, T + 1, C, M, 1, qv, key_update, 21, "sigmoid", "normal002")
    q, v, g = gen_qvg(w)
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, m) for m in range(M)])

    def dev(x):
        t = torch.from_numpy(np.ascontiguousarray(x.view(np.int16) if x.dtype == np.uint16 else x)).cuda()
        return t.view(torch.bfloat16) if x.dtype == np.uint16 else t

    qd, vd, gd = dev(q), dev(v), dev(g)
    cfg = fwpkm.make_config(n, d, dv, k, C, M, qv == "bf16", key_update=key_update, lr_key=10.0)
    a = [dev(K1), dev(K2), dev(V)]
    b = [dev(K1), dev(K2), dev(V)]
    st = fwpkm.State(cfg, b[0], b[1], b[2], C)
    Tp = w.T
    oa = torch.zeros(M, Tp, dv, device="cuda")
    ob = torch.zeros(M, Tp, dv, device="cuda")
    for t0 in (0, C):  # two calls in a row; the second starts from the first one's state
        fwpkm.chunk_step_noalloc(cfg, a[0], a[1], a[2], qd[:, t0:], vd[:, t0:], gd[:, t0:], oa[:, t0:], C,
                                 seq_stride=Tp, v_next=vd[:, t0 + C])
        st.forward_chunk(qd[:, t0:], vd[:, t0:], gd[:, t0:], ob[:, t0:], C, seq_stride=Tp)
        st.write_chunk(vd[:, t0 + C])
        torch.cuda.synchronize()
        assert close(oa[:, t0:t0 + C], ob[:, t0:t0 + C]), f"o differs after the call at token {t0}"
        for x, y, name in zip(a, b, ("K1", "K2", "V")):
            assert close(x, y), f"{name} differs after the call at token {t0}"
    assert not torch.equal(a[2], dev(V)), "the memory was not written"
    st.destroy()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    cfg = fwpkm.make_config(1024, 256, 256, 32, 256, 8, True, key_update=True)  # ~20 MiB of scratch
    z = torch.zeros(16, device="cuda")
    with pytest.raises(fwpkm.FwpkmError) as e:
        fwpkm.chunk_step_noalloc(cfg, z, z, z, z, z, z, z, 256)
    assert e.value.status == fwpkm.ERR_UNSUPPORTED
