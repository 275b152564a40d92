"""fwpkm_run_sequence_host (page-locked host q, v, g in; host o out; copies overlapped with
the compute chunk by chunk) against fwpkm_run_sequence on the same inputs already on the
device: o, V, K1, K2 bit-for-bit, on every schedule the call can take (tensor-core key
update, frozen keys over several addressing windows with the value loop, CUDA-core
scoring), with two passes, and the argument checks (pageable host memory, short scratch).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import Workload, gen_keys, gen_qvg, gen_values  # noqa: E402

from parity import to_device  # noqa: E402

# name: (n, d, dv, k, C, M, T, qv, key_update)
CASES = {
    "key_update_tc": (256, 128, 128, 16, 128, 2, 300, "bf16", True),
    "frozen_windows": (1024, 256, 64, 8, 256, 8, 2600, "bf16", False),  # 1024-token windows
    "simt_f32": (64, 64, 64, 8, 64, 2, 250, "f32", True),
}


def setup(name):
    n, d, dv, k, C, M, T, qv, ku = CASES[name]
    w = Workload(name, n, d, dv, k, T, C, M, 1, qv, ku, 5, "sigmoid", "normal002")
    q, v, g = gen_qvg(w)
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, m) for m in range(M)])
    cfg = fwpkm.make_config(n, d, dv, k, C, M, qv == "bf16", lr_key=10.0, key_update=ku)
    return w, (q, v, g, K1, K2, V), cfg


def state(w, data, cfg):
    q, v, g, K1, K2, V = data
    dev = dict(K1=torch.from_numpy(K1).cuda(), K2=torch.from_numpy(K2).cuda(), V=torch.from_numpy(V).cuda())
    return fwpkm.State(cfg, dev["K1"], dev["K2"], dev["V"], w.T), dev


@pytest.mark.parametrize("n_iter", [1, 2])
@pytest.mark.parametrize("name", list(CASES))
def test_host_buffers_match_device_buffers(name, n_iter):
    w, data, cfg = setup(name)
    q, v, g = data[:3]
    qd, vd, gd = to_device(q, w.qv, torch), to_device(v, w.qv, torch), torch.from_numpy(g).cuda()
    st_a, dev_a = state(w, data, cfg)
    o_a = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st_a.run_sequence(qd, vd, gd, o_a, n_iter=n_iter)
    st_a.sync()

    qh, vh, gh = (x.cpu().pin_memory() for x in (qd, vd, gd))
    oh = torch.full((w.M, w.T, w.d_v), float("nan")).pin_memory()
    st_b, dev_b = state(w, data, cfg)
    scratch = st_b.run_sequence_host(qh, vh, gh, oh, n_iter=n_iter)
    st_b.sync()
    torch.cuda.synchronize()
    assert torch.equal(oh, o_a.cpu()), f"{name}: host-buffer o differs"
    for key in ("V", "K1", "K2"):
        assert torch.equal(dev_b[key], dev_a[key]), f"{name}: host-buffer {key} differs"
    # a second call reuses the cached graph and the scratch: same result from the new state
    st_b2, dev_b2 = state(w, data, cfg)
    oh2 = torch.zeros_like(oh).pin_memory()
    st_b2.run_sequence_host(qh, vh, gh, oh2, n_iter=n_iter, scratch=scratch)
    st_b2.sync()
    torch.cuda.synchronize()
    assert torch.equal(oh2, oh) and torch.equal(dev_b2["V"], dev_a["V"])


def test_host_buffers_heads_sharing_v():
    """Heads sharing one value table: q per memory, v, g, o per sequence, copied through the
    host-buffer call; bits of fwpkm_run_sequence on the same inputs."""
    n, d, dv, k, C, B, H, T = 256, 128, 64, 8, 128, 2, 2, 300
    for ku in (True, False):
        w = Workload("heads_io", n, d, dv, k, T, C, B * H, 1, "bf16", ku, 9, "sigmoid", "normal002")
        q, v_all, g_all = gen_qvg(w)
        v, g = np.ascontiguousarray(v_all[:B]), np.ascontiguousarray(g_all[:B])
        K1, K2 = gen_keys(w)
        V = np.stack([gen_values(w, b) for b in range(B)])
        cfg = fwpkm.make_config(n, d, dv, k, C, B * H, True, key_update=ku, v_heads=H)
        qd, vd, gd = to_device(q, "bf16", torch), to_device(v, "bf16", torch), torch.from_numpy(g).cuda()
        outs = []
        for host in (False, True):
            K1d, K2d, Vd = (torch.from_numpy(x).cuda() for x in (K1, K2, V))
            st = fwpkm.State(cfg, K1d, K2d, Vd, T)
            if host:
                # the host buffers must outlive the asynchronous copies: keep references
                qh, vh, gh = qd.cpu().pin_memory(), vd.cpu().pin_memory(), gd.cpu().pin_memory()
                o = torch.zeros(B, T, dv).pin_memory()
                st.run_sequence_host(qh, vh, gh, o)
            else:
                o = torch.zeros(B, T, dv, device="cuda")
                st.run_sequence(qd, vd, gd, o)
            st.sync()
            torch.cuda.synchronize()
            outs.append((o.cpu(), Vd.cpu(), K1d.cpu()))
        assert all(torch.equal(a, b) for a, b in zip(*outs)), f"heads, key update {ku}: host-buffer call differs"


def test_host_buffer_argument_checks():
    w, data, cfg = setup("key_update_tc")
    q, v, g = data[:3]
    st, _ = state(w, data, cfg)
    qd = to_device(q, w.qv, torch)
    qh, vh = qd.cpu().pin_memory(), to_device(v, w.qv, torch).cpu().pin_memory()
    gh = torch.from_numpy(g).pin_memory()
    oh = torch.zeros(w.M, w.T, w.d_v).pin_memory()
    with pytest.raises(fwpkm.FwpkmError) as e:  # pageable host memory
        st.run_sequence_host(qd.cpu(), vh, gh, oh)
    assert e.value.status == fwpkm.ERR_INVALID_ARG
    with pytest.raises(fwpkm.FwpkmError) as e:  # device memory where host memory is expected
        st.run_sequence_host(qd, vh, gh, oh)
    assert e.value.status == fwpkm.ERR_INVALID_ARG
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(fwpkm.FwpkmError) as e:
        st.run_sequence_host(qh, vh, gh, oh, scratch=small)
    assert e.value.status == fwpkm.ERR_WORKSPACE
    assert fwpkm.run_sequence_host_scratch_size(cfg, w.T) >= 2 * w.M * w.T * (w.d + w.d_v) + 4 * w.M * w.T * w.d_v
