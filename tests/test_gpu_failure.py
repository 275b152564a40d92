"""Failure detection on the GPU without a fault: a bounded device-side wait is made to run
out, and the error must come back through the C ABI with the context still usable.

fwpkm_test_stall_waits(1) makes the next tensor-core launch wait on a barrier that
nothing completes.  Its wait is bounded like every wait in those kernels, so it gives up
after 0.2 s: the kernel drains its in-flight copies, frees its tensor memory and latches
FWPKM_ERR_TIMEOUT.  The test checks that
  * a later call on the same handle sees the latched error (through the host copy of the
    status word) and enqueues nothing;
  * fwpkm_sync / fwpkm_layer_sync return it and clear it;
  * the next chunk on the same state runs cleanly and matches the oracle (tensor memory
    was released: another tensor-core launch on every SM allocates it again).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import WORKLOADS, gen_layer  # noqa: E402

from parity import as_f64, assert_close, oracle_chunk_against_gpu  # noqa: E402
from test_gpu_layer import bf16_dev  # noqa: E402
from test_gpu_parity import device_state, make_case  # noqa: E402


def test_memory_wait_timeout_is_reported_then_the_state_runs_clean():
    w, data, gcfg, ocfg = make_case("mid_key")  # bf16 q/v, d/2 = 64: tensor-core scoring and key step
    q, v, g, K1, K2, V = data
    st, dev = device_state(w, data, gcfg, w.T)
    C, T = w.C, w.T
    o = torch.zeros(w.M, T, w.d_v, device="cuda")
    fwpkm.test_stall_waits(1)
    st.forward_chunk(dev["q"], dev["v"], dev["g"], o, C, seq_stride=T)  # its scoring GEMM stalls
    torch.cuda.synchronize()  # the kernel has given up and latched the error
    with pytest.raises(fwpkm.FwpkmError) as e:
        st.write_chunk(dev["v"][:, C])
    assert e.value.status == fwpkm.ERR_TIMEOUT
    with pytest.raises(fwpkm.FwpkmError) as e:
        st.forward_chunk(dev["q"], dev["v"], dev["g"], o, C, seq_stride=T)
    assert e.value.status == fwpkm.ERR_TIMEOUT
    with pytest.raises(fwpkm.FwpkmError) as e:
        st.sync()
    assert e.value.status == fwpkm.ERR_TIMEOUT
    st.sync()  # cleared

    # the next chunk on the same state: from its current values, against the oracle
    K1pre, K2pre = dev["K1"].cpu().numpy().copy(), dev["K2"].cpu().numpy().copy()
    Vpre = dev["V"].cpu().numpy().copy()
    idx = torch.empty(w.M, C, w.k, dtype=torch.int32, device="cuda")
    st.forward_chunk(dev["q"], dev["v"], dev["g"], o, C, seq_stride=T, idx_out=idx)
    st.write_chunk(dev["v"][:, C])
    st.sync()
    qf, vf = as_f64(q, w.qv), as_f64(v, w.qv)
    idx_g = idx.cpu().numpy()
    for m in range(w.M):
        k1, k2, vv = K1pre[m].copy(), K2pre[m].copy(), Vpre[m].copy()
        o_o, _, _, _ = oracle_chunk_against_gpu(ocfg, qf[m, :C], vf[m, :C], g[m, :C].astype(np.float64),
                                                vf[m, C], k1, k2, vv, idx_g[m])
        assert_close(o[m, :C].cpu().numpy(), o_o, f"mem {m}: o after the timeout")
        assert_close(dev["V"][m].cpu().numpy(), vv, f"mem {m}: V after the timeout")
        assert_close(dev["K1"][m].cpu().numpy(), k1, f"mem {m}: K1 after the timeout")
        assert_close(dev["K2"][m].cpu().numpy(), k2, f"mem {m}: K2 after the timeout")


def test_layer_wait_timeout_is_reported_then_the_handle_runs_clean():
    w5 = WORKLOADS[5]
    rows = 200
    L = gen_layer(w5, B=1, T=rows)
    lay = fwpkm.Layer(w5.d_model, w5.d, w5.d_v, rows)
    Wd = {name: bf16_dev(L[name]) for name in ("Wq", "Wv", "wg", "Wo")}
    lay.set_params(Wd["Wq"], Wd["Wv"], Wd["wg"], Wd["Wo"])
    h = bf16_dev(L["h"][0])
    q = torch.empty(rows, w5.d, device="cuda")
    v = torch.empty(rows, w5.d_v, device="cuda")
    g = torch.empty(rows, device="cuda")
    lay.project_in(h, q, v, g)
    lay.sync()
    q_ref = q.clone()
    fwpkm.test_stall_waits(1)
    lay.project_in(h, q, v, g)  # its GEMM stalls and gives up
    torch.cuda.synchronize()
    with pytest.raises(fwpkm.FwpkmError) as e:
        lay.project_in(h, q, v, g)
    assert e.value.status == fwpkm.ERR_TIMEOUT
    with pytest.raises(fwpkm.FwpkmError) as e:
        lay.sync()
    assert e.value.status == fwpkm.ERR_TIMEOUT
    lay.sync()
    lay.project_in(h, q, v, g)
    lay.sync()
    assert torch.equal(q, q_ref), "the projection after the timeout differs from the one before"
