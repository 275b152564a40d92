"""The persistent value loop of fwpkm_run_sequence with frozen keys (one cooperative launch
runs the read and the write of every chunk of an addressing window, ordered by grid-wide
arrival counts) against the per-chunk calls, whose every chunk the other GPU tests compare
with the oracle.

  * several addressing windows (n = 1024, M = 8: 1024-token windows, the last one ragged)
    and two passes: o, V bit-for-bit against forward_chunk + write_chunk chunk by chunk,
    and a sample of the first window against the oracle directly;
  * the loop's bounded wait: fwpkm_test_stall_waits(1) makes its first arrival wait for a
    count no launch reaches; the wait gives up after 0.2 s, FWPKM_ERR_TIMEOUT comes back
    through fwpkm_sync, and the same state then runs cleanly (the arrival counters were
    cleared) with the bits of a fresh state.

Method: "Fast-weight Product Key Memory" (rainbus summary), method steps 2-4; the
iterative reading of the paperlayer summary §4.3 (passes over the same input).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import Workload, gen_keys, gen_qvg, gen_values  # noqa: E402

import oracle  # noqa: E402
from parity import as_f64, assert_close, oracle_chunk_against_gpu, to_device  # noqa: E402


def build(n, d, dv, k, C, M, T, qv, seed=21):
    w = Workload("vloop", n, d, dv, k, T, C, M, 1, qv, False, seed, "sigmoid", "normal002")
    q, v, g = gen_qvg(w)
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, m) for m in range(M)])
    gcfg = fwpkm.make_config(n, d, dv, k, C, M, qv == "bf16", key_update=False)
    ocfg = oracle.make_cfg(n, d, dv, k, C, key_update=False)
    return w, (q, v, g, K1, K2, V), gcfg, ocfg


def to_dev(w, data):
    q, v, g, K1, K2, V = data
    return dict(q=to_device(q, w.qv, torch), v=to_device(v, w.qv, torch), g=torch.from_numpy(g).cuda(),
                K1=torch.from_numpy(K1).cuda(), K2=torch.from_numpy(K2).cuda(), V=torch.from_numpy(V).cuda())


def chunk_calls(w, dev, gcfg, n_iter):
    st = fwpkm.State(gcfg, dev["K1"], dev["K2"], dev["V"], w.C)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    for _ in range(n_iter):
        for t0 in range(0, w.T, w.C):
            ln = min(w.C, w.T - t0)
            st.forward_chunk(dev["q"][:, t0:], dev["v"][:, t0:], dev["g"][:, t0:], o[:, t0:], ln, seq_stride=w.T)
            st.write_chunk(dev["v"][:, t0 + ln] if t0 + ln < w.T else None)
    st.sync()
    return o


@pytest.mark.parametrize("n_iter", [1, 2])
def test_value_loop_over_windows_matches_chunk_calls(n_iter):
    # 8 memories of 2^20 slots: the addressing window is 1024 tokens, so T = 2600 gives
    # windows of 4, 4 and 3 chunks (the last chunk 40 tokens)
    w, data, gcfg, ocfg = build(1024, 256, 64, 8, 256, 8, 2600, "bf16")
    dev_a = to_dev(w, data)
    st = fwpkm.State(gcfg, dev_a["K1"], dev_a["K2"], dev_a["V"], w.T)
    o_a = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.profile_kernel("value_loop")
    st.run_sequence(dev_a["q"], dev_a["v"], dev_a["g"], o_a, n_iter=n_iter)
    st.sync()
    ms, launches = st.kernel_time()
    st.profile_kernel(0)
    assert launches == 3 + (n_iter - 1), f"value loop launches {launches}"  # 3 windows, then 1 per pass

    dev_b = to_dev(w, data)
    o_b = chunk_calls(w, dev_b, gcfg, n_iter)
    assert torch.equal(o_a, o_b), "value loop o differs from the chunk calls"
    assert torch.equal(dev_a["V"], dev_b["V"]), "value loop V differs from the chunk calls"

    if n_iter == 1:
        # memory 0, first window (chunks 0..3): the loop's o against the oracle chained from
        # the initial V (o of chunk c reads the rows the loop wrote for chunks < c), with
        # the slot lists of a one-memory per-chunk state
        q, v, g, K1, K2, V = data
        qf, vf = as_f64(q, w.qv), as_f64(v, w.qv)
        cfg1 = fwpkm.make_config(w.n, w.d, w.d_v, w.k, w.C, 1, True, key_update=False)
        st1 = fwpkm.State(cfg1, dev_b["K1"][:1].contiguous(), dev_b["K2"][:1].contiguous(),
                          torch.from_numpy(V[:1]).cuda(), w.C)
        Vo = V[0].copy()
        for t0 in range(0, 1024, w.C):
            idx = torch.empty(1, w.C, w.k, dtype=torch.int32, device="cuda")
            o1 = torch.empty(1, w.C, w.d_v, device="cuda")
            st1.forward_chunk(dev_b["q"][:1, t0:], dev_b["v"][:1, t0:], dev_b["g"][:1, t0:], o1, w.C,
                              seq_stride=w.T, idx_out=idx)
            st1.write_chunk(dev_b["v"][:1, t0 + w.C])
            st1.sync()
            o_o, _, _, _ = oracle_chunk_against_gpu(ocfg, qf[0, t0:t0 + w.C], vf[0, t0:t0 + w.C],
                                                    g[0, t0:t0 + w.C].astype(np.float64), vf[0, t0 + w.C],
                                                    K1[0].copy(), K2[0].copy(), Vo, idx.cpu().numpy()[0])
            assert_close(o_a[0, t0:t0 + w.C].cpu().numpy(), o_o, f"chunk@{t0}: loop o against the oracle")


def test_value_loop_wait_timeout_then_clean_run():
    w, data, gcfg, _ = build(64, 64, 64, 8, 64, 2, 250, "f32")  # CUDA-core scoring: the loop takes the stall
    dev = to_dev(w, data)
    st = fwpkm.State(gcfg, dev["K1"], dev["K2"], dev["V"], w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    V0 = dev["V"].clone()
    fwpkm.test_stall_waits(1)
    st.run_sequence(dev["q"], dev["v"], dev["g"], o)
    torch.cuda.synchronize()
    with pytest.raises(fwpkm.FwpkmError) as e:
        st.sync()
    assert e.value.status == fwpkm.ERR_TIMEOUT
    st.sync()  # cleared
    # the loop gave up at its first wait, before any write: V is untouched
    assert torch.equal(dev["V"], V0)
    st.run_sequence(dev["q"], dev["v"], dev["g"], o)
    st.sync()
    dev2 = to_dev(w, data)
    st2 = fwpkm.State(gcfg, dev2["K1"], dev2["K2"], dev2["V"], w.T)
    o2 = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st2.run_sequence(dev2["q"], dev2["v"], dev2["g"], o2)
    st2.sync()
    assert torch.equal(o, o2) and torch.equal(dev["V"], dev2["V"])
