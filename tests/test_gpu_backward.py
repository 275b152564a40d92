"""The read path's backward on the GPU (fwpkm_read_backward through the C ABI) against the
oracle (oracle/backward.py, pinned by finite differences of the forward oracle), chunk by
chunk: every chunk is read on the GPU (forward_chunk with its slot lists), its backward is
taken from a seeded upstream gradient with the state the chunk was read with, both are
compared element by element (dq, dv, dg), then the chunk is written and the next one read.

Reading ("Fast-weight Product Key Memory" (paperlayer summary) §2 / Figure 1, §3.1-§3.2):
the fast weights at the read are constants of the backward and the discrete selection
passes no gradient.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import Workload, gen_keys, gen_qvg, gen_values  # noqa: E402

from oracle.backward import read_backward as oracle_read_backward  # noqa: E402
from parity import as_f64, assert_close, to_device  # noqa: E402

# name: (n, d, dv, k, C, M, T, qv, key_update)
CASES = {
    "tiny_f32": (64, 64, 64, 8, 64, 1, 150, "f32", True),
    "mid_bf16": (256, 128, 128, 16, 128, 2, 260, "bf16", False),
    "paper_shapes": (1024, 256, 256, 32, 256, 2, 300, "bf16", True),
    "odd_dims": (48, 40, 36, 5, 32, 2, 70, "f32", True),  # h = 20, d_v = 36: partial lanes
    "k1_bf16": (64, 128, 64, 1, 32, 2, 70, "bf16", True),  # one slot: s' = 1, so dq = 0
}


@pytest.mark.parametrize("name", list(CASES))
def test_read_backward_matches_oracle_every_chunk(name):
    n, d, dv, k, C, M, T, qv, ku = CASES[name]
    w = Workload(name, n, d, dv, k, T, C, M, 1, qv, ku, 17, "sigmoid", "normal002")
    q, v, g = gen_qvg(w)
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, m) for m in range(M)])
    cfg = fwpkm.make_config(n, d, dv, k, C, M, qv == "bf16", lr_key=10.0, key_update=ku)
    qd, vd, gd = to_device(q, qv, torch), to_device(v, qv, torch), torch.from_numpy(g).cuda()
    K1d, K2d, Vd = (torch.from_numpy(x).cuda() for x in (K1, K2, V))
    st = fwpkm.State(cfg, K1d, K2d, Vd, C)
    o = torch.zeros(M, T, dv, device="cuda")
    rng = np.random.default_rng(3)
    d_o = torch.from_numpy(rng.normal(size=(M, T, dv)).astype(np.float32)).cuda()
    dq = torch.full((M, T, d), float("nan"), device="cuda")
    dvv = torch.full((M, T, dv), float("nan"), device="cuda")
    dg = torch.full((M, T), float("nan"), device="cuda")
    qf, vf = as_f64(q, qv), as_f64(v, qv)
    for t0 in range(0, T, C):
        ln = min(C, T - t0)
        idx = torch.empty(M, ln, k, dtype=torch.int32, device="cuda")
        st.forward_chunk(qd[:, t0:], vd[:, t0:], gd[:, t0:], o[:, t0:], ln, seq_stride=T, idx_out=idx)
        st.sync()
        K1s, K2s, Vs = K1d.cpu().numpy(), K2d.cpu().numpy(), Vd.cpu().numpy()
        fwpkm.read_backward(cfg, K1d, K2d, Vd, qd[:, t0:], vd[:, t0:], gd[:, t0:], idx, d_o[:, t0:],
                            dq[:, t0:], dvv[:, t0:], dg[:, t0:], len_=ln, seq_stride=T)
        torch.cuda.synchronize()
        I = idx.cpu().numpy()
        for m in range(M):
            rq, rv, rg = oracle_read_backward(n, cfg.eps_idw, qf[m, t0:t0 + ln], vf[m, t0:t0 + ln],
                                              g[m, t0:t0 + ln], K1s[m], K2s[m], Vs[m], I[m],
                                              d_o[m, t0:t0 + ln].cpu().numpy())
            assert_close(dq[m, t0:t0 + ln].cpu().numpy(), rq, f"{name} chunk@{t0} mem {m}: dq")
            assert_close(dvv[m, t0:t0 + ln].cpu().numpy(), rv, f"{name} chunk@{t0} mem {m}: dv")
            assert_close(dg[m, t0:t0 + ln].cpu().numpy(), rg, f"{name} chunk@{t0} mem {m}: dg")
        st.write_chunk(vd[:, t0 + ln] if t0 + ln < T else None)
    st.sync()


def test_read_backward_argument_checks():
    n, d, dv, k, C, M, T, qv, ku = CASES["tiny_f32"]
    cfg = fwpkm.make_config(n, d, dv, k, C, M, False)
    z = lambda *s: torch.zeros(*s, device="cuda")  # noqa: E731
    K1, K2, V = z(M, n, d // 2), z(M, n, d // 2), z(M, n * n, dv)
    q, v, g, d_o = z(M, T, d), z(M, T, dv), z(M, T), z(M, T, dv)
    idx = torch.zeros(M, C, k, dtype=torch.int32, device="cuda")
    out = (z(M, T, d), z(M, T, dv), z(M, T))
    with pytest.raises(fwpkm.FwpkmError) as e:  # seq_stride < len
        fwpkm.read_backward(cfg, K1, K2, V, q, v, g, idx, d_o, *out, len_=C, seq_stride=C - 1)
    assert e.value.status == fwpkm.ERR_INVALID_ARG
    heads = fwpkm.make_config(n, d, dv, k, C, 2, False, v_heads=2)
    with pytest.raises(fwpkm.FwpkmError) as e:
        fwpkm.read_backward(heads, K1, K2, V, q, v, g, idx, d_o, *out, len_=C, seq_stride=T)
    assert e.value.status == fwpkm.ERR_UNSUPPORTED
    fwpkm.read_backward(cfg, K1, K2, V, q, v, g, idx, d_o, *out, len_=0, seq_stride=T)  # no-op


def test_read_backward_drops_slots_outside_the_memory():
    """Slots outside [0, N) contribute nothing: the token's softmax runs over its valid
    slots only (the oracle is given just those), and a token with none has vhat = 0, so
    dq = 0, dv = (1 - g) dL/do, dg = -<dL/do, v>."""
    n, d, dv, k, C, M, T = 64, 64, 64, 8, 64, 2, 40
    N = n * n
    w = Workload("drop", n, d, dv, k, T, C, M, 1, "f32", False, 23, "sigmoid", "normal002")
    q, v, g = gen_qvg(w)
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, m) for m in range(M)])
    cfg = fwpkm.make_config(n, d, dv, k, C, M, False)
    rng = np.random.default_rng(11)
    I = np.stack([np.stack([rng.choice(N, size=k, replace=False) for _ in range(T)]) for _ in range(M)])
    I = I.astype(np.int32)
    drop = rng.random(I.shape) < 0.3
    I[drop] = np.where(rng.random(int(drop.sum())) < 0.5, -1, N + 5).astype(np.int32)
    I[0, 3, :] = -1                       # a token with no valid slot
    I[1, 7, :] = N                        # another one, past the end
    d_o = rng.normal(size=(M, T, dv)).astype(np.float32)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()  # noqa: E731
    dq = torch.full((M, T, d), float("nan"), device="cuda")
    dvv = torch.full((M, T, dv), float("nan"), device="cuda")
    dg = torch.full((M, T), float("nan"), device="cuda")
    fwpkm.read_backward(cfg, dev(K1), dev(K2), dev(V), dev(q), dev(v), dev(g), dev(I), dev(d_o),
                        dq, dvv, dg, len_=T, seq_stride=T)
    torch.cuda.synchronize()
    dq, dvv, dg = dq.cpu().numpy(), dvv.cpu().numpy(), dg.cpu().numpy()
    for m in range(M):
        for t in range(T):
            ok = I[m, t][(I[m, t] >= 0) & (I[m, t] < N)]
            if ok.size == 0:
                assert np.all(dq[m, t] == 0.0), f"mem {m} token {t}: dq"
                assert np.array_equal(dvv[m, t], (np.float32(1.0) - g[m, t]) * d_o[m, t]), f"mem {m} token {t}: dv"
                assert_close(np.array([dg[m, t]]), np.array([-np.dot(d_o[m, t].astype(np.float64), v[m, t])]),
                             f"mem {m} token {t}: dg")
                continue
            rq, rv, rg = oracle_read_backward(n, cfg.eps_idw, q[m, t:t + 1], v[m, t:t + 1], g[m, t:t + 1],
                                              K1[m], K2[m], V[m], ok[None, :], d_o[m, t:t + 1])
            assert_close(dq[m, t:t + 1], rq, f"mem {m} token {t}: dq")
            assert_close(dvv[m, t:t + 1], rv, f"mem {m} token {t}: dv")
            assert_close(dg[m, t:t + 1], rg, f"mem {m} token {t}: dg")
