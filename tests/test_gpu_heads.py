"""Heads sharing one value table on the GPU (cfg.v_heads = H > 1, through the C ABI)
against the oracle (oracle.chunk_heads), chunk by chunk.

Reading ("Fast-weight Product Key Memory" (paperlayer summary) §D.1, §D.3; pinned in
tests/test_oracle_heads_pins.py): each head has its own codebooks and query and selects
its own k slots; the read is the mean of the heads' reads; the write is the gradient of
the gated reconstruction loss on the shared rows, divided by the number of tokens that
read a row through any head; each head takes its own addressing step.  After every
chunk: o, every head's weights and keys (and the key step itself), value rows; slot
lists bit-exact except counted near-ties (the oracle then adopts the GPU's slots for that
head-token).  Then fwpkm_run_sequence must give the chunk calls' bits.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import Workload, gen_keys, gen_qvg, gen_values  # noqa: E402

import oracle  # noqa: E402
from parity import as_f64, assert_close, classify_selection, to_device  # noqa: E402

# name: (n, d, d_v, k, C, B, H, T, qv, key_update)
CASES = {
    "simt_f32": (64, 64, 64, 8, 64, 2, 2, 150, "f32", True),      # CUDA-core scoring and key step
    "tc_fused": (256, 128, 128, 16, 128, 2, 2, 300, "bf16", True),  # one-launch addressing step
    "rows64": (256, 256, 256, 32, 128, 1, 2, 260, "bf16", False),   # k H = 64 rows per token
    "three_heads": (128, 128, 64, 8, 64, 2, 3, 140, "bf16", True),
}


def make(name):
    n, d, dv, k, C, B, H, T, qv, ku = CASES[name]
    M = B * H
    w = Workload(name, n, d, dv, k, T, C, M, 1, qv, ku, 31, "sigmoid", "normal002")
    q, v_all, g_all = gen_qvg(w)
    v, g = np.ascontiguousarray(v_all[:B]), np.ascontiguousarray(g_all[:B])  # one value stream per sequence
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, b) for b in range(B)])
    gcfg = fwpkm.make_config(n, d, dv, k, C, M, qv == "bf16", lr_key=10.0, key_update=ku, v_heads=H)
    ocfg = oracle.make_cfg(n, d, dv, k, C, lr_key=10.0, key_update=ku)
    return (n, d, dv, k, C, B, H, T, qv, ku), (q, v, g, K1, K2, V), gcfg, ocfg


def device(shape, data, gcfg, max_T):
    qv = shape[8]
    q, v, g, K1, K2, V = data
    dev = dict(q=to_device(q, qv, torch), v=to_device(v, qv, torch), g=torch.from_numpy(g).cuda(),
               K1=torch.from_numpy(K1).cuda(), K2=torch.from_numpy(K2).cuda(), V=torch.from_numpy(V).cuda())
    return fwpkm.State(gcfg, dev["K1"], dev["K2"], dev["V"], max_T), dev


@pytest.mark.parametrize("name", list(CASES))
def test_heads_sharing_v_match_oracle_every_chunk(name):
    shape, data, gcfg, ocfg = make(name)
    n, d, dv, k, C, B, H, T, qv, ku = shape
    q, v, g, K1, K2, V = data
    st, dev = device(shape, data, gcfg, C)
    o_d = torch.zeros(B, T, dv, device="cuda")
    qf, vf = as_f64(q, qv), as_f64(v, qv)
    V_orc = V.copy()
    ties = 0
    for t0 in range(0, T, C):
        ln = min(C, T - t0)
        K1pre, K2pre = dev["K1"].cpu().numpy().copy(), dev["K2"].cpu().numpy().copy()
        idx_d = torch.empty(B * H, ln, k, dtype=torch.int32, device="cuda")
        w_d = torch.empty(B * H, ln, k, device="cuda")
        st.forward_chunk(dev["q"][:, t0:], dev["v"][:, t0:], dev["g"][:, t0:], o_d[:, t0:], ln, seq_stride=T,
                         idx_out=idx_d, w_out=w_d)
        has_next = t0 + ln < T
        st.write_chunk(dev["v"][:, t0 + ln] if has_next else None)
        st.sync()
        idx_g, w_g = idx_d.cpu().numpy(), w_d.cpu().numpy()
        o_g = o_d[:, t0:t0 + ln].cpu().numpy()
        for b in range(B):
            heads = range(b * H, b * H + H)
            force = np.zeros((H, ln), np.int32)
            for j, m in enumerate(heads):
                for t in range(ln):
                    verdict = classify_selection(ocfg, qf[m, t0 + t], K1pre[m], K2pre[m], idx_g[m, t])
                    if verdict == "near_tie":
                        force[j, t] = 1
                        ties += 1
                    elif verdict != "exact":
                        raise AssertionError(f"{name} chunk@{t0} head {m} token {t}: {verdict}")
            k1, k2 = K1pre[b * H:b * H + H].copy(), K2pre[b * H:b * H + H].copy()
            vn = vf[b, t0 + ln] if has_next else None
            o_o, I_o, w_o = oracle.chunk_heads(ocfg, qf[b * H:b * H + H, t0:t0 + ln], vf[b, t0:t0 + ln],
                                               g[b, t0:t0 + ln].astype(np.float64), vn, k1, k2, V_orc[b],
                                               forced=idx_g[b * H:b * H + H], force_mask=force)
            assert_close(o_g[b], o_o, f"{name} chunk@{t0} seq {b}: o")
            assert_close(w_g[b * H:b * H + H], w_o, f"{name} chunk@{t0} seq {b}: w", atol=1e-6)
            if ku:
                for j in range(H):
                    m = b * H + j
                    K1g, K2g = dev["K1"][m].cpu().numpy(), dev["K2"][m].cpu().numpy()
                    assert_close(K1g, k1[j], f"{name} chunk@{t0} head {m}: K1")
                    assert_close(K2g, k2[j], f"{name} chunk@{t0} head {m}: K2")
            if n * n * dv <= (1 << 22):
                rows = np.arange(n * n)
            else:
                touched = np.unique(idx_g[b * H:b * H + H].reshape(-1))
                rows = np.unique(np.concatenate([touched, np.random.default_rng(0).integers(0, n * n, 1024)]))
            Vg = dev["V"][b][torch.from_numpy(rows).cuda()].cpu().numpy()
            assert_close(Vg, V_orc[b][rows], f"{name} chunk@{t0} seq {b}: V")
    print(f"{name}: near-ties {ties}")
    # the production schedule gives the chunk calls' bits
    st2, dev2 = device(shape, data, gcfg, T)
    o2 = torch.zeros(B, T, dv, device="cuda")
    st2.run_sequence(dev2["q"], dev2["v"], dev2["g"], o2)
    st2.sync()
    assert torch.equal(o2, o_d), f"{name}: run_sequence o differs from chunk-by-chunk"
    assert torch.equal(dev2["V"], dev["V"]), f"{name}: run_sequence V differs"
    assert torch.equal(dev2["K1"], dev["K1"]) and torch.equal(dev2["K2"], dev["K2"])


def test_heads_argument_rules():
    shape, data, gcfg, _ = make("tc_fused")
    n, d, dv, k, C, B, H, T, qv, ku = shape
    st, dev = device(shape, data, gcfg, C)
    o = torch.zeros(B, T, dv, device="cuda")
    with pytest.raises(fwpkm.FwpkmError) as e:  # token-at-a-time reads take independent memories only
        st.stream_tokens(dev["q"], dev["v"], dev["g"], o, n_tok=1, seq_stride=T)
    assert e.value.status == fwpkm.ERR_UNSUPPORTED
    with pytest.raises(fwpkm.FwpkmError) as e:
        fwpkm.chunk_step_noalloc(gcfg, dev["K1"], dev["K2"], dev["V"], dev["q"], dev["v"], dev["g"], o, C,
                                 seq_stride=T)
    assert e.value.status == fwpkm.ERR_UNSUPPORTED
    bad = fwpkm.make_config(n, d, dv, k, C, 3, True, v_heads=2)  # memories not a multiple of the heads
    with pytest.raises(fwpkm.FwpkmError) as e:
        fwpkm.workspace_size(bad, C)
    assert e.value.status == fwpkm.ERR_INVALID_ARG
