"""GPU (libfwpkm.so through the C ABI) against the CPU oracle on the same seeded inputs.

Element-by-element, after every chunk, at sizes the oracle finishes in seconds: the
five workload shapes (n, d, d_v, k, C, dtype) with reduced M and T, ragged tails,
key update on and off.  The production entry point (fwpkm_run_sequence) is then
checked bit-for-bit against the chunk-by-chunk entry points on the same inputs.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import Workload, gen_keys, gen_qvg, gen_values  # noqa: E402

import oracle  # noqa: E402
from parity import as_f64, assert_close, oracle_chunk_against_gpu, to_device  # noqa: E402

# name: (n, d, d_v, k, C, M, T, qv, key_update, lr_key, v_init)
CASES = {
    "tiny": (64, 64, 64, 8, 64, 1, 256, "f32", False, 1.0, "zero"),
    "tiny_key_ragged": (64, 64, 64, 8, 64, 2, 250, "f32", True, 100.0, "normal002"),
    "mid": (256, 128, 128, 16, 128, 3, 300, "bf16", False, 1.0, "normal002"),
    "mid_key": (256, 128, 128, 16, 128, 2, 300, "bf16", True, 100.0, "normal002"),
    "paper": (1024, 256, 256, 32, 256, 2, 600, "bf16", True, 1.0, "normal002"),
    "needle_chunk": (1024, 256, 256, 32, 512, 1, 1100, "bf16", False, 1.0, "normal002"),
    "layer_shape": (512, 256, 256, 32, 256, 2, 520, "f32", True, 1.0, "normal002"),
    # degenerate and extreme shapes
    "k_equals_n": (8, 16, 8, 8, 4, 2, 21, "f32", True, 10.0, "normal002"),   # every sub-key survives
    "k1": (64, 128, 64, 1, 32, 2, 70, "bf16", True, 10.0, "normal002"),       # single slot per token
    "chunk1": (64, 128, 64, 4, 1, 1, 9, "bf16", True, 10.0, "normal002"),     # one token per chunk
    "n_max": (4096, 256, 32, 32, 16, 1, 40, "bf16", True, 1.0, "normal002"),  # largest codebook
}


def make_case(name, seed=10, **flags):
    n, d, dv, k, C, M, T, qv, ku, lr, vinit = CASES[name]
    w = Workload(name, n, d, dv, k, T, C, M, 1, qv, ku, seed, "sigmoid", vinit)
    q, v, g = gen_qvg(w)
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, m) for m in range(M)])
    gcfg = fwpkm.make_config(n, d, dv, k, C, M, qv == "bf16", lr_key=lr, key_update=ku, **flags)
    ocfg = oracle.make_cfg(n, d, dv, k, C, lr_key=lr, key_update=ku, **flags)
    return w, (q, v, g, K1, K2, V), gcfg, ocfg


def device_state(w, data, gcfg, max_T):
    q, v, g, K1, K2, V = data
    dev = dict(q=to_device(q, w.qv, torch), v=to_device(v, w.qv, torch), g=torch.from_numpy(g).cuda(),
               K1=torch.from_numpy(K1).cuda(), K2=torch.from_numpy(K2).cuda(), V=torch.from_numpy(V).cuda())
    st = fwpkm.State(gcfg, dev["K1"], dev["K2"], dev["V"], max_T)
    return st, dev


def workload_case(w):
    """A benchmark workload at its full size, with the benchmark's own seed (same inputs)."""
    q, v, g = gen_qvg(w)
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, m) for m in range(w.M)])
    gcfg = fwpkm.make_config(w.n, w.d, w.d_v, w.k, w.C, w.M, w.qv == "bf16", key_update=w.key_update)
    ocfg = oracle.make_cfg(w.n, w.d, w.d_v, w.k, w.C, key_update=w.key_update)
    return w, (q, v, g, K1, K2, V), gcfg, ocfg


def streaming_vs_oracle(name, **flags):
    return compare_streaming(name, *make_case(name, **flags))


def compare_streaming(name, w, data, gcfg, ocfg, n_iter=1):
    """Chunk by chunk (n_iter passes over the sequence, the state carried across them):
    forward_chunk + write_chunk on the GPU against the oracle's chunk from the GPU's own
    pre-chunk state; o, weights, keys (and the key step itself) and value rows compared
    after every chunk.  Returns the final GPU tensors, the near-tie count and every
    chunk's slot lists (idx: list of [M][len][k] arrays, in order)."""
    q, v, g, K1, K2, V = data
    M, T, C, k, dv, N = w.M, w.T, w.C, w.k, w.d_v, w.N
    st, dev = device_state(w, data, gcfg, C)
    o_d = torch.zeros(M, T, dv, device="cuda")
    qf, vf = as_f64(q, w.qv), as_f64(v, w.qv)
    V_orc = V.copy()
    small = N * dv <= (1 << 22)
    rng = np.random.default_rng(0)
    ties = 0
    idx_all = []
    for _pass in range(n_iter):
        for t0 in range(0, T, C):
            ln = min(C, T - t0)
            K1pre, K2pre = dev["K1"].cpu().numpy().copy(), dev["K2"].cpu().numpy().copy()
            idx_d = torch.empty(M, ln, k, dtype=torch.int32, device="cuda")
            w_d = torch.empty(M, ln, k, device="cuda")
            st.forward_chunk(dev["q"][:, t0:], dev["v"][:, t0:], dev["g"][:, t0:], o_d[:, t0:], ln, seq_stride=T,
                             idx_out=idx_d, w_out=w_d)
            has_next = t0 + ln < T
            st.write_chunk(dev["v"][:, t0 + ln] if has_next else None)
            st.sync()
            idx_g, w_g = idx_d.cpu().numpy(), w_d.cpu().numpy()
            idx_all.append(idx_g)
            o_g = o_d[:, t0:t0 + ln].cpu().numpy()
            for m in range(M):
                k1, k2 = K1pre[m].copy(), K2pre[m].copy()
                vn = vf[m, t0 + ln] if has_next else None
                o_o, I_o, w_o, nt = oracle_chunk_against_gpu(ocfg, qf[m, t0:t0 + ln], vf[m, t0:t0 + ln],
                                                             g[m, t0:t0 + ln].astype(np.float64), vn, k1, k2,
                                                             V_orc[m], idx_g[m])
                ties += nt
                assert_close(o_g[m], o_o, f"{name} chunk@{t0} mem {m}: o")
                assert_close(w_g[m], w_o, f"{name} chunk@{t0} mem {m}: w", atol=1e-6)
                if w.key_update:
                    K1g, K2g = dev["K1"][m].cpu().numpy(), dev["K2"][m].cpu().numpy()
                    assert_close(K1g, k1, f"{name} chunk@{t0} mem {m}: K1")
                    assert_close(K2g, k2, f"{name} chunk@{t0} mem {m}: K2")
                    # the step itself (tiny next to K) must agree, not just the keys
                    for Kg, Ko, Kp in ((K1g, k1, K1pre[m]), (K2g, k2, K2pre[m])):
                        dg = Kg.astype(np.float64) - Kp
                        do = Ko.astype(np.float64) - Kp
                        ulp = np.spacing(np.abs(Ko)).astype(np.float64)
                        assert np.all(np.abs(dg - do) <= 2 * ulp + 2e-3 * np.abs(do) + 1e-9), f"{name}: dK"
                if small:
                    rows = np.arange(N)
                else:
                    touched = np.unique(idx_g[m].reshape(-1))
                    rows = np.unique(np.concatenate([touched, rng.integers(0, N, 2048)]))
                Vg = dev["V"][m][torch.from_numpy(rows).cuda()].cpu().numpy()
                assert_close(Vg, V_orc[m][rows], f"{name} chunk@{t0} mem {m}: V")
    # full-size states stay on the device (8 GiB of V)
    return dict(o=o_d.cpu(), V=dev["V"].cpu() if small else dev["V"], K1=dev["K1"].cpu(), K2=dev["K2"].cpu(), ties=ties,
                w=w, data=data, gcfg=gcfg, idx=idx_all)


@pytest.mark.parametrize("name", list(CASES))
def test_streaming_matches_oracle_every_chunk(name):
    res = streaming_vs_oracle(name)
    print(f"{name}: near-ties {res['ties']}")
    # the production schedule computes the same bits
    w, data, gcfg = res["w"], res["data"], res["gcfg"]
    st, dev = device_state(w, data, gcfg, w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(dev["q"], dev["v"], dev["g"], o)
    st.sync()
    assert torch.equal(o.cpu(), res["o"]), "run_sequence o differs from chunk-by-chunk"
    assert torch.equal(dev["V"].cpu(), res["V"].cpu()), "run_sequence V differs"
    assert torch.equal(dev["K1"].cpu(), res["K1"]) and torch.equal(dev["K2"].cpu(), res["K2"])


def test_paper_workload_full_size():
    """The paper-scale workload at the benchmark's full size and seed (8 memories of
    N = 1,048,576 slots, T = 4096, C = 256, key update on): every chunk's outputs, weights,
    keys and sampled value rows against the oracle, then the benchmark's entry point
    (fwpkm_run_sequence, one captured graph) bit-for-bit against the chunk-by-chunk run."""
    from sparse_weight_memory_chunk_b200.inputs import WORKLOADS
    w = WORKLOADS[3]
    res = compare_streaming("paper_full", *workload_case(w))
    print(f"paper full size: near-ties {res['ties']}")
    data, gcfg = res["data"], res["gcfg"]
    st, dev = device_state(w, data, gcfg, w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(dev["q"], dev["v"], dev["g"], o)
    st.sync()
    assert torch.equal(o.cpu(), res["o"]), "run_sequence o differs from chunk-by-chunk"
    assert torch.equal(dev["V"], res["V"]), "run_sequence V differs from chunk-by-chunk"
    assert torch.equal(dev["K1"].cpu(), res["K1"]) and torch.equal(dev["K2"].cpu(), res["K2"])


def test_mid_workload_full_size():
    """The mid workload at its full size and seed (16 memories of 65,536 slots, T = 4096,
    C = 128, frozen keys): every chunk's outputs, weights and sampled value rows against the
    oracle, then fwpkm_run_sequence (two addressing windows, the persistent value loop) bit
    for bit against the chunk-by-chunk run."""
    from sparse_weight_memory_chunk_b200.inputs import WORKLOADS
    w = WORKLOADS[2]
    res = compare_streaming("mid_full", *workload_case(w))
    print(f"mid full size: near-ties {res['ties']}")
    data, gcfg = res["data"], res["gcfg"]
    st, dev = device_state(w, data, gcfg, w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(dev["q"], dev["v"], dev["g"], o)
    st.sync()
    assert torch.equal(o.cpu(), res["o"]), "run_sequence o differs from chunk-by-chunk"
    assert torch.equal(dev["V"], res["V"].cuda() if not res["V"].is_cuda else res["V"]), "run_sequence V differs"


@pytest.mark.parametrize("flags", [dict(lookahead=False), dict(target_norm=False), dict(gate_weight=False)])
def test_flag_variants(flags):
    streaming_vs_oracle("tiny_key_ragged", **flags)


@pytest.mark.parametrize("flags", [dict(lookahead=False), dict(target_norm=False), dict(gate_weight=False)])
def test_flag_variants_frozen_keys(flags):
    """The flag variants with frozen keys on the tensor-core shapes: chunk by chunk against
    the oracle, then fwpkm_run_sequence (addressing windows and the persistent value loop)
    bit-for-bit against those calls."""
    res = streaming_vs_oracle("mid", **flags)
    w, data, gcfg = res["w"], res["data"], res["gcfg"]
    st, dev = device_state(w, data, gcfg, w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(dev["q"], dev["v"], dev["g"], o)
    st.sync()
    assert torch.equal(o.cpu(), res["o"]), f"{flags}: run_sequence o differs from chunk-by-chunk"
    assert torch.equal(dev["V"].cpu(), res["V"].cpu()), f"{flags}: run_sequence V differs"


@pytest.mark.parametrize("name", ["mid", "mid_key"])
def test_passes_compose_and_determinism(name):
    w, data, gcfg, _ = make_case(name)
    outs = []
    for _ in range(2):
        st, dev = device_state(w, data, gcfg, w.T)
        o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
        st.run_sequence(dev["q"], dev["v"], dev["g"], o, n_iter=2)
        st.sync()
        outs.append((o.cpu(), dev["V"].cpu(), dev["K1"].cpu()))
    assert all(torch.equal(a, b) for a, b in zip(*outs)), "two identical runs differ"
    st, dev = device_state(w, data, gcfg, w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(dev["q"], dev["v"], dev["g"], o, n_iter=1)
    st.run_sequence(dev["q"], dev["v"], dev["g"], o, n_iter=1)
    st.sync()
    assert torch.equal(o.cpu(), outs[0][0]) and torch.equal(dev["V"].cpu(), outs[0][1])
    assert torch.equal(dev["K1"].cpu(), outs[0][2])


def test_needle_stream_two_passes():
    """The needle workload's shapes (N = 1,048,576 slots, C = 512, frozen keys) with its
    planted (q*, v*) needle pairs, read in two passes over the same input (paperlayer §4.3
    iterative reading): every chunk of both passes against the oracle, then
    fwpkm_run_sequence(n_iter = 2) bit-for-bit against those chunk-by-chunk calls."""
    from dataclasses import replace

    from sparse_weight_memory_chunk_b200.inputs import gen_needles
    w, data, gcfg, ocfg = make_case("needle_chunk")
    w = replace(w, needles=64)
    q, v, g, K1, K2, V = data
    gen_needles(w, q, v)  # in place: 64 needles planted 3 times each, queried once late
    res = compare_streaming("needle_2pass", w, (q, v, g, K1, K2, V), gcfg, ocfg, n_iter=2)
    print(f"needle two passes: near-ties {res['ties']}")
    st, dev = device_state(w, (q, v, g, K1, K2, V), gcfg, w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(dev["q"], dev["v"], dev["g"], o, n_iter=2)
    st.sync()
    assert torch.equal(o.cpu(), res["o"]), "run_sequence(n_iter=2) o differs from chunk-by-chunk"
    assert torch.equal(dev["V"], res["V"]), "run_sequence(n_iter=2) V differs from chunk-by-chunk"


def test_needle_workload_full_size_sampled():
    """The needle workload at its full size and seed (N = 2^20 slots, T = 131,072, C = 512,
    frozen keys, 64 planted needles): fwpkm_run_sequence, in the launch configuration the
    benchmark times (addressing windows and the persistent value loop), bit-for-bit against
    the chunk-by-chunk calls over all 256 chunks; every 16th of those chunks, and the last,
    against the oracle from the GPU's own pre-chunk state (o, weights and every value row the
    chunk writes)."""
    from sparse_weight_memory_chunk_b200.inputs import WORKLOADS, gen_needles
    w = WORKLOADS[4]
    _, data, gcfg, ocfg = workload_case(w)
    q, v, g, K1, K2, V = data
    gen_needles(w, q, v)
    M, T, C, k, dv = w.M, w.T, w.C, w.k, w.d_v
    st, dev = device_state(w, (q, v, g, K1, K2, V), gcfg, C)
    o_d = torch.zeros(M, T, dv, device="cuda")
    qf, vf = as_f64(q, w.qv), as_f64(v, w.qv)
    nch = (T + C - 1) // C
    sampled = set(range(0, nch, 16)) | {nch - 1}
    ties = 0
    for ci in range(nch):
        t0 = ci * C
        ln = min(C, T - t0)
        check = ci in sampled
        if check:
            st.sync()
            Vpre = dev["V"][0].cpu().numpy().copy()
            idx_d = torch.empty(M, ln, k, dtype=torch.int32, device="cuda")
            w_d = torch.empty(M, ln, k, device="cuda")
        st.forward_chunk(dev["q"][:, t0:], dev["v"][:, t0:], dev["g"][:, t0:], o_d[:, t0:], ln, seq_stride=T,
                         idx_out=idx_d if check else None, w_out=w_d if check else None)
        has_next = t0 + ln < T
        st.write_chunk(dev["v"][:, t0 + ln] if has_next else None)
        if check:
            st.sync()
            idx_g = idx_d.cpu().numpy()[0]
            vn = vf[0, t0 + ln] if has_next else None
            Vo = Vpre  # the oracle updates it in place
            o_o, I_o, w_o, nt = oracle_chunk_against_gpu(ocfg, qf[0, t0:t0 + ln], vf[0, t0:t0 + ln],
                                                         g[0, t0:t0 + ln].astype(np.float64), vn, K1[0].copy(),
                                                         K2[0].copy(), Vo, idx_g)
            ties += nt
            assert_close(o_d[0, t0:t0 + ln].cpu().numpy(), o_o, f"needle chunk {ci}: o")
            assert_close(w_d.cpu().numpy()[0], w_o, f"needle chunk {ci}: w", atol=1e-6)
            rows = np.unique(idx_g.reshape(-1))
            Vg = dev["V"][0][torch.from_numpy(rows).cuda()].cpu().numpy()
            assert_close(Vg, Vo[rows], f"needle chunk {ci}: written V rows")
    st.sync()
    print(f"needle full size: {len(sampled)} chunks against the oracle, near-ties {ties}")
    st2, dev2 = device_state(w, (q, v, g, K1, K2, V), gcfg, T)
    o2 = torch.zeros(M, T, dv, device="cuda")
    st2.run_sequence(dev2["q"], dev2["v"], dev2["g"], o2)
    st2.sync()
    assert torch.equal(o2, o_d), "needle full size: run_sequence o differs from chunk-by-chunk"
    assert torch.equal(dev2["V"], dev["V"]), "needle full size: run_sequence V differs from chunk-by-chunk"


def test_edge_cases():
    w, data, gcfg, ocfg = make_case("tiny_key_ragged")
    st, dev = device_state(w, data, gcfg, w.T)
    V0, K10 = dev["V"].clone(), dev["K1"].clone()
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(dev["q"], dev["v"], dev["g"], o, T=0)  # no-op
    st.sync()
    assert torch.equal(dev["V"], V0)
    # one token: nothing to write (no lookahead target) but the keys still take their step
    st.run_sequence(dev["q"][:, :1].contiguous(), dev["v"][:, :1].contiguous(), dev["g"][:, :1].contiguous(),
                    o[:, :1].contiguous(), T=1)
    st.sync()
    assert torch.equal(dev["V"], V0)
    assert not torch.equal(dev["K1"], K10)
    with pytest.raises(fwpkm.FwpkmError) as e:
        st.write_chunk(None)
    assert e.value.status == fwpkm.ERR_STATE
    with pytest.raises(fwpkm.FwpkmError) as e:
        st.run_sequence(dev["q"], dev["v"], dev["g"], o, T=w.T + 1)
    assert e.value.status == fwpkm.ERR_INVALID_ARG


@pytest.mark.parametrize("name,groups", [("mid", 2), ("mid", 3), ("mid_key", 2), ("tiny_key_ragged", 2)])
def test_memory_groups_give_the_same_bits(name, groups, monkeypatch):
    """run_sequence splits the memories into groups with their own chains; the split
    changes only the schedule, so every output bit equals the one-group run (which the
    test above ties to the oracle through the chunk-by-chunk entry points)."""
    w, data, gcfg, _ = make_case(name)
    outs = []
    for gr in (1, groups):
        monkeypatch.setenv("FWPKM_GROUPS", str(gr))
        st, dev = device_state(w, data, gcfg, w.T)
        o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
        st.run_sequence(dev["q"], dev["v"], dev["g"], o, n_iter=2)
        st.sync()
        outs.append((o.cpu(), dev["V"].cpu(), dev["K1"].cpu(), dev["K2"].cpu()))
    assert all(torch.equal(a, b) for a, b in zip(*outs)), f"{name}: {groups} groups differ from one"
