"""Token-at-a-time inference on the GPU (fwpkm_stream_tokens / fwpkm_stream_flush through
the C ABI).

Feeding a sequence in arbitrary groups of tokens, then flushing, is compared directly
with the oracle's own token-at-a-time loop (oracle/stream.py: each token read as it
arrives, a chunk written when its lookahead arrives; "Fast-weight Product Key Memory"
(paperlayer summary) §A.1), and must also give the bits of the production entry point
(fwpkm_run_sequence) on the same inputs: the reads are per token and the writes are the
same kernels on the same chunk contents.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402

from oracle.stream import stream_sequence  # noqa: E402
from parity import as_f64, assert_close  # noqa: E402
from test_gpu_parity import device_state, make_case  # noqa: E402


def groups_for(T, C, seed):
    rng = np.random.default_rng(seed)
    sizes = [1, 2, 3, max(1, C - 1), C, C + 1, 2 * C + 3]
    out, t = [], 0
    while t < T:
        n = min(T - t, int(rng.choice(sizes)))
        out.append(n)
        t += n
    return out


def reference(w, data, gcfg):
    st, dev = device_state(w, data, gcfg, w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(dev["q"], dev["v"], dev["g"], o)
    st.sync()
    return o, dev


@pytest.mark.parametrize("name", ["tiny_key_ragged", "mid", "mid_key", "k1", "chunk1", "k_equals_n", "paper"])
def test_token_stream_gives_the_bits_of_run_sequence(name):
    w, data, gcfg, _ = make_case(name)
    o_ref, dev_ref = reference(w, data, gcfg)
    st, dev = device_state(w, data, gcfg, w.C)  # a chunk of workspace is enough
    o = torch.full((w.M, w.T, w.d_v), float("nan"), device="cuda")
    t = 0
    for n in groups_for(w.T, w.C, seed=len(name)):
        st.stream_tokens(dev["q"][:, t:], dev["v"][:, t:], dev["g"][:, t:], o[:, t:], n_tok=n, seq_stride=w.T)
        t += n
        if t == w.C + 3 or (t > w.C + 3 and t - n < w.C + 3):
            # outputs are final as soon as their tokens are read
            st.sync()
            assert torch.equal(o[:, :t], o_ref[:, :t]), f"{name}: o of the first {t} tokens"
    st.stream_flush()
    st.sync()
    assert torch.equal(o, o_ref), f"{name}: o differs from run_sequence"
    for key in ("V", "K1", "K2"):
        assert torch.equal(dev[key], dev_ref[key]), f"{name}: {key} differs from run_sequence"


@pytest.mark.parametrize("name", ["tiny_key_ragged", "mid_key", "k1", "chunk1"])
def test_token_stream_matches_oracle_stream(name):
    """o of every token and the final V, K1, K2 against oracle.stream_sequence fed the same
    arrival groups (parity tolerances: 1e-4 relative + 1e-5 absolute)."""
    w, data, gcfg, ocfg = make_case(name)
    q, v, g, K1, K2, V = data
    st, dev = device_state(w, data, gcfg, w.C)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    groups = groups_for(w.T, w.C, seed=7 + len(name))
    t = 0
    for n in groups:
        st.stream_tokens(dev["q"][:, t:], dev["v"][:, t:], dev["g"][:, t:], o[:, t:], n_tok=n, seq_stride=w.T)
        t += n
    st.stream_flush()
    st.sync()
    qf, vf = as_f64(q, w.qv), as_f64(v, w.qv)
    for m in range(w.M):
        k1, k2, vv = K1[m].copy(), K2[m].copy(), V[m].copy()
        o_o = stream_sequence(ocfg, qf[m], vf[m], g[m].astype(np.float64), k1, k2, vv, groups)
        assert_close(o[m].cpu().numpy(), o_o, f"{name} mem {m}: o")
        assert_close(dev["V"][m].cpu().numpy(), vv, f"{name} mem {m}: V")
        assert_close(dev["K1"][m].cpu().numpy(), k1, f"{name} mem {m}: K1")
        assert_close(dev["K2"][m].cpu().numpy(), k2, f"{name} mem {m}: K2")


def test_one_token_at_a_time_and_state_rules():
    w, data, gcfg, _ = make_case("mid_key")
    o_ref, dev_ref = reference(w, data, gcfg)
    st, dev = device_state(w, data, gcfg, w.T)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    st.stream_flush()  # nothing pending: no-op
    for t in range(w.T):
        st.stream_tokens(dev["q"][:, t:], dev["v"][:, t:], dev["g"][:, t:], o[:, t:], n_tok=1, seq_stride=w.T)
        assert st.stream_pending() == t % w.C + 1
        if t == 5:
            with pytest.raises(fwpkm.FwpkmError) as e:  # chunk mode while tokens are pending
                st.run_sequence(dev["q"], dev["v"], dev["g"], o)
            assert e.value.status == fwpkm.ERR_STATE
            with pytest.raises(fwpkm.FwpkmError) as e:
                st.forward_chunk(dev["q"], dev["v"], dev["g"], o, 4, seq_stride=w.T)
            assert e.value.status == fwpkm.ERR_STATE
    st.stream_flush()
    assert st.stream_pending() == 0
    st.sync()
    assert torch.equal(o, o_ref)
    assert torch.equal(dev["V"], dev_ref["V"]) and torch.equal(dev["K1"], dev_ref["K1"])
    # after the flush the state takes chunk-mode calls again
    o2 = torch.zeros_like(o)
    st.run_sequence(dev["q"], dev["v"], dev["g"], o2, T=w.C)
    st.sync()


def test_resume_from_a_checkpoint_mid_chunk():
    w, data, gcfg, _ = make_case("mid_key")
    o_ref, dev_ref = reference(w, data, gcfg)
    st, dev = device_state(w, data, gcfg, w.C)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    t0 = w.C + 37  # inside the second chunk
    st.stream_tokens(dev["q"], dev["v"], dev["g"], o, n_tok=t0, seq_stride=w.T)
    pend = st.stream_pending()
    assert pend == 37
    st.sync()
    ck = {key: dev[key].clone() for key in ("K1", "K2", "V")}  # the state after the last write
    # a new handle from the checkpoint: the pending tokens again, then the rest
    st2 = fwpkm.State(gcfg, ck["K1"], ck["K2"], ck["V"], w.C)
    o2 = torch.zeros_like(o)
    a = t0 - pend
    st2.stream_tokens(dev["q"][:, a:], dev["v"][:, a:], dev["g"][:, a:], o2[:, a:], n_tok=w.T - a, seq_stride=w.T)
    st2.stream_flush()
    st2.sync()
    assert torch.equal(o2[:, a:], o_ref[:, a:])
    for key in ("K1", "K2", "V"):
        assert torch.equal(ck[key], dev_ref[key]), key


def test_stream_needs_a_chunk_of_workspace():
    w, data, gcfg, _ = make_case("mid")
    st, dev = device_state(w, data, gcfg, w.C - 1)
    o = torch.zeros(w.M, w.T, w.d_v, device="cuda")
    with pytest.raises(fwpkm.FwpkmError) as e:
        st.stream_tokens(dev["q"], dev["v"], dev["g"], o, n_tok=1, seq_stride=w.T)
    assert e.value.status == fwpkm.ERR_UNSUPPORTED
