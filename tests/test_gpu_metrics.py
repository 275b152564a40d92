"""Addressing metrics on the GPU (fwpkm_addressing_metrics through the C ABI) against the
oracle (oracle/metrics.py) on the same selections.

The row counts, accesses, competitive accesses and invalid entries are integers and must
match exactly; coverage and collision rate are ratios of those integers (one fp64
division on both sides), so they match bit for bit; KLD is summed in another order on
the two sides, so it agrees to 1e-12 (fp64 sums of <= 2^20 terms of size <= S log S).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import WORKLOADS, gen_keys, gen_qvg, gen_values  # noqa: E402

from oracle.metrics import addressing_metrics as oracle_metrics  # noqa: E402

KLD_TOL = 1e-12


def selections(M, T, k, N, seed, zipf=None, invalid=0):
    """Seeded synthetic selections [M][T][k]: uniform slots, or Zipf-skewed slot popularity."""
    rng = np.random.default_rng(seed)
    if zipf is None:
        idx = rng.integers(0, N, size=(M, T, k), dtype=np.int64)
    else:
        ranks = np.minimum(rng.zipf(zipf, size=(M, T, k)), N) - 1
        perm = rng.permutation(N)  # popular ranks land on scattered slots
        idx = perm[ranks]
    idx = idx.astype(np.int32)
    for _ in range(invalid):
        idx[rng.integers(M), rng.integers(T), rng.integers(k)] = rng.choice([-1, N, N + 7])
    return idx


def check(idx, N, window, **kw):
    met, cnt = fwpkm.addressing_metrics(torch.from_numpy(idx).cuda(), N, window, **kw)
    torch.cuda.synchronize()
    met, cnt = met.cpu().numpy(), cnt.cpu().numpy()
    ref_met, ref_cnt = oracle_metrics(idx, N, window)
    np.testing.assert_array_equal(cnt, ref_cnt)
    np.testing.assert_array_equal(met[..., :2], ref_met[..., :2])
    np.testing.assert_allclose(met[..., 2], ref_met[..., 2], rtol=KLD_TOL, atol=KLD_TOL)
    return met, cnt


@pytest.mark.parametrize("M,T,k,N,window,zipf,invalid", [
    (3, 1000, 8, 4096, 256, None, 5),       # ragged last window (1000 = 3 * 256 + 232)
    (2, 777, 32, 65536, 100, 1.3, 0),       # skewed use, many collisions
    (1, 5, 3, 10, 2, None, 2),              # tiny memory, windows of 2 tokens
    (4, 64, 16, 1021, 64, None, 0),         # N not a multiple of 4 (padded counters)
    (1, 300, 1, 1 << 20, 1, None, 0),       # one token per window
])
def test_metrics_match_oracle(M, T, k, N, window, zipf, invalid):
    idx = selections(M, T, k, N, seed=M * 1000 + T, zipf=zipf, invalid=invalid)
    check(idx, N, window)


def test_paper_scale_window_and_batching_is_deterministic():
    # 8 memories of 4096 tokens, top-32 over 2^20 slots: one 32K-token window is longer than
    # the sequence, so each memory is one (ragged) window
    M, T, k, N = 8, 4096, 32, 1 << 20
    idx = selections(M, T, k, N, seed=7, zipf=1.1)
    met, cnt = check(idx, N, 32768)
    # a workspace for one window at a time: same bits
    one = fwpkm.metrics_workspace_size(1, 1, N, 32768)
    ws = torch.empty(one, dtype=torch.uint8, device="cuda")
    met1, cnt1 = fwpkm.addressing_metrics(torch.from_numpy(idx).cuda(), N, 32768, workspace=ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(met1.cpu().numpy(), met)
    np.testing.assert_array_equal(cnt1.cpu().numpy(), cnt)
    # more windows than one batch holds (40 windows of 1024 tokens, batches of 32)
    idx2 = selections(5, 8 * 1024, 4, 4096, seed=8)
    check(idx2, 4096, 1024)


def test_empty_sequence_is_a_no_op():
    met, cnt = fwpkm.addressing_metrics(torch.zeros(2, 0, 4, dtype=torch.int32, device="cuda"), 64, 8)
    assert met.shape == (2, 0, 3) and cnt.shape == (2, 0, 4)


def test_metrics_of_the_read_path():
    # the selections the memory actually made (tensor-core path, key step on) over a sequence
    from dataclasses import replace
    w = replace(WORKLOADS[2], B=2, H=2, T=1000)
    q, v, g = gen_qvg(w)
    K1, K2 = gen_keys(w)
    V = np.stack([gen_values(w, m) for m in range(w.M)])
    bf = lambda x: torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    cfg = fwpkm.make_config(w.n, w.d, w.d_v, w.k, w.C, w.M, True, key_update=True)
    Kd1, Kd2, Vd = (torch.from_numpy(x).cuda() for x in (K1, K2, V))
    st = fwpkm.State(cfg, Kd1, Kd2, Vd, w.T)
    o = torch.empty(w.M, w.T, w.d_v, device="cuda")
    st.run_sequence(bf(q), bf(v), torch.from_numpy(g).cuda(), o)
    idx = torch.empty(w.M, w.T, w.k, dtype=torch.int32, device="cuda")
    st.last_addressing(w.T, idx_out=idx)
    st.sync()
    N = w.n * w.n
    met, cnt = check(idx.cpu().numpy(), N, 256)
    # every token reads k distinct slots, all valid
    assert (cnt[..., 1] == np.array([256, 256, 256, 232]) * w.k).all()
    assert (cnt[..., 3] == 0).all()
    assert ((met[..., 0] > 0) & (met[..., 0] <= 1)).all() and (met[..., 2] >= 0).all()
