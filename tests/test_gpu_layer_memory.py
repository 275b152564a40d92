"""The whole layer on the GPU (fwpkm_run_layer through the C ABI) against the oracle chain
on the layer workload's defining inputs: hidden states from Gaussian clusters with
Zipf-skewed cluster weights (the workload's 64 clusters, s = 1.1, and a hotter variant
of the same recipe, 4 clusters with s = 2, in which one cluster holds ~70% of the
tokens), the workload's shapes (n = 512, d = d_v = 256, k = 32, C = 256, bf16 q/v, so
the memory takes the tensor-core scoring path) and the entropy key update on, at
reduced B and T with a ragged last chunk.

Source: "快速权重积键值记忆 Fast-weight Product Key Memory" (rainbus summary), method
steps 1-5: q, v, g from h through RMSNorm + Linear, the chunk-sequential memory, the
output projection.  Checked, element by element:
  * q, v, g left by the call against the oracle's projections (oracle/layer.py);
  * the memory, chunk by chunk, against the oracle (oracle.chunk) on those same q, v, g
    from the same initial state (after every chunk: o, weights, K1, K2, the key step,
    value rows), then the call's o and final state bit-for-bit against that run;
  * o' against the oracle's output projection of the call's o.
Skewed slot use is what these inputs are for, so the test also asserts that it reached
the two skew paths of the write: a chunk whose (slot, token) pairs overflow one hash
bucket of the pair sort (more than 128 keys: ranked by a whole CTA instead of a warp),
and, in the hot variant, a row read by at least half the chunk's tokens (one segment of
the write carried across many batches and windows of its warp).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import (WORKLOADS, Workload, bf16_to_f32, gen_keys, gen_layer,  # noqa: E402
                                                    gen_values)

import oracle  # noqa: E402
from oracle import layer as orc  # noqa: E402
from test_gpu_layer import BF16_REL, RTOL, accum_bound, assert_within, bf16_dev, bf16_host  # noqa: E402
from test_gpu_parity import compare_streaming  # noqa: E402

SORT_BUCKET_CAP = 128  # largest hash bucket the pair sort ranks in place


def bucket_sizes(slots):
    """Sizes of the pair sort's hash buckets for one chunk's slot list.  This mirrors the
    kernel's bucketing (multiplicative hash of the slot, ~64 keys per bucket, bucket count
    a power of two >= keys / 64) so the test can tell which path of the sort ran."""
    P = slots.size
    ppad = 256
    while ppad < P:
        ppad *= 2
    nb = ppad // 64
    lg = int(np.log2(nb))
    b = ((slots.astype(np.uint64) * np.uint64(2654435761)) & np.uint64(0xFFFFFFFF)) >> np.uint64(32 - lg)
    return np.bincount(b.astype(np.int64), minlength=nb)


@pytest.mark.parametrize("variant", ["workload", "hot"])
def test_run_layer_matches_oracle_chain(variant):
    w5 = WORKLOADS[5]
    B, T = 2, 520
    clusters, zipf = (64, 1.1) if variant == "workload" else (4, 2.0)
    L = gen_layer(w5, B=B, T=T, clusters=clusters, zipf=zipf)
    K1, K2 = gen_keys(w5, M=B)
    V = np.stack([gen_values(w5, m) for m in range(B)])
    D, d, dv, C, k = w5.d_model, w5.d, w5.d_v, w5.C, w5.k
    gcfg = fwpkm.make_config(w5.n, d, dv, k, C, B, True, key_update=True)
    ocfg = oracle.make_cfg(w5.n, d, dv, k, C, key_update=True)

    lay = fwpkm.Layer(D, d, dv, B * T, qv_bf16=True)
    Wd = {name: bf16_dev(L[name]) for name in ("Wq", "Wv", "wg", "Wo")}
    lay.set_params(Wd["Wq"], Wd["Wv"], Wd["wg"], Wd["Wo"])
    K1d, K2d, Vd = (torch.from_numpy(x).cuda() for x in (K1, K2, V))
    st = fwpkm.State(gcfg, K1d, K2d, Vd, T)
    h = bf16_dev(L["h"])
    o_out = torch.empty(B, T, D, device="cuda", dtype=torch.bfloat16)
    scratch = lay.run_layer(st, h, o_out)
    st.sync()
    lay.sync()
    q, v, g, o = (x.clone() for x in fwpkm.run_layer_parts(gcfg, T, scratch))

    # method step 1 against the oracle's projections
    hf = bf16_to_f32(L["h"].reshape(B * T, D))
    ones = np.ones(D)
    Wq, Wv, wg, Wo = (bf16_to_f32(L[name]) for name in ("Wq", "Wv", "wg", "Wo"))
    qo, vo, go = orc.project_in(hf, ones, Wq, None, ones, Wv, None, ones, wg, 0.0)
    nrm = orc.rmsnorm(hf, ones, 1e-6)
    assert_within(bf16_host(q.reshape(B * T, d)), qo, accum_bound(nrm, Wq), BF16_REL, "q")
    assert_within(bf16_host(v.reshape(B * T, dv)), vo, accum_bound(nrm, Wv), BF16_REL, "v")
    assert_within(g.reshape(-1).cpu().numpy(), go, accum_bound(nrm, wg[None, :])[:, 0] * 0.25, RTOL, "g")

    # the memory, chunk by chunk, on the call's own q, v, g from the initial state
    def bits(x):
        return x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    w = Workload("layer_chain", w5.n, d, dv, k, T, C, B, 1, "bf16", True, w5.seed, "sigmoid", "normal002")
    data = (bits(q), bits(v), g.cpu().numpy(), K1, K2, V)
    res = compare_streaming(f"layer_{variant}", w, data, gcfg, ocfg)
    print(f"layer chain ({variant}): near-ties {res['ties']}")
    assert torch.equal(o.cpu(), res["o"]), "run_layer o differs from the chunk-by-chunk memory"
    assert torch.equal(Vd, res["V"]), "run_layer V differs from the chunk-by-chunk memory"
    assert torch.equal(K1d.cpu(), res["K1"]) and torch.equal(K2d.cpu(), res["K2"])

    # method step 3 (output side) against the oracle's projection of the call's o
    of = o.reshape(B * T, dv).cpu().numpy()
    want = orc.project_out(of, np.ones(dv), Wo, None)
    assert_within(bf16_host(o_out.reshape(B * T, D)), want, accum_bound(orc.rmsnorm(of, np.ones(dv), 1e-6), Wo),
                  BF16_REL, "o'")

    # the skew paths were taken (pair tokens: all but the last token of the sequence)
    max_bucket, max_nread = 0, 0
    for ci, idx in enumerate(res["idx"]):
        for m in range(B):
            last = ci == len(res["idx"]) - 1
            pairs = idx[m][:-1] if last else idx[m]
            slots = pairs.reshape(-1)
            max_bucket = max(max_bucket, int(bucket_sizes(slots).max()))
            max_nread = max(max_nread, int(np.unique(slots, return_counts=True)[1].max()))
    print(f"layer chain ({variant}): largest sort bucket {max_bucket}, largest N_read {max_nread}")
    assert max_bucket > SORT_BUCKET_CAP, "no chunk reached the pair sort's oversized-bucket path"
    if variant == "hot":
        assert max_nread >= C // 2, "no row was read by half a chunk's tokens"


def test_run_layer_full_size():
    """The layer workload at its full size and seed (B = 16 sequences, T = 4096, d_model =
    2048, n = 512, 64 Zipf-weighted clusters), through fwpkm_run_layer as the benchmark
    times it: q, v, g on 512 sampled rows against the oracle's projections, the memory chunk
    by chunk against the oracle on the call's own q, v, g, the call's o and final state bit
    for bit against that run, and o' on the sampled rows against the oracle's output
    projection of the call's o."""
    w5 = WORKLOADS[5]
    B, T = w5.B, w5.T
    L = gen_layer(w5, B=B, T=T)
    K1, K2 = gen_keys(w5, M=B)
    V = np.stack([gen_values(w5, m) for m in range(B)])
    D, d, dv, C, k = w5.d_model, w5.d, w5.d_v, w5.C, w5.k
    gcfg = fwpkm.make_config(w5.n, d, dv, k, C, B, True, key_update=True)
    ocfg = oracle.make_cfg(w5.n, d, dv, k, C, key_update=True)
    lay = fwpkm.Layer(D, d, dv, B * T, qv_bf16=True)
    Wd = {name: bf16_dev(L[name]) for name in ("Wq", "Wv", "wg", "Wo")}
    lay.set_params(Wd["Wq"], Wd["Wv"], Wd["wg"], Wd["Wo"])
    K1d, K2d, Vd = (torch.from_numpy(x).cuda() for x in (K1, K2, V))
    st = fwpkm.State(gcfg, K1d, K2d, Vd, T)
    o_out = torch.empty(B, T, D, device="cuda", dtype=torch.bfloat16)
    scratch = lay.run_layer(st, bf16_dev(L["h"]), o_out)
    st.sync()
    lay.sync()
    q, v, g, o = (x.clone() for x in fwpkm.run_layer_parts(gcfg, T, scratch))

    rows = np.random.default_rng(5).choice(B * T, 512, replace=False)
    ri = torch.from_numpy(rows).cuda()
    hf = bf16_to_f32(L["h"].reshape(B * T, D)[rows])
    ones = np.ones(D)
    Wq, Wv, wg, Wo = (bf16_to_f32(L[name]) for name in ("Wq", "Wv", "wg", "Wo"))
    qo, vo, go = orc.project_in(hf, ones, Wq, None, ones, Wv, None, ones, wg, 0.0)
    nrm = orc.rmsnorm(hf, ones, 1e-6)
    assert_within(bf16_host(q.reshape(B * T, d)[ri]), qo, accum_bound(nrm, Wq), BF16_REL, "q")
    assert_within(bf16_host(v.reshape(B * T, dv)[ri]), vo, accum_bound(nrm, Wv), BF16_REL, "v")
    assert_within(g.reshape(-1).cpu().numpy()[rows], go, accum_bound(nrm, wg[None, :])[:, 0] * 0.25, RTOL, "g")

    def bits(x):
        return x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    w = Workload("layer_full", w5.n, d, dv, k, T, C, B, 1, "bf16", True, w5.seed, "sigmoid", "normal002")
    res = compare_streaming("layer_full", w, (bits(q), bits(v), g.cpu().numpy(), K1, K2, V), gcfg, ocfg)
    print(f"layer full size: near-ties {res['ties']}")
    assert torch.equal(o.cpu(), res["o"]), "run_layer o differs from the chunk-by-chunk memory"
    assert torch.equal(Vd, res["V"].cuda() if not res["V"].is_cuda else res["V"]), "run_layer V differs"
    assert torch.equal(K1d.cpu(), res["K1"]) and torch.equal(K2d.cpu(), res["K2"])
    of = o.reshape(B * T, dv)[ri].cpu().numpy()
    want = orc.project_out(of, np.ones(dv), Wo, None)
    assert_within(bf16_host(o_out.reshape(B * T, D)[ri]), want,
                  accum_bound(orc.rmsnorm(of, np.ones(dv), 1e-6), Wo), BF16_REL, "o'")


def test_run_layer_argument_checks():
    w5 = WORKLOADS[5]
    B, T = 1, 64
    gcfg = fwpkm.make_config(w5.n, w5.d, w5.d_v, w5.k, w5.C, B, True, key_update=True)
    K1, K2 = (torch.zeros(B, w5.n, w5.h, device="cuda") for _ in range(2))
    V = torch.zeros(B, w5.N, w5.d_v, device="cuda")
    st = fwpkm.State(gcfg, K1, K2, V, T)
    lay = fwpkm.Layer(w5.d_model, w5.d, w5.d_v, B * T, qv_bf16=True)
    L = gen_layer(w5, B=1, T=8)
    Wd = {name: bf16_dev(L[name]) for name in ("Wq", "Wv", "wg", "Wo")}
    lay.set_params(Wd["Wq"], Wd["Wv"], Wd["wg"], Wd["Wo"])
    h = torch.zeros(B, T, w5.d_model, device="cuda", dtype=torch.bfloat16)
    out = torch.empty_like(h)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fwpkm.FwpkmError) as e:
        lay.run_layer(st, h, out, scratch=small)
    assert e.value.status == fwpkm.ERR_WORKSPACE
    lay32 = fwpkm.Layer(w5.d_model, w5.d, w5.d_v, B * T, qv_bf16=False)  # q/v dtype differs from the state's
    lay32.set_params(Wd["Wq"], Wd["Wv"], Wd["wg"], Wd["Wo"])
    with pytest.raises(fwpkm.FwpkmError) as e:
        lay32.run_layer(st, h, out)
    assert e.value.status == fwpkm.ERR_INVALID_ARG
    with pytest.raises(fwpkm.FwpkmError) as e:  # more tokens than the state was made for
        lay.run_layer(st, torch.zeros(B, T + 1, w5.d_model, device="cuda", dtype=torch.bfloat16),
                      torch.empty(B, T + 1, w5.d_model, device="cuda", dtype=torch.bfloat16))
    assert e.value.status == fwpkm.ERR_INVALID_ARG
    lay.run_layer(st, h, out, T=0)  # no-op
