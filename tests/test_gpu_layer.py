"""Slow-weight projections on the GPU (fwpkm_layer_in / fwpkm_layer_out through the C ABI)
against the fp64 oracle (oracle/layer.py) on the layer workload's shapes and value
distributions, with ragged row counts (not multiples of the 128-row GEMM tile).

Tolerances follow from the arithmetic: h and W are exact bf16 operands; a folded norm
weight enters the input GEMM as three bf16 pieces (residual <= 2^-27 relative per
weight) and o as two pieces; the accumulation is fp32 over K = d_model (or d_v) terms,
whose rounding error grows like sqrt(K) * 2^-24 * sum_e |x_e W_e| (random-walk bound;
measured ~1e-5 absolute on q of magnitude 2 at K = 2048).  fp32 outputs must agree to
1e-4 relative plus that bound; bf16 outputs (o', or q and v in bf16) are one rounding
of the fp32 result, so they agree to one bf16 unit in the last place (2^-8 relative)
plus the same bound.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from sparse_weight_memory_chunk_b200 import fwpkm  # noqa: E402
from sparse_weight_memory_chunk_b200.inputs import WORKLOADS, bf16_to_f32, f32_to_bf16, gen_layer  # noqa: E402

from oracle import layer as orc  # noqa: E402

RTOL, ATOL = 1e-4, 1e-5
BF16_REL = 2.0 ** -8


def accum_bound(x, W):
    """sqrt(K) * 2^-24 * sum_e |x_e W_e| per output: fp32 accumulation over K terms."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    W = np.abs(np.asarray(W, dtype=np.float64))
    return np.sqrt(x.shape[1]) * 2.0 ** -24 * (x @ W.T)


def assert_within(got, want, bound, rel, what):
    err = np.abs(np.asarray(got, dtype=np.float64) - want)
    lim = rel * np.abs(want) + bound + ATOL
    bad = err > lim
    assert not bad.any(), f"{what}: {int(bad.sum())} outside, worst err {float(err[bad].max())}"


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def bf16_host(t):
    return bf16_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def params(seed, d_model, d, d_v, with_gamma):
    w = WORKLOADS[5]
    L = gen_layer(w, B=1, T=8)
    rng = np.random.default_rng(seed)
    gam = (lambda n: rng.uniform(0.5, 1.5, n).astype(np.float32)) if with_gamma else (lambda n: None)
    p = dict(Wq=L["Wq"][:d, :d_model], Wv=L["Wv"][:d_v, :d_model], wg=L["wg"][:d_model], Wo=L["Wo"][:d_model, :d_v],
             gq=gam(d_model), gv=gam(d_model), gg=gam(d_model), go=gam(d_v),
             bq=rng.normal(0, 0.1, d).astype(np.float32), bv=rng.normal(0, 0.1, d_v).astype(np.float32),
             bg=float(rng.normal(0, 0.5)), bo=rng.normal(0, 0.1, d_model).astype(np.float32))
    return {k: (np.ascontiguousarray(v) if isinstance(v, np.ndarray) else v) for k, v in p.items()}


def make_layer(p, d_model, d, d_v, rows, qv_bf16=False):
    lay = fwpkm.Layer(d_model, d, d_v, rows, qv_bf16=qv_bf16)
    dev = lambda a: None if a is None else torch.from_numpy(a).cuda()  # noqa: E731
    keep = dict(Wq=bf16_dev(p["Wq"]), Wv=bf16_dev(p["Wv"]), wg=bf16_dev(p["wg"]), Wo=bf16_dev(p["Wo"]),
                gq=dev(p["gq"]), gv=dev(p["gv"]), gg=dev(p["gg"]), go=dev(p["go"]),
                bq=dev(p["bq"]), bv=dev(p["bv"]), bo=dev(p["bo"]))
    lay.set_params(keep["Wq"], keep["Wv"], keep["wg"], keep["Wo"], gamma_q=keep["gq"], gamma_v=keep["gv"],
                   gamma_g=keep["gg"], gamma_o=keep["go"], b_q=keep["bq"], b_v=keep["bv"], b_g=p["bg"],
                   b_o=keep["bo"])
    torch.cuda.synchronize()
    return lay, keep


def in_bounds(p, h_bits):
    """Accumulation bounds of q and v (the gate is a dot product of the same length)."""
    D = h_bits.shape[1]
    ones = np.ones(D)
    h = bf16_to_f32(h_bits)
    bq = accum_bound(orc.rmsnorm(h, p["gq"] if p["gq"] is not None else ones, 1e-6), bf16_to_f32(p["Wq"]))
    bv = accum_bound(orc.rmsnorm(h, p["gv"] if p["gv"] is not None else ones, 1e-6), bf16_to_f32(p["Wv"]))
    bg = accum_bound(orc.rmsnorm(h, p["gg"] if p["gg"] is not None else ones, 1e-6),
                     bf16_to_f32(p["wg"])[None, :])[:, 0] * 0.25  # sigmoid' <= 1/4
    return bq, bv, bg


def oracle_in(p, h_bits):
    return orc.project_in(bf16_to_f32(h_bits), p["gq"] if p["gq"] is not None else np.ones(h_bits.shape[1]),
                          bf16_to_f32(p["Wq"]), p["bq"],
                          p["gv"] if p["gv"] is not None else np.ones(h_bits.shape[1]), bf16_to_f32(p["Wv"]), p["bv"],
                          p["gg"] if p["gg"] is not None else np.ones(h_bits.shape[1]), bf16_to_f32(p["wg"]), p["bg"])


@pytest.mark.parametrize("with_gamma", [False, True])
@pytest.mark.parametrize("rows", [1, 300])
def test_project_in_matches_oracle(with_gamma, rows):
    d_model, d, d_v = 2048, 256, 256
    p = params(11, d_model, d, d_v, with_gamma)
    w = WORKLOADS[5]
    h_bits = gen_layer(w, B=1, T=max(rows, 8))["h"][0, :rows]
    lay, _ = make_layer(p, d_model, d, d_v, rows)
    q = torch.empty(rows, d, device="cuda")
    v = torch.empty(rows, d_v, device="cuda")
    g = torch.empty(rows, device="cuda")
    lay.project_in(bf16_dev(h_bits), q, v, g)
    lay.sync()
    qo, vo, go = oracle_in(p, h_bits)
    bq, bv, bg = in_bounds(p, h_bits)
    assert_within(q.cpu().numpy(), qo, bq, RTOL, "q")
    assert_within(v.cpu().numpy(), vo, bv, RTOL, "v")
    assert_within(g.cpu().numpy(), go, bg, RTOL, "g")


def test_project_in_bf16_outputs():
    d_model, d, d_v, rows = 2048, 256, 256, 200
    p = params(12, d_model, d, d_v, True)
    h_bits = gen_layer(WORKLOADS[5], B=1, T=rows)["h"][0]
    lay, _ = make_layer(p, d_model, d, d_v, rows, qv_bf16=True)
    q = torch.empty(rows, d, device="cuda", dtype=torch.bfloat16)
    v = torch.empty(rows, d_v, device="cuda", dtype=torch.bfloat16)
    g = torch.empty(rows, device="cuda")
    lay.project_in(bf16_dev(h_bits), q, v, g)
    lay.sync()
    qo, vo, _ = oracle_in(p, h_bits)
    bq, bv, _ = in_bounds(p, h_bits)
    assert_within(bf16_host(q), qo, bq, BF16_REL, "q (bf16)")
    assert_within(bf16_host(v), vo, bv, BF16_REL, "v (bf16)")


@pytest.mark.parametrize("with_gamma", [False, True])
def test_project_out_matches_oracle(with_gamma):
    d_model, d, d_v, rows = 2048, 256, 256, 333
    p = params(13, d_model, d, d_v, with_gamma)
    rng = np.random.default_rng(14)
    o = (rng.normal(size=(rows, d_v)) * rng.uniform(0.01, 3, size=(rows, 1))).astype(np.float32)
    lay, _ = make_layer(p, d_model, d, d_v, rows)
    out = torch.empty(rows, d_model, device="cuda", dtype=torch.bfloat16)
    lay.project_out(torch.from_numpy(o).cuda(), out)
    lay.sync()
    go = p["go"] if p["go"] is not None else np.ones(d_v)
    want = orc.project_out(o, go, bf16_to_f32(p["Wo"]), p["bo"])
    bound = accum_bound(orc.rmsnorm(o, go, 1e-6), bf16_to_f32(p["Wo"]))
    assert_within(bf16_host(out), want, bound, BF16_REL, "o'")


def test_layer_argument_checks():
    lay = fwpkm.Layer(2048, 256, 256, 16)
    q = torch.empty(16, 256, device="cuda")
    with pytest.raises(fwpkm.FwpkmError) as e:
        lay.project_in(torch.empty(16, 2048, device="cuda", dtype=torch.bfloat16), q, q, q[:, 0])
    assert e.value.status == fwpkm.ERR_STATE  # parameters not set yet
    lay.project_in(q, q, q, q, rows=0)  # no-op
    with pytest.raises(fwpkm.FwpkmError) as e:
        lay.project_out(q, q, rows=17)
    assert e.value.status == fwpkm.ERR_INVALID_ARG
