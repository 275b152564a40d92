"""FwPKM retrieve + chunk-write loop: throughput on B200 against the HBM roofline.

One step = one pass of the whole hot path (addressing, gather + gated output,
sorted write, entropy key step) over one batch of the workload, i.e. one call of
fwpkm_run_sequence over B sequences x H heads x T tokens.  Default workload: the
paper-scale memory (n=1024 -> N=1,048,576 slots, d=d_v=256, k=32, C=256, B=4, H=2,
T=4096, bf16 q/v, fp32 state, key update on).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload paper|mid|tiny|needle|layer]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

The default run measures the paper-scale workload (the headline `value`) and then the
other four workloads (tiny, mid, needle at n_iter = 1, 2 and 4 with its read-back, and
the full layer), each reported under `configs` in the same JSON line with its own
step time, throughput, roofline fractions, clocks and a selection check against the
oracle.  `--workload X` measures X alone; `--no-configs` skips the other workloads.

Multi-GPU (torchrun): every rank runs its own independent memories (different
sequences); there is no collective on the data path ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_weight_memory_chunk_b200.inputs import (WORKLOADS, gen_keys, gen_layer, gen_needles, gen_qvg,  # noqa: E402
                                                    gen_values)

BY_NAME = {w.name: (i, w) for i, w in WORKLOADS.items()}

# DRAM bytes (read + write) per launch and per memory of the paper-scale kernels, from one
# ncu capture of a 2-memory case of the paper shapes (the capture and its command are kept
# with the profiles): dram__bytes_read.sum + dram__bytes_write.sum of the captured launch
# / 2; a full launch scales with the memories it processes (each memory's work is the
# same).  A kernel changed since that capture is missing here and reports null.
TRAFFIC = {
    "fused": {"per_mem": (5_873_920 + 0) / 2},
    "topk": {"per_mem": (4_266_240 + 0) / 2},
    "sort": {"per_mem": (97_024 + 0) / 2},
    "gather": {"per_mem": (15_792_128 + 0) / 2},
    "write": {"per_mem": (16_094_464 + 0) / 2},
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None, choices=["tiny", "mid", "paper", "needle", "layer"],
                    help="measure this workload alone (default: paper, plus the others under `configs`)")
    ap.add_argument("--n-iter", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-metrics", action="store_true", help="skip the addressing-metrics measurement")
    ap.add_argument("--no-stream", action="store_true", help="skip the token-at-a-time measurement")
    ap.add_argument("--no-configs", action="store_true", help="measure the headline workload only")
    ap.add_argument("--config-steps", type=int, default=5, help="timed steps of each extra workload")
    ap.add_argument("--batch", type=int, default=None, help="override the number of sequences B (profiling)")
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling)")
    ap.add_argument("--kernel", default=None,
                    help="kernel kind timed for the roofline (default: the slowest kind, found by one timed step "
                         "each; 'none': no timing events in the timed region)")
    return ap.parse_args()


def describe(w, n_iter):
    lay = (f", d_model={w.d_model} bf16 hidden states through RMSNorm+Linear in/out projections"
           if w.d_model else "")
    ndl = f", {w.needles} planted needles" if w.name == "needle" else ""
    return (f"{w.name}: n={w.n} (N={w.N:,} slots), d={w.d}, d_v={w.d_v}, k={w.k}, C={w.C}, "
            f"B={w.B} x H={w.H} memories, T={w.T}, {w.qv} q/v, fp32 V/K, key update "
            f"{'on' if w.key_update else 'off'}, n_iter={n_iter}{lay}{ndl}")


# --------------------------------------------------------------------------- oracle leg
_SAMPLE_CACHE = {}


def host_cpu():
    """(hardware threads of this host, CPU model) for the CPU-baseline record."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def _oracle_inputs(w, seqs, T):
    """fp64 inputs, initial fp32 state and (layer workload) W_o of sequences 0..seqs-1."""
    from sparse_weight_memory_chunk_b200.inputs import bf16_to_f32
    M = seqs * w.H
    K1, K2 = gen_keys(w, M=M)
    V = np.stack([gen_values(w, m) for m in range(M)])
    if w.d_model:
        # layer workload: the projections' oracle turns the hidden states into q, v, g
        from oracle import layer as orc_layer
        L = gen_layer(w, B=seqs, T=T)
        ones = np.ones(w.d_model)
        qs, vs, gs = [], [], []
        for b in range(seqs):
            qf, vf, gf = orc_layer.project_in(bf16_to_f32(L["h"][b]), ones, bf16_to_f32(L["Wq"]), None, ones,
                                              bf16_to_f32(L["Wv"]), None, ones, bf16_to_f32(L["wg"]), 0.0)
            qs.append(qf); vs.append(vf); gs.append(gf)
        return np.stack(qs), np.stack(vs), np.stack(gs), K1, K2, V, bf16_to_f32(L["Wo"])
    q, v, g = gen_qvg(w, M=M)
    if w.needles:
        gen_needles(w, q, v)  # planted over the whole stream, as on the GPU; the sample reads its head
    q, v, g = q[:, :T], v[:, :T], g[:, :T]
    qf = (bf16_to_f32(q) if w.qv == "bf16" else q).astype(np.float64)
    vf = (bf16_to_f32(v) if w.qv == "bf16" else v).astype(np.float64)
    return qf, vf, g.astype(np.float64), K1, K2, V, None


def oracle_sample(w, n_chunks, seqs=None, threads=None):
    """CPU-baseline leg: time the oracle (as it stands) on sequences 0..seqs-1 (every head),
    first n_chunks chunks, on all host threads (memories in parallel; with more threads
    than memories each chunk's read phase is split over token ranges).

    The inputs are drawn once per process; every call starts from a fresh copy of the
    initial state (the oracle updates it in place)."""
    import oracle
    cores, model = host_cpu()
    seqs = seqs or w.B
    T = min(w.T, n_chunks * w.C)
    key = (w.name, T, seqs)
    if key not in _SAMPLE_CACHE:
        oracle.build()
        _SAMPLE_CACHE[key] = _oracle_inputs(w, seqs, T)
    qf, vf, gf, K1, K2, V, Wo = _SAMPLE_CACHE[key]
    k1, k2, vv = K1.copy(), K2.copy(), V.copy()
    cfg = oracle.make_cfg(w.n, w.d, w.d_v, w.k, w.C, key_update=w.key_update)
    t0 = time.perf_counter()
    res, used = oracle.run_sequence_multi(cfg, qf, vf, gf, k1, k2, vv, 1, nthreads=threads or cores)
    if Wo is not None:
        from oracle import layer as orc_layer
        for b in range(seqs):
            orc_layer.project_out(res[b], np.ones(w.d_v), Wo, None)
    dt = time.perf_counter() - t0
    M = seqs * w.H
    return dict(tokens=seqs * T, seconds=dt, threads=used, cpu_model=model, host_threads=cores,
                sample=f"sequences 0..{seqs - 1} ({M} memories of N={w.N:,} slots), tokens 0..{T - 1} "
                       f"({n_chunks} chunks of {w.C}), {used} threads of {cores} on {model}")


TIE_REL = 1e-6


def selection_check(w, q_bits, K1, K2, idx):
    """Part of the CPU-baseline leg: the GPU's slot lists of chunk 0 (initial keys) against
    the oracle's, per token of memories 0..H-1 (sequence 0): exact, near-tie (at every rank
    the GPU's slot score, recomputed in fp64, within 1e-6 max(1, |S|) of the oracle's) or
    mismatch."""
    import math

    import oracle
    from sparse_weight_memory_chunk_b200.inputs import bf16_to_f32
    cfg = oracle.make_cfg(w.n, w.d, w.d_v, w.k, w.C)
    h, n = w.h, w.n
    out = {"tokens": 0, "exact": 0, "near_tie": 0, "mismatch": 0}
    for m in range(idx.shape[0]):
        qm = (bf16_to_f32(q_bits[m]) if q_bits.dtype == np.uint16 else q_bits[m]).astype(np.float64)
        for t in range(idx.shape[1]):
            D1 = oracle.subkey_dist(cfg, qm[t, :h], K1[m])
            D2 = oracle.subkey_dist(cfg, qm[t, h:], K2[m])
            I_o, S_o, _ = oracle.select(cfg, D1, D2)
            out["tokens"] += 1
            I_g = idx[m, t]
            if np.array_equal(I_o, I_g):
                out["exact"] += 1
                continue
            ok = len(set(I_g.tolist())) == w.k and I_g.min() >= 0 and I_g.max() < n * n
            if ok:
                S_g = np.array([-math.log(cfg.eps_idw + D1[s // n]) - math.log(cfg.eps_idw + D2[s % n]) for s in I_g])
                ok = bool(np.all(np.abs(S_g - S_o) <= TIE_REL * np.maximum(1.0, np.abs(S_o))))
            out["near_tie" if ok else "mismatch"] += 1
    out["definition"] = ("chunk 0 of sequence 0's memories from the initial keys: GPU slot lists against the "
                         "oracle's (exact; near-tie = scores within 1e-6 relative at every rank; mismatch)")
    return out


def run_reference(args, w, rank):
    if rank != 0:
        return
    n_chunks = 8 if w.name in ("paper", "needle") else 16
    times = []
    info = None
    for i in range(args.warmup + args.steps):
        info = oracle_sample(w, n_chunks, seqs=None if w.name in ("paper", "mid", "tiny") else 1)
        if i >= args.warmup:
            times.append(info["seconds"])
    ms = 1000.0 * sum(times) / len(times)
    val = info["tokens"] / (ms / 1000.0)
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(w, 1), "sample": info["sample"]},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": info["threads"], "kind": "oracle",
                             "sample": info["sample"], "host_threads": info["host_threads"],
                             "cpu_model": info["cpu_model"]},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


METRIC = "FwPKM layer tokens/s (retrieve+chunk write) at 1M slots; % of HBM roofline"


# --------------------------------------------------------------------------- clocks
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        for line in out.strip().splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"), p[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- ours
def algorithmic_bytes(w, idx, T):
    """B_VK of one step (each touched V row loaded once and stored once, K read + written)
    and the gather kernel's bytes per launch.  idx: [M][T][k] final addressing."""
    import torch
    C, k, dv = w.C, w.k, w.d_v
    U_total = 0
    for t0 in range(0, T, C):
        t1 = min(T, t0 + C)
        npair = (t1 - t0) - (1 if t1 == T else 0)
        blk = idx[:, t0:t0 + npair, :].reshape(idx.shape[0], -1)
        s, _ = torch.sort(blk, dim=1)
        U_total += int((s[:, 1:] != s[:, :-1]).sum().item()) + blk.shape[0]
    key_bytes = (2 * 4 * w.n * w.d) * w.M * ((T + C - 1) // C) if w.key_update else 0
    b_vk = 2 * U_total * dv * 4 + key_bytes
    es = 2 if w.qv == "bf16" else 4
    gather_per_token = k * dv * 4 + k * 8 + dv * es + dv * 4
    return b_vk, gather_per_token, U_total


# --------------------------------------------------------------------------- ranks
def rank_workload(w, rank):
    """Each rank runs its own independent memories: rank r draws its sequences with seed
    offset 1000 r (rank 0 is the workload itself)."""
    from dataclasses import replace
    return replace(w, seed=w.seed + 1000 * rank) if rank else w


def max_over_ranks(x, world, device):
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, world, ms_step):
    """Whole-job units per second: every rank processes units_per_rank_step per step."""
    return units_per_rank_step * world / (ms_step / 1000.0)


def load_peaks():
    peaks = {}
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        peaks = json.load(open(pp))
    return (float(peaks.get("hbm_gbs", 6650.0)), float(peaks.get("bf16_tflops_sustained", 1400.0)),
            "measured" if peaks else "fallback", peaks)


def measure(args, w, rank, world, local_rank, n_iter, steps, warmup, full):
    """Measure one workload: `steps` timed steps after `warmup` (each step one call of the
    public entry point over the whole batch: fwpkm_run_sequence, or fwpkm_run_layer for
    the layer workload).  `full`: also the end-to-end, addressing-metrics and
    token-at-a-time measurements and the CPU-baseline leg's timing.  Returns the line."""
    import torch
    import torch.distributed as dist

    from sparse_weight_memory_chunk_b200 import fwpkm
    dev = torch.device("cuda", local_rank)
    hbm_peak, tc_peak, peak_src, peaks = load_peaks()

    # inputs (per-rank independent sequences: seed offset by rank)
    wr = rank_workload(w, rank)
    q, v, g = gen_qvg(wr)
    K1, K2 = gen_keys(wr)
    needles = gen_needles(wr, q, v) if w.needles else None

    def to_dev(x):
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(x).to(dev)

    K1d, K2d = to_dev(K1), to_dev(K2)
    Vd = torch.empty(w.M, w.N, w.d_v, device=dev)
    for m in range(w.M):
        Vd[m].copy_(torch.from_numpy(gen_values(wr, m)))
    cfg = fwpkm.make_config(w.n, w.d, w.d_v, w.k, w.C, w.M, w.qv == "bf16", key_update=w.key_update)
    st = fwpkm.State(cfg, K1d, K2d, Vd, w.T)
    o = torch.empty(w.M, w.T, w.d_v, device=dev)
    stream = torch.cuda.current_stream()
    layer = None
    if w.d_model:
        # full layer through fwpkm_run_layer: h -> (RMSNorm + Linear) q, v, g -> memory ->
        # (RMSNorm + Linear) o'; the memory's q, v, g, o live in the call's scratch
        Ld = gen_layer(wr)
        hd = to_dev(Ld["h"])
        layer = fwpkm.Layer(w.d_model, w.d, w.d_v, w.M * w.T, qv_bf16=w.qv == "bf16", device=dev)
        lw = {k_: to_dev(Ld[k_]) for k_ in ("Wq", "Wv", "wg", "Wo")}
        layer.set_params(lw["Wq"], lw["Wv"], lw["wg"], lw["Wo"])
        scratch = torch.empty(fwpkm.run_layer_scratch_size(cfg, w.T), dtype=torch.uint8, device=dev)
        qd, vd, gd, o = fwpkm.run_layer_parts(cfg, w.T, scratch)
        o_out = torch.empty(w.M, w.T, w.d_model, device=dev, dtype=torch.bfloat16)

        def step():
            layer.run_layer(st, hd, o_out, n_iter=n_iter, scratch=scratch)
    else:
        qd, vd, gd = to_dev(q), to_dev(v), to_dev(g)

        def step():
            st.run_sequence(qd, vd, gd, o, n_iter=n_iter)
    K1_init, K2_init = K1d.clone(), K2d.clone()
    state0 = (Vd.clone(),) if needles is not None else None

    # warm-up; find the dominant kernel kind by timing each kind once
    for _ in range(max(warmup, 1)):
        step()
    kinds = {}
    if args.kernel is None:
        for name in ("gather", "write", "score", "topk", "cartesian", "sort", "pbar", "wbuild", "address", "fused",
                     "value_loop", "prep", "other"):
            st.profile_kernel(name)
            step()
            ms, n = st.kernel_time()
            kinds[name] = (ms, n)
        st.profile_kernel(0)
        dominant = max(kinds, key=lambda k_: kinds[k_][0])
    else:
        dominant = args.kernel
    # the timed region replays the plain graph, and in its last step the same graph with
    # CUDA events around every launch of the dominant kernel ("none": never)
    timed_kind = 0 if dominant == "none" else dominant
    for kind_ in (timed_kind, 0):  # capture both graphs outside the timed region
        st.profile_kernel(kind_)
        step()
    st.sync()

    clocks = Clocks(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    l0 = fwpkm.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for s_ in range(steps):
        if s_ == steps - 1:
            st.profile_kernel(timed_kind)
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    launches = fwpkm.launch_count() - l0
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms_total = ev0.elapsed_time(ev1)
    dom_ms, dom_n = st.kernel_time()
    st.profile_kernel(0)
    st.sync()
    if layer is not None:
        layer.sync()
    ms_step = max_over_ranks(ms_total / steps, world, dev)
    tokens_per_step = w.B * w.T * n_iter
    value = job_throughput(tokens_per_step, world, ms_step)

    # algorithmic traffic of the step (measured unique rows) and roofline
    idx = torch.empty(w.M, w.T, w.k, dtype=torch.int32, device=dev)
    st.last_addressing(w.T, idx_out=idx)
    torch.cuda.synchronize()
    b_vk, gather_per_token, U = algorithmic_bytes(w, idx, w.T)
    b_vk *= n_iter
    flops = 2 * w.n * w.d * w.M * w.T * n_iter * (2 if w.key_update else 1)
    if w.d_model:  # the slow-weight projections (in: q, v, gate; out: o')
        flops += 2 * w.M * w.T * w.d_model * (w.d + w.d_v + 1 + w.d_v)
    t_roof = max(b_vk / (hbm_peak * 1e9), flops / (tc_peak * 1e12))
    step_frac = t_roof / (ms_step / 1000.0)
    nchunks = (w.T + w.C - 1) // w.C
    # algorithmic work of one step of each kernel kind, as (bytes against HBM, FLOPs against
    # the tensor peak, ALU ops against the fp32 lanes); a launch's share is the step's work
    # over the kind's launches in the step.  The addressing of frozen keys runs once per
    # call, the rest once per pass.
    alu_peak = 148 * 128 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12  # Tops/s
    cand = sum(w.k // (i + 1) for i in range(w.k))  # staircase candidates per token-memory
    P, h = 2 * w.M, w.d // 2
    es = 2 if w.qv == "bf16" else 4
    tm_val = w.M * w.T * n_iter                                # token-memories through the value path
    tm_adr = w.M * w.T * (n_iter if w.key_update else 1)       # token-memories addressed
    gather_b = gather_per_token * tm_val
    write_b = 2 * U * w.d_v * 4 * n_iter
    tc = w.qv == "bf16" and h in (64, 128)                     # tensor-core scoring (else CUDA cores)
    pieces = 3 * P * w.n * h * 2 if tc else 0                  # bf16 key pieces read per scoring launch
    work = {
        "gather": (gather_b, 0, 0),
        "write": (write_b, 0, 0),
        # tensor cores: distance rows written + key pieces read per launch (added below), 2 n d
        # FLOP per token-memory; CUDA cores (scoring fused with the per-half top-k): keys and
        # queries read, the same products as fp32 FMAs
        "score": ((2 * w.n * 4 * tm_adr, 2 * w.n * w.d * tm_adr, 0) if tc else
                  (w.d * es * tm_adr, 0, 2 * w.n * w.d * tm_adr)),
        "address": (0, 2 * w.n * w.d * tm_adr, 0),
        "topk": (2 * w.n * 4 * tm_adr, 0, 0),                  # distance rows read
        "pbar": (2 * w.n * 4 * tm_adr, 0, 0),                  # distance rows read
        "wbuild": (2 * w.n * 4 * tm_adr * 2 + 2 * w.n * 2 * 2 * tm_adr, 0, 0),  # rows read twice, 2 bf16 pieces out
        "sort": (w.k * tm_adr * (4 + 8), 0, 0),                # slots read, pair keys written
        "cartesian": (0, 0, cand * 2 * tm_adr),                # one add + one compare per candidate
        # one-launch addressing step: distance rows written, half-queries read (both layouts);
        # per launch the key pieces read and, with the key step, keys read + written and
        # their pieces rewritten; FLOPs of the scoring and key-step contractions
        "fused": (2 * w.n * 4 * tm_adr + 2 * 2 * h * es * tm_adr,
                  2 * w.n * w.d * tm_adr * (2 if w.key_update else 1), 0),
        # the persistent value loop (frozen keys): every chunk's gather and write
        "value_loop": (gather_b + write_b, 0, 0),
    }
    per_launch_extra = {"score": pieces,
                        "fused": pieces + ((2 * P * w.n * h * 4 + 3 * P * w.n * h * 2) if w.key_update else 0)}

    def kind_roofline(kind, ms, n):
        if kind not in work or n == 0:
            return None
        b, f, a = work[kind]
        b = b / n + per_launch_extra.get(kind, 0)
        f, a = f / n, a / n
        avg_s = (ms / 1000.0) / n
        # the bound is the roofline the launch's work takes longest on
        t = {"hbm": b / (hbm_peak * 1e9), "tensor": f / (tc_peak * 1e12), "alu": a / (alu_peak * 1e12)}
        bound = max(t, key=t.get)
        per_launch = {"hbm": b, "tensor": f, "alu": a}[bound]
        if bound == "hbm":
            ach, peak, unit, src = per_launch / avg_s / 1e9, hbm_peak, "GB/s", "hbm_gbs"
        elif bound == "tensor":
            ach, peak, unit, src = per_launch / avg_s / 1e12, tc_peak, "TFLOP/s", "bf16_tflops_sustained"
        else:
            ach, peak, unit, src = per_launch / avg_s / 1e12, alu_peak, "Tops/s", "148 SMs x 128 fp32 lanes x max clock"
        traffic = TRAFFIC.get(kind, {}).get("per_mem", 0) * w.M if w.name == "paper" else 0
        return {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
                "traffic": traffic or None,
                "kernel": kind, "peak_source": f"{peak_src if bound != 'alu' else 'derived'} ({src})",
                "avg_launch_us": avg_s * 1e6, "launches_timed": n,
                "algorithmic_per_launch": per_launch,
                "roofline_us": {k_: round(v_ * 1e6, 3) for k_, v_ in t.items() if v_ > 0}}

    roof = kind_roofline(dominant, dom_ms, dom_n) or {"bound": None, "kernel": dominant}
    kind_table = {k_: {"ms_per_step": round(v_[0], 4),
                       "frac": (round(r_["frac"], 4) if (r_ := kind_roofline(k_, v_[0], v_[1])) else None),
                       "bound": r_["bound"] if r_ else None}
                  for k_, v_ in kinds.items()}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": describe(w, n_iter),
                       "l2": "inputs larger than L2: V is 8 GiB per GPU and a step touches ~2.1 GB of V rows"
                             if w.name == "paper" else "V state larger than L2" if w.N * w.d_v * 4 * w.M > 126e6
                             else "L2-resident (tiny)",
                       "parallelism": f"{world} GPU(s), independent memories per rank"},
            "roofline": roof,
            "step_roofline": {"t_roof_ms": t_roof * 1e3, "frac": step_frac, "bytes_VK": b_vk, "flops_tc": flops,
                              "unique_rows": U, "definition": "max(F_tc/P_tc, B_VK/BW_HBM) / t_step"},
            "kernels_one_step": kind_table,
            "clocks": clk, "gpu_launches": int(launches)}

    # chunk 0 of sequence 0's memories at the initial keys, for the selection check of the
    # CPU-baseline leg (the selections do not depend on V)
    chk = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cfg0 = fwpkm.make_config(w.n, w.d, w.d_v, w.k, w.C, w.H, w.qv == "bf16")
        st0 = fwpkm.State(cfg0, K1_init[:w.H].contiguous(), K2_init[:w.H].contiguous(), Vd[:w.H], w.C)
        idx0 = torch.empty(w.H, w.C, w.k, dtype=torch.int32, device=dev)
        o0 = torch.empty(w.H, w.C, w.d_v, device=dev)
        st0.forward_chunk(qd[:w.H], vd[:w.H], gd[:w.H], o0, w.C, seq_stride=qd.shape[1], idx_out=idx0)
        st0.sync()
        qb = qd[:w.H, :w.C]
        q_bits = (qb.contiguous().view(torch.int16).cpu().numpy().view(np.uint16) if qb.dtype == torch.bfloat16
                  else qb.cpu().numpy())
        chk = (q_bits, K1_init[:w.H].cpu().numpy(), K2_init[:w.H].cpu().numpy(), idx0.cpu().numpy())
        st0.destroy()

    # addressing metrics of the final pass's selections (windows of 32K tokens per memory),
    # timed apart from the step
    if full and not args.no_metrics:
        mwin = 32768
        mws = torch.empty(fwpkm.metrics_workspace_size(w.M, w.T, w.N, mwin), dtype=torch.uint8, device=dev)
        for _ in range(3):
            met, mcnt = fwpkm.addressing_metrics(idx, w.N, mwin, workspace=mws, stream=stream)
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        m0.record(stream)
        for _ in range(reps):
            fwpkm.addressing_metrics(idx, w.N, mwin, workspace=mws, stream=stream, out=(met, mcnt))
        m1.record(stream)
        torch.cuda.synchronize()
        mms = m0.elapsed_time(m1) / reps
        nwin = met.shape[0] * met.shape[1]
        mbytes = idx.numel() * 4 + nwin * w.N * 4 * 2  # selections read; counters zero-filled and read once
        mv = met.cpu().numpy().reshape(-1, 3)
        line["addressing_metrics"] = {
            "window_tokens": mwin, "windows": int(nwin), "ms": mms,
            "coverage_mean": float(mv[:, 0].mean()), "collision_mean": float(mv[:, 1].mean()),
            "kld_mean": float(mv[:, 2].mean()),
            "roofline": {"bound": "hbm", "achieved": mbytes / (mms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": mbytes / (mms / 1e3) / 1e9 / hbm_peak, "algorithmic_bytes": mbytes,
                         "definition": "selections read once + N 32-bit counters per window written and read once"}}

    # the read path's backward (dq, dv, dg from a seeded dL/do) for the first chunk of every
    # memory, timed apart from the step; its slots are the final pass's
    if full and layer is None and not args.no_metrics:
        Cb = min(w.C, w.T)
        idx_b = idx[:, :Cb].contiguous()
        gen = torch.Generator(device=dev).manual_seed(5)
        d_o = torch.randn(w.M, w.T, w.d_v, device=dev, generator=gen)
        bq = torch.empty(w.M, w.T, w.d, device=dev)
        bv = torch.empty(w.M, w.T, w.d_v, device=dev)
        bg = torch.empty(w.M, w.T, device=dev)

        def bwd():
            fwpkm.read_backward(cfg, K1d, K2d, Vd, qd, vd, gd, idx_b, d_o, bq, bv, bg, len_=Cb, seq_stride=w.T,
                                stream=stream)

        for _ in range(3):
            bwd()
        # its rows (~84 MB at the paper scale) fit in L2: a 256 MiB buffer is read before
        # each timed launch (read, not written, so that no dirty lines are written back
        # inside the timed launch), and each launch is timed alone
        scrub = torch.zeros(64 << 20, dtype=torch.float32, device=dev)
        reps = 10
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        with torch.cuda.stream(stream):
            for b0, b1 in evs:
                scrub.sum()
                b0.record(stream)
                bwd()
                b1.record(stream)
        torch.cuda.synchronize()
        bms = sum(b0.elapsed_time(b1) for b0, b1 in evs) / reps
        del scrub
        tm = w.M * Cb
        es_b = 2 if w.qv == "bf16" else 4
        bbytes = (tm * (w.k * w.d_v * 4 + w.k * 4 + (w.d + w.d_v) * es_b + 4 + w.d_v * 4 + (w.d + w.d_v + 1) * 4)
                  + w.M * 2 * w.n * (w.d // 2) * 4)
        line["read_backward"] = {
            "token_memories": tm, "ms": bms, "token_memories_per_s": tm / (bms / 1e3),
            "roofline": {"bound": "hbm", "achieved": bbytes / (bms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": bbytes / (bms / 1e3) / 1e9 / hbm_peak, "algorithmic_bytes": bbytes},
            "definition": "fwpkm_read_backward over the first chunk of every memory: the selected V rows, q, v, g, "
                          "slots and dL/do read once, dq, dv, dg written once, the keys read once per memory; "
                          "L2 flushed before each timed launch"}

    # end to end through the public API with host buffers: fwpkm_run_sequence_host (inputs
    # copied in and o copied out chunk by chunk, overlapped with the compute); the layer
    # workload copies h in and o' out around fwpkm_run_layer
    if full and not args.no_e2e:
        dev_in = [hd] if layer is not None else [qd, vd, gd]
        dev_out = o_out if layer is not None else o
        host_in = [torch.empty_like(x, device="cpu").pin_memory() for x in dev_in]
        host_out = torch.empty_like(dev_out, device="cpu").pin_memory()
        for hx, dx in zip(host_in, dev_in):
            hx.copy_(dx)
        torch.cuda.synchronize()
        if layer is None:
            io_scratch = torch.empty(fwpkm.run_sequence_host_scratch_size(cfg, w.T), dtype=torch.uint8, device=dev)

            def e2e_step():
                st.run_sequence_host(*host_in, host_out, n_iter=n_iter, scratch=io_scratch)
        else:
            def e2e_step():
                for hx, dx in zip(host_in, dev_in):
                    dx.copy_(hx, non_blocking=True)
                step()
                host_out.copy_(dev_out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
        bi = sum(x.numel() * x.element_size() for x in host_in)
        line["e2e"] = {"value": job_throughput(tokens_per_step, world, ems), "unit": "tokens/s",
                       "h2d_bytes_per_step": bi, "d2h_bytes_per_step": host_out.numel() * host_out.element_size(),
                       "ms_per_step": ems,
                       "call": ("fwpkm_run_sequence_host (per-chunk copies overlapped with the compute)"
                                if layer is None else "copies of h in and o' out around fwpkm_run_layer")}

    if needles is not None:
        # read-back: from the initial state, n_iter passes; vhat at each needle's query
        # position recovered from o = g vhat + (1 - g) v, against the normalised needle value
        from sparse_weight_memory_chunk_b200.inputs import bf16_to_f32
        K1d.copy_(K1_init); K2d.copy_(K2_init); Vd.copy_(state0[0])
        step()
        st.sync()
        pos, qpos, _, vs = needles
        of = o[0].cpu().numpy().astype(np.float64)
        vf = (bf16_to_f32(v[0]) if w.qv == "bf16" else v[0]).astype(np.float64)
        gf = g[0].astype(np.float64)
        vsf = (bf16_to_f32(vs) if w.qv == "bf16" else vs).astype(np.float64)
        cos = []
        for i, r in enumerate(qpos):
            vhat = (of[r] - (1.0 - gf[r]) * vf[r]) / gf[r]
            z = (vsf[i] - vsf[i].mean()) / np.sqrt(vsf[i].var() + 1e-5)
            cos.append(float(vhat @ z / (np.linalg.norm(vhat) * np.linalg.norm(z) + 1e-30)))
        line["needle_readback"] = {"n_iter": n_iter, "mean_cos": float(np.mean(cos)),
                                   "min_cos": float(np.min(cos)), "needles": len(cos),
                                   "definition": "cos(vhat_r, z(v*)) at each needle's query position r, final pass, "
                                                 "run from the initial state"}

    if full and not args.no_stream and layer is None:
        # token-at-a-time inference: the first 2C + 1 tokens of every memory fed 1 (then 16)
        # per call through fwpkm_stream_tokens (two chunk writes, each when its lookahead
        # arrives), then a flush; timed with events on the launching stream
        S = min(w.T, 2 * w.C + 1)
        for t_ in range(0, 8, 4):  # warm-up of the streaming launches
            st.stream_tokens(qd[:, t_:], vd[:, t_:], gd[:, t_:], o[:, t_:], n_tok=4, seq_stride=w.T, stream=stream)
        st.stream_flush(stream=stream)
        torch.cuda.synchronize()
        per = {}
        for per_call in (1, 16):
            l0s = fwpkm.launch_count()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            t_ = 0
            while t_ < S:
                n_ = min(per_call, S - t_)
                st.stream_tokens(qd[:, t_:], vd[:, t_:], gd[:, t_:], o[:, t_:], n_tok=n_, seq_stride=w.T,
                                 stream=stream)
                t_ += n_
            st.stream_flush(stream=stream)
            s1.record(stream)
            torch.cuda.synchronize()
            sms = s0.elapsed_time(s1)
            per[str(per_call)] = {"us_per_token": sms * 1e3 / S, "tokens_per_s": w.B * S / (sms / 1e3),
                                  "launches_per_token": (fwpkm.launch_count() - l0s) / S}
        st.sync()
        line["token_stream"] = {
            "tokens": S, "per_call": per,
            "hbm_bytes_per_token_max": w.M * 3 * w.k * w.d_v * 4,
            "definition": "tokens of the first 2C+1 positions of every sequence fed n per fwpkm_stream_tokens call, "
                          "then fwpkm_stream_flush; tokens/s counts sequence tokens (B per position); "
                          "hbm_bytes_per_token_max: gathered rows + the same rows read and written by the chunk "
                          "write (unique rows), all memories; latency-bound: a token's read is a chain of four "
                          "dependent launches (staging with the query norms, scoring, selection, gather)"}

    st.destroy()
    if layer is not None:
        layer.destroy()
    del Vd, K1d, K2d, o
    torch.cuda.empty_cache()

    # CPU-baseline leg (rank 0, one GPU): the oracle's selection check of chunk 0, and
    # (full) the oracle timed on a bounded sample of the same workload
    if chk is not None:
        line["selection_check"] = selection_check(w, *chk)
        # the headline workload's sample is ~10-30 s of CPU work; the other workloads' are
        # kept to a few seconds each (fewer chunks)
        n_chunks = (8 if w.name in ("paper", "needle") else 16) if full else (2 if w.name == "needle" else 4)
        info = oracle_sample(w, n_chunks, seqs=None if w.name in ("paper", "mid", "tiny") else 1)
        line["cpu_baseline"] = {"value": info["tokens"] / info["seconds"], "unit": "tokens/s",
                                "cores": info["threads"], "kind": "oracle", "sample": info["sample"],
                                "host_threads": info["host_threads"], "cpu_model": info["cpu_model"]}
        if w.name == "tiny":  # and one thread, for the single-memory workload
            one = oracle_sample(w, n_chunks, threads=1)
            line["cpu_baseline"]["one_thread"] = {"value": one["tokens"] / one["seconds"], "threads": one["threads"]}
    return line


def run_ours(args, w, rank, world, local_rank):
    import torch

    from sparse_weight_memory_chunk_b200 import build
    build.build()
    torch.cuda.set_device(local_rank)
    line = measure(args, w, rank, world, local_rank, args.n_iter, args.steps, args.warmup, full=True)
    if args.workload is None and not args.no_configs:
        # the other workloads, each under `configs`: fewer timed steps, the same rules
        configs = {}
        for name, n_iter in (("tiny", 1), ("mid", 1), ("needle", 1), ("needle", 2), ("needle", 4), ("layer", 1)):
            key = name if name != "needle" else f"needle_n{n_iter}"
            _, wc = BY_NAME[name]
            try:
                sub = measure(args, wc, rank, world, local_rank, n_iter, max(1, args.config_steps),
                              max(3, args.warmup), full=False)
                keep = ("ms_per_step", "value", "unit", "steps", "warmup", "config", "roofline", "step_roofline",
                        "kernels_one_step", "clocks", "gpu_launches", "selection_check", "needle_readback",
                        "cpu_baseline")
                configs[key] = {k_: sub[k_] for k_ in keep if k_ in sub}
            except Exception as e:  # one workload failing must not hide the others
                configs[key] = {"error": f"{type(e).__name__}: {e}"}
        line["configs"] = configs
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    _, w = BY_NAME[args.workload or "paper"]
    if args.batch or args.tokens:
        from dataclasses import replace
        w = replace(w, B=args.batch or w.B, T=args.tokens or w.T)
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
