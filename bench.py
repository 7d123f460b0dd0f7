"""Benchmark of the chunked TTT / linear-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llm_d64|momentum_d128|long_d128] [--chunk C] [--segments P]

A step is one chunked forward of the whole layer (all heads, all tokens, final
state) over one batch of synthetic inputs already resident in HBM.  Default
workload: the long-context layer the tensor-peak fraction is quoted on (B=1,
H=8, T=65536, d=128, bf16, constant learning rate, chunk 128).  The same line
carries the chunk sweep (64, 128), the LLM-shaped and momentum layers, the
decode step, the feature-mapped layer and the backward as sub-objects.
Prints ONE JSON line on rank 0.

Multi-GPU (torchrun): every rank runs its own batch (independent sequences,
no collective on the data path: weak scaling); value = tokens of all ranks /
max-over-ranks device time.  `--impl reference` times the float64 CPU oracle
on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import CONFIGS, make_case  # noqa: E402

METRIC = "TTT-layer tokens/sec (chunked fwd, 1 B200) and % tensor peak; decode HBM GB/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def algorithmic_bytes(c, B, H, T):
    """Minimum HBM bytes of one forward: read q, k, v (and eta), write o and
    the final state once."""
    el = 2 if c.dtype == "bf16" else 4
    qkvo = B * H * T * (2 * c.d_k + 2 * c.d_v) * el
    eta = B * H * T * 4 if c.eta_mode == "token" else 0
    state = B * H * c.d_v * c.d_k * 4 * (2 if c.beta else 1)
    return qkvo + eta + state


def executed_flops(c, B, H, T, chunk):
    """Tensor-core flops the chunked kernel executes (full C x C score tiles):
    per token-head 2*C*d (Q K^T) + 2*C*d (P V) + 2*d*d (Q W^T) + 2*d*d (V^T K)."""
    d = c.d_k
    per = 4 * chunk * d + 4 * d * d
    return B * H * T * per


CHUNKED_SOURCES = ("chunked_tc.cuh", "chunked_tc_mom.cuh", "common.cuh", "ttt_la.cu")


def src_hash():
    """Hash of the chunked kernels' sources and their launch planner (the files
    they are compiled and planned from; the other kernels' headers and the
    host-buffer pipeline do not change what a chunked launch reads or writes)."""
    h = hashlib.sha1()
    cdir = os.path.join(ROOT, "test_layers_causal_b200", "csrc")
    for f in CHUNKED_SOURCES:
        with open(os.path.join(cdir, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def read_traffic(workload, chunk):
    """DRAM bytes per forward from a committed ncu summary, if it was taken on
    the current kernel sources (profiles/<workload>_c<chunk>.traffic.txt holds
    lines `src_hash=...` and `dram_bytes_per_call=...`)."""
    p = os.path.join(ROOT, "profiles", f"{workload}_c{chunk}.traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if "=" in line:
                a, b = line.strip().split("=", 1)
                kv[a.strip()] = b.strip()
    if kv.get("src_hash") != src_hash():
        return None
    try:
        return float(kv["dram_bytes_per_call"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.tmp = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [l.strip().split(", ") for l in self.tmp.read().splitlines() if l.strip()]
        os.unlink(self.tmp.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            if len(r) >= 9:
                for n, val in zip(names, r[5:9]):
                    if val.strip().lower() == "active":
                        reasons.add(n)
        busy = [s for s in sm if mx and s > 0.3 * max(mx)]
        return {"sm_mhz": statistics.median(busy or sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons), "samples": len(rows)}


def dist_init():
    from test_layers_causal_b200 import ranks
    info = ranks.init()
    return info.world, info.rank, info.local, info


def barrier(info):
    from test_layers_causal_b200 import ranks
    ranks.barrier(info)


def max_over_ranks(x, info):
    from test_layers_causal_b200 import ranks
    return ranks.max_over_ranks(x, info)


# --------------------------------------------------------------- oracle ----
# Tokens of every (b, h) sequence in one bounded oracle sample: the reference
# arm's steps (about 1 s of float64 work each) and the cpu_baseline leg (about
# 5-10 s).  The oracle's cost per token is constant, so its tokens/s over a
# prefix of every sequence is its tokens/s over the whole layer.
REF_TOKENS = {"long_d128": 2048, "llm_d64": 1024, "momentum_d128": 256, "tiny_f32": 256}
CPU_TOKENS = {"long_d128": 16384, "llm_d64": 4096, "momentum_d128": 2048, "tiny_f32": 256}


def oracle_sample(c, tokens, x=None):
    """Runs the float64 oracle on the first `tokens` tokens of every (b, h)
    sequence of the workload's inputs `x` (make_case(c) when None); returns
    (wall seconds, process CPU seconds, o [B*H, tokens, d_v])."""
    import oracle
    x = make_case(c) if x is None else x
    tokens = min(tokens, c.T)
    f = lambda t: t[:, :, :tokens].float().double().reshape(-1, tokens, *t.shape[3:]).numpy()  # noqa: E731
    eta = f(x["eta"]) if x["eta"] is not None else x["eta_const"]
    q, k, v = f(x["q"]), f(x["k"]), f(x["v"])
    t0, c0 = time.perf_counter(), time.process_time()
    o, _, _ = oracle.ttt_recurrence_f64(q, k, v, eta, beta=c.beta)
    return time.perf_counter() - t0, time.process_time() - c0, o


def parity(o_gpu, o_ref, tol=2e-2):
    """Worst relative Frobenius error over the (b, h) sequences of the GPU
    output's first o_ref.shape[1] tokens against the oracle's."""
    import numpy as np
    n = o_ref.shape[1]
    g = o_gpu[:, :, :n].float().double().reshape(-1, n, o_gpu.shape[-1]).numpy()
    err = np.linalg.norm(g - o_ref, axis=(1, 2)) / np.maximum(np.linalg.norm(o_ref, axis=(1, 2)), 1e-30)
    worst = float(err.max())
    return {"sequences": int(o_ref.shape[0]), "tokens_each": int(n), "rel_frobenius_max": worst, "tolerance": tol,
            "pass": worst <= tol}


def cpu_line(c, tokens, wall, cpu, what):
    """cpu_baseline object: tokens/s of the layer (B sequences x `tokens`
    tokens, all heads) over the oracle's wall time; `cores` is the number of
    threads the oracle kept busy (process CPU time / wall time)."""
    n = min(tokens, c.T)
    return {"value": c.B * n / wall, "unit": "tokens/s", "cores": max(1, round(cpu / wall)),
            "host_cpu_count": os.cpu_count(), "kind": "oracle",
            "sample": f"{what}: the first {n} of {c.T} tokens of all {c.B * c.H} (b,h) sequences of the benchmark's "
                      f"own inputs ({wall:.1f} s of float64 numpy, {c.B * n} layer tokens; the oracle's per-token "
                      "cost does not depend on the position, so this is its rate on the whole layer)"}


def cpu_baseline(c, tokens, x=None):
    """The oracle timed on a bounded sample of the workload's inputs; also
    returns its outputs, for the parity check of the GPU result."""
    wall, cpu, o_ref = oracle_sample(c, tokens, x)
    return cpu_line(c, tokens, wall, cpu, "one run"), o_ref


def run_reference(args, c, ws, rank, info):
    if rank != 0:
        return
    tokens = min(c.T, args.ref_tokens or REF_TOKENS.get(c.name, 1024))
    x = make_case(c)
    for _ in range(args.warmup):
        oracle_sample(c, tokens, x)
    walls, cpus = [], []
    for _ in range(args.steps):
        wall, cpu, _ = oracle_sample(c, tokens, x)
        walls.append(wall)
        cpus.append(cpu)
    t = sum(walls) / len(walls)
    line_cpu = cpu_line(c, tokens, t, sum(cpus) / len(cpus), f"each of {args.steps} steps")
    val = line_cpu["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(c, args), step_tokens=c.B * tokens),
        "cpu_baseline": line_cpu,
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def graph_time_us(fns, reps_min=20, min_ms=300.0, sampler=None):
    """Device time per call of `fns` (a list of callables, one per rotating
    input set): one CUDA graph holds a call on every set; it is replayed for
    about a second untimed, then at least `reps_min` times and `min_ms`
    milliseconds between CUDA events on the launching stream."""
    for f in fns:
        f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fns:
            f()
    stream = torch.cuda.current_stream()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    per_replay_ms = max(e0.elapsed_time(e1), 1e-3)
    t_end = time.time() + 1.0
    while time.time() < t_end:
        for _ in range(max(1, int(50.0 / per_replay_ms))):
            g.replay()
        torch.cuda.synchronize()
    reps = max(reps_min, int(min_ms / per_replay_ms))
    if sampler is not None:
        sampler.mark_start()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.mark_end()
    del g
    return e0.elapsed_time(e1) * 1e3 / (reps * len(fns))


def forward_measure(ttt, dev, c, chunk, peaks, sets=4, segments=0):
    """One workload's chunked forward: device time per call over `sets`
    rotating input sets (together larger than L2), algorithmic bytes, the HBM
    and executed-tensor-flop fractions of the measured peaks, the launch plan
    and the clocks seen meanwhile."""
    x = make_case(c)
    bufs = []
    for _ in range(sets):
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        eta = x["eta"].to(dev) if x["eta"] is not None else None
        o = torch.empty_like(v)
        S = torch.empty(c.B, c.H, c.d_v, c.d_k, device=dev, dtype=torch.float32)
        M = torch.empty_like(S) if c.beta else None
        bufs.append((q, k, v, eta, o, S, M))
    wsb = ttt.workspace_bytes(bufs[0][0], bufs[0][2], chunk=chunk, beta=c.beta, segments=segments)
    work = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)

    def call(i):
        q, k, v, eta, o, S, M = bufs[i]
        return lambda: ttt.forward_chunked(q, k, v, eta, eta_const=x["eta_const"], beta=c.beta, chunk=chunk,
                                           segments=segments, out=o, state_out=S, mom_out=M, workspace=work)
    sampler = ClockSampler(dev.index or 0)
    sampler.start()
    us = graph_time_us([call(i) for i in range(sets)], sampler=sampler)
    clocks = sampler.stop()
    if ttt.device_status() != 0:
        raise SystemExit(f"device status reports a timed-out wait ({c.name}, chunk {chunk})")
    nbytes = algorithmic_bytes(c, c.B, c.H, c.T)
    gbs = nbytes / (us * 1e-6) / 1e9
    flops = executed_flops(c, c.B, c.H, c.T, chunk)
    tf = flops / (us * 1e-6) / 1e12
    plan = ttt.chunked_plan(c.B, c.H, c.T, c.d_k, c.d_v, chunk=chunk, beta=c.beta, segments=segments,
                            eta=c.eta_mode == "token")
    del bufs, work
    torch.cuda.empty_cache()
    return {"workload": c.name, "chunk": chunk, "us_per_call": us, "tokens_per_s": c.B * c.T / (us * 1e-6),
            "algorithmic_bytes": nbytes, "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
            "executed_tflops": tf, "tensor_frac": tf / peaks["bf16_tflops"],
            "traffic": read_traffic(c.name, chunk), "plan": plan, "clocks": clocks,
            "gpu_launches_per_call": launches_per_forward(plan)}


def launches_per_forward(plan):
    """Kernels one ttt_la_forward_chunked call launches: the chunked kernel,
    preceded by the flag-zeroing kernel when the plan has several segments."""
    return 2 if plan["segments"] > 1 else 1


def decode_measure(ttt, dev, peaks):
    """The batched decode workload: 256 sequences x 16 heads, d = 128, state
    carried from a 2048-token chunked prefill, then 512 timed single-token
    steps.  Every step streams the 256 MiB fp32 state in and out of HBM."""
    from synth import make_decode_inputs
    x = make_decode_inputs(dev)
    pq, pk, pv = x["prefill"]
    sq, sk, sv = x["steps"]
    ec = x["eta_const"]
    _, S, _ = ttt.forward_chunked(pq, pk, pv, None, eta_const=ec, chunk=128)
    del pq, pk, pv
    n = sq.shape[0]
    out = torch.empty_like(sq[0])
    Sw = S.clone()
    for t in range(3):
        ttt.decode_step(sq[t], sk[t], sv[t], Sw, eta_const=ec, out=out)
    del Sw
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for t in range(n):
        ttt.decode_step(sq[t], sk[t], sv[t], S, eta_const=ec, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / n
    nbytes = 2 * S.numel() * 4 + 3 * sq[0].numel() * sq.element_size() + out.numel() * out.element_size()
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"workload": "decode N256 H16 d128 (2048-token prefill, 512 steps)", "us_per_step": us,
            "bytes_per_step": nbytes, "hbm_gbs": gbs, "peak": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
            "tokens_per_s": sq.shape[1] / (us * 1e-6), "gpu_launches": n}


def phi_measure(ttt, dev, peaks, reps=100):
    """The layer whose fast weight is the last layer of a frozen gated MLP,
    on the llm_d64 shape (B4 H16 T4096, per-token eta): phi(q), phi(k) =
    silu(W1 x) * (W3 x) with d_in = d_out = 64 (one feature-map launch for
    both), then the chunked forward on (phi(q), phi(k), v).  Four rotating
    input sets (512 MB) keep consecutive steps out of L2; one CUDA graph holds
    a step on each set."""
    from synth import make_feature_weights
    c = CONFIGS["llm_d64"]
    x = make_case(c)
    W1, W3 = (w.to(dev) for w in make_feature_weights(c.H, c.d_k, c.d_k, 7))
    B, H, T, d = c.B, c.H, c.T, c.d_k
    sets = []
    for _ in range(4):
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        eta = x["eta"].to(dev)
        fq, fk = torch.empty_like(q), torch.empty_like(k)
        o = torch.empty_like(v)
        S = torch.empty(B, H, d, d, device=dev, dtype=torch.float32)
        sets.append((q, k, v, eta, fq, fk, o, S))
    work = torch.empty(max(ttt.workspace_bytes(sets[0][0], sets[0][2], chunk=c.chunk), 16), dtype=torch.uint8,
                       device=dev)

    def phi_only(i):
        q, k, _, _, fq, fk, _, _ = sets[i]
        ttt.feature_map([q, k], W1, W3, out=[fq, fk])

    def layer(i):
        q, k, v, eta, fq, fk, o, S = sets[i]
        ttt.feature_map([q, k], W1, W3, out=[fq, fk])
        ttt.forward_chunked(fq, fk, v, eta, eta_const=x["eta_const"], chunk=c.chunk, out=o, state_out=S,
                            workspace=work)

    def timed(fn):
        for i in range(4):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(4):
                fn(i)
        for _ in range(3):
            g.replay()
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / (4 * reps)

    phi_us = timed(phi_only)
    layer_us = timed(layer)
    if ttt.device_status() != 0:
        raise SystemExit("device status reports a timed-out wait")
    n_tok = B * H * T
    phi_bytes = 2 * n_tok * d * 2 + 2 * n_tok * d * 2 + 2 * H * d * d * 2
    gbs = phi_bytes / (phi_us * 1e-6) / 1e9
    return {"workload": "llm_d64 with the frozen gated-MLP feature map (d_in 64 -> d_out 64)",
            "phi_us": phi_us, "phi_bytes": phi_bytes, "phi_hbm_gbs": gbs, "phi_frac": gbs / peaks["hbm_gbs"],
            "layer_us_per_step": layer_us, "tokens_per_s": B * T / (layer_us * 1e-6),
            "gpu_launches_per_step": 1 + launches_per_forward(ttt.chunked_plan(B, H, T, d, d, chunk=c.chunk, beta=0.0,
                                                                                eta=True))}


def backward_measure(ttt, dev, peaks, name="llm_d64", reps=5):
    """The layer's backward on a workload's inputs with a seeded upstream
    gradient dL/do, dL/dW_T (and dL/dM_T with momentum): dq, dk, dv, per-token
    deta, dW0 (and dM0), in both forms -- the recurrent kernel (one block per
    head) and the chunk-parallel one.  Without momentum that is a transpose of
    dL/dW_T and three chunked forward runs, the two reverse-time ones writing
    dv, deta and dk themselves (four launches); with momentum, one transpose
    launch, the momentum forward for dq, the reverse chunkwise kernel twice
    and the deta kernel (five).  Workspaces are allocated once; CUDA events
    over `reps` calls (the chunked form 20x as many) after one warm-up call of
    each."""
    c = CONFIGS[name]
    x = make_case(c)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    eta = x["eta"].to(dev)
    g = torch.Generator(device=dev).manual_seed(11)
    dO = torch.randn(v.shape, generator=g, device=dev).to(v.dtype)
    dW = torch.randn(c.B, c.H, c.d_v, c.d_k, generator=g, device=dev)
    dM = torch.randn(c.B, c.H, c.d_v, c.d_k, generator=g, device=dev) if c.beta else None
    stream = torch.cuda.current_stream()
    # bytes a backward must move: q, k, v, dO read, dq, dk, dv written (bf16),
    # eta read and deta written (fp32), dL/dW_T read and dL/dW_0 written (and
    # the same pair for M with momentum)
    nstates = 4 if c.beta else 2
    nbytes = c.B * c.H * (c.T * (2 * (2 * c.d_k + 2 * c.d_v) + 2 * (2 * c.d_k + c.d_v) + 8)
                          + nstates * 4 * c.d_v * c.d_k)
    what = "dq, dk, dv, deta, dW0, dM0 from dL/do, dL/dW_T and dL/dM_T" if c.beta else \
        "dq, dk, dv, deta, dW0 from dL/do and dL/dW_T"
    out = {"workload": f"{name} backward ({what})", "algorithmic_bytes": nbytes}
    # generous preallocated scratch (the recurrent form keeps checkpoints of W and M)
    ws = {"recurrent": torch.empty(3 << 30, dtype=torch.uint8, device=dev),
          "chunked": torch.empty(256 << 20, dtype=torch.uint8, device=dev)}
    kw = dict(eta_const=x["eta_const"], grad_state=dW)
    if c.beta:
        kw.update(beta=c.beta, grad_mom=dM)
    for form, fn, n in (("recurrent", ttt.backward_recurrent, reps), ("chunked", ttt.backward_chunked, 20 * reps)):
        def call():
            return fn(q, k, v, dO, eta, workspace=ws[form], **kw)
        r = call()
        del r
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            r = call()
        e1.record(stream)
        torch.cuda.synchronize()
        del r
        if ttt.device_status() != 0:
            raise SystemExit("device status reports a timed-out wait")
        us = e0.elapsed_time(e1) * 1e3 / n
        gbs = nbytes / (us * 1e-6) / 1e9
        out[form] = {"us_per_call": us, "tokens_per_s": c.B * c.T / (us * 1e-6), "hbm_gbs": gbs,
                     "hbm_frac": gbs / peaks["hbm_gbs"],
                     # chunked: the state transposes, then (flag zeroing + forward) for dq and, without
                     # momentum, for each of the two reverse passes; with momentum also the two reverse
                     # launches, the dL/dW_0 reduction and its sum, and the deta launch
                     "gpu_launches_per_call": 1 if form == "recurrent" else (8 if c.beta else 7)}
    out["chunked_speedup_over_recurrent"] = out["recurrent"]["us_per_call"] / out["chunked"]["us_per_call"]
    del ws
    torch.cuda.empty_cache()
    return out


def workload_config(c, args):
    return {"workload": c.name, "B": c.B, "H": c.H, "T": c.T, "d_k": c.d_k, "d_v": c.d_v,
            "chunk": args.chunk or c.chunk, "eta": "per-token" if c.eta_mode == "token" else "constant",
            "beta": c.beta, "global_batch": c.B, "seq_len": c.T, "parallelism": f"dp{args.gpus}",
            "l2": f"{args.sets} rotating input sets (inputs larger than L2)"}


# ----------------------------------------------------------------- ours ----
def run_ours(args, c, ws, rank, local, info):
    import test_layers_causal_b200 as ttt
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, src = load_peaks()
    chunk = args.chunk or c.chunk
    x = make_case(c)
    qh, kh, vh = x["q"], x["k"], x["v"]
    etah = x["eta"]
    # rotating device copies so that consecutive steps do not hit in L2
    sets = []
    for _ in range(args.sets):
        q, k, v = qh.to(dev), kh.to(dev), vh.to(dev)
        eta = etah.to(dev) if etah is not None else None
        o = torch.empty_like(v)
        S = torch.empty(c.B, c.H, c.d_v, c.d_k, device=dev, dtype=torch.float32)
        M = torch.empty_like(S) if c.beta else None
        sets.append((q, k, v, eta, o, S, M))
    wsb = ttt.workspace_bytes(sets[0][0], sets[0][2], chunk=chunk, beta=c.beta, segments=args.segments)
    work = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        q, k, v, eta, o, S, M = sets[i % len(sets)]
        ttt.forward_chunked(q, k, v, eta, eta_const=x["eta_const"], beta=c.beta, chunk=chunk,
                            segments=args.segments, out=o, state_out=S, mom_out=M, workspace=work)

    # CUDA graph per input set: one replay = one step, no host launch overhead
    for i in range(len(sets)):
        step(i)
    torch.cuda.synchronize()
    graphs = []
    for i in range(len(sets)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(i)
        graphs.append(g)
    # one graph that runs a step on every input set in turn: fewer graph
    # launches per step (the work per step is unchanged)
    big = torch.cuda.CUDAGraph()
    with torch.cuda.graph(big):
        for i in range(len(sets)):
            step(i)
    torch.cuda.synchronize()

    def run_steps(n):
        for _ in range(n // len(sets)):
            big.replay()
        for i in range(n % len(sets)):
            graphs[i].replay()
    status = ttt.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    sampler = ClockSampler(local)
    sampler.start()
    for i in range(args.warmup):
        graphs[i % len(graphs)].replay()
    # keep the GPU busy ~1 s right before the timed region so the clock
    # samples describe the loaded state
    t_end = time.time() + 1.0
    i = 0
    while time.time() < t_end:
        graphs[i % len(graphs)].replay()
        i += 1
        if i % 200 == 0:
            torch.cuda.synchronize()
    barrier(info)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark_start()
    ev0.record(stream)
    run_steps(args.steps)
    ev1.record(stream)
    torch.cuda.synchronize()
    sampler.mark_end()
    barrier(info)
    clocks = sampler.stop()
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, info)
    ms_per_step = ms_max / args.steps
    tokens_per_step = c.B * c.T
    from test_layers_causal_b200 import ranks
    value = ranks.weak_scaling_tokens_per_s(tokens_per_step, ws, ms_per_step)
    if ttt.device_status() != 0:
        raise RuntimeError("device status reports a timed-out wait")
    del graphs, big
    plan = ttt.chunked_plan(c.B, c.H, c.T, c.d_k, c.d_v, chunk=chunk, beta=c.beta, segments=args.segments,
                            eta=c.eta_mode == "token")

    # ---- end to end: pinned host buffers in, o (and final state) back out
    qp, kp, vp = (t.pin_memory() for t in (qh, kh, vh))
    ep = etah.pin_memory() if etah is not None else None
    oh = torch.empty(vh.shape, dtype=vh.dtype, pin_memory=True)
    Sh = torch.empty(c.B, c.H, c.d_v, c.d_k, dtype=torch.float32, pin_memory=True)
    bufs = ttt.host.HostStaging()
    kw = dict(eta_const=x["eta_const"], beta=c.beta, chunk=chunk, segments=args.segments)
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        ttt.forward_chunked_host(qp, kp, vp, ep, o_host=oh, bufs=bufs, state_host=Sh, **kw)
    torch.cuda.synchronize()
    barrier(info)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        _, h2d, d2h = ttt.forward_chunked_host(qp, kp, vp, ep, o_host=oh, bufs=bufs, state_host=Sh, **kw)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), info) / e2e_steps
    e2e_val = tokens_per_step * ws / (e2e_ms * 1e-3)
    del bufs

    # ---- roofline of the forward call (one kernel launch after a flag memset)
    nbytes = algorithmic_bytes(c, c.B, c.H, c.T)
    achieved = nbytes / (ms_per_step * 1e-3) / 1e9
    flops = executed_flops(c, c.B, c.H, c.T, chunk)
    tflops = flops / (ms_per_step * 1e-3) / 1e12
    traffic = read_traffic(c.name, chunk)
    kname = ("chunked_tc_mom_kernel" if c.beta else f"chunked_tc_kernel<{chunk},{c.d_k}>")
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if c.dtype == "bf16" else "f32", "data": "synthetic",
        "config": workload_config(c, args),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "kernel": kname,
                     "algorithmic_bytes": nbytes, "peak_source": f"{src} copy bandwidth (of {src})",
                     "timed_unit": "one forward call per step: the flag-zeroing kernel (segmented plans) and "
                                   "the chunked kernel"},
        "tensor": {"achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                   "frac": tflops / peaks["bf16_tflops"], "executed_flops": flops,
                   "peak_source": f"{src} cuBLAS bf16 burst (of {src})"},
        "plan": plan,
        "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * launches_per_forward(plan),
        "clocks": clocks,
    }
    del sets, work
    torch.cuda.empty_cache()
    if ws == 1 and not args.no_extra:
        # chunk sweep of the headline workload, then the other layer workloads
        sweep = {}
        for C in (64, 128):
            if C != chunk and c.beta == 0:
                sweep[str(C)] = forward_measure(ttt, dev, c, C, peaks)
        if sweep:
            line["chunk_sweep"] = sweep
        others = {}
        for name in ("llm_d64", "momentum_d128", "long_d128"):
            if name != c.name:
                oc = CONFIGS[name]
                others[name] = forward_measure(ttt, dev, oc, oc.chunk, peaks)
        line["workloads"] = others
        line["decode"] = decode_measure(ttt, dev, peaks)
        torch.cuda.empty_cache()
        line["phi_layer"] = phi_measure(ttt, dev, peaks)
        torch.cuda.empty_cache()
        line["backward"] = backward_measure(ttt, dev, peaks)
        line["backward_momentum"] = backward_measure(ttt, dev, peaks, "momentum_d128", reps=2)
    if rank == 0 and not args.no_cpu_baseline:
        tokens = args.cpu_tokens or CPU_TOKENS.get(c.name, c.T)
        line["cpu_baseline"], o_ref = cpu_baseline(c, tokens, x)
        # the end-to-end run's output (public host-buffer API) against the oracle on the same inputs
        line["parity"] = parity(oh, o_ref)
    if rank == 0:
        print(json.dumps(line), flush=True)


def profile_run(args):
    """Plain launches (no graphs, no timing) for ncu: --warmup + --steps calls
    of the workload's forward, of the decode step on a random 256 MiB state,
    (phi) of the feature map plus chunked forward on the llm_d64 shape, or of
    the chunk-parallel backward on the llm_d64 (backward) or momentum_d128
    (backward_momentum) inputs."""
    import test_layers_causal_b200 as ttt
    dev = torch.device("cuda", 0)
    if args.workload == "decode":
        from synth import DECODE
        N, H, d = DECODE["N"], DECODE["H"], DECODE["d"]
        g = torch.Generator(device=dev).manual_seed(DECODE["seed"])
        S = 0.1 * torch.randn(N, H, d, d, generator=g, device=dev)
        q, k, v = (torch.randn(N, H, d, generator=g, device=dev).to(torch.bfloat16) for _ in range(3))
        for _ in range(args.warmup + args.steps):
            ttt.decode_step(q, k, v, S, eta_const=1.0 / math.sqrt(d))
    elif args.workload == "phi":
        from synth import make_feature_weights
        c = CONFIGS["llm_d64"]
        x = make_case(c)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        W1, W3 = (w.to(dev) for w in make_feature_weights(c.H, c.d_k, c.d_k, 7))
        for _ in range(args.warmup + args.steps):
            ttt.forward_chunked_phi(q, k, v, W1, W3, x["eta"].to(dev), eta_const=x["eta_const"], chunk=c.chunk)
    elif args.workload in ("backward", "backward_momentum"):
        c = CONFIGS["llm_d64" if args.workload == "backward" else "momentum_d128"]
        x = make_case(c)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        g = torch.Generator(device=dev).manual_seed(11)
        dO = torch.randn(v.shape, generator=g, device=dev).to(v.dtype)
        kw = dict(eta_const=x["eta_const"], grad_state=torch.randn(c.B, c.H, c.d_v, c.d_k, generator=g, device=dev),
                  workspace=torch.empty(256 << 20, dtype=torch.uint8, device=dev))
        if c.beta:
            kw.update(beta=c.beta, grad_mom=torch.randn(c.B, c.H, c.d_v, c.d_k, generator=g, device=dev))
        for _ in range(args.warmup + args.steps):
            ttt.backward_chunked(q, k, v, dO, x["eta"].to(dev), **kw)
    else:
        c = CONFIGS[args.workload]
        x = make_case(c)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        eta = x["eta"].to(dev) if x["eta"] is not None else None
        for _ in range(args.warmup + args.steps):
            ttt.forward_chunked(q, k, v, eta, eta_const=x["eta_const"], beta=c.beta, chunk=args.chunk or c.chunk,
                                segments=args.segments)
    torch.cuda.synchronize()
    if ttt.device_status() != 0:
        raise SystemExit("device status reports a timed-out wait")
    print(f"profile run ok: {args.workload}, {args.warmup + args.steps} calls")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long_d128",
                    choices=sorted(CONFIGS) + ["decode", "phi", "backward", "backward_momentum"])
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--segments", type=int, default=0)
    ap.add_argument("--sets", type=int, default=4)
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="tokens of every sequence per reference-arm step (0: the workload's default sample)")
    ap.add_argument("--cpu-tokens", type=int, default=0,
                    help="tokens of every sequence in the cpu_baseline sample (0: the workload's default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="headline only: no chunk sweep, other workloads, decode, feature map or backward")
    ap.add_argument("--profile-run", action="store_true",
                    help="plain launches for a profiler: no graphs, timing, decode or CPU baseline")
    args = ap.parse_args()
    if args.profile_run:
        profile_run(args)
        return
    if args.workload in ("decode", "phi", "backward", "backward_momentum"):
        raise SystemExit(f"{args.workload} is measured inside every chunked run (its own object in the line)")
    c = CONFIGS[args.workload]
    if c.dtype != "bf16":
        raise SystemExit("bench workloads are the bf16 layers")
    ws, rank, local, info = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, c, ws, rank, info)
        else:
            run_ours(args, c, ws, rank, local, info)
    finally:
        from test_layers_causal_b200 import ranks
        ranks.finalize(info)


if __name__ == "__main__":
    main()
