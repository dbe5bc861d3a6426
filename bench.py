#!/usr/bin/env python
"""GPT-2 124M training throughput on B200: tokens/s (fwd + bwd + clip + AdamW,
T=1024, bf16 compute with fp32 master weights) and MFU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

One step = zero_grad, forward + mean cross-entropy, backward, global-norm clip
and AdamW over all 124.5M parameters, on B=16 sequences of T=1024 tokens cut
from a device-resident synthetic token stream (consecutive windows; rank r
starts at B*T*r and advances B*T*N).  Weights are random (N(0, 0.02)); the
stream is Zipf(1.1) ids with an end-of-text id before every document of
geometric length (mean 600): a stand-in for a tokenised web corpus.

With N > 1 (torchrun) every rank trains its own shard and the library
averages the gradient arena bucket by bucket (one NCCL all-reduce per layer's
weight matrices, issued on its communication stream as the backward finishes
that layer, then one for the embeddings and vectors; recorded into the step's
CUDA graph) before clip + AdamW (data parallel; per-GPU work is fixed, so
scaling is weak).

`--impl reference` times the CPU oracle (test infrastructure) on the same
workload, each step a bounded sample of it.  Rank 0 prints one JSON line.
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOADS = {
    "gpt2-124m": dict(n_layer=12, n_embd=768, n_head=12, vocab_size=50257, padded_vocab=50304,
                      max_T=1024, B=16, T=1024),
    "gpt2-350m": dict(n_layer=24, n_embd=1024, n_head=16, vocab_size=50257, padded_vocab=50304,
                      max_T=1024, B=16, T=1024),
    # micro-batch 64 x 8 accumulation (524,288 tokens per optimizer step), warmup + cosine LR,
    # then a 20-batch evaluation pass on a separate stream (seed 4)
    "gpt2-124m-accum": dict(n_layer=12, n_embd=768, n_head=12, vocab_size=50257,
                            padded_vocab=50304, max_T=1024, B=64, T=1024, accum=8, eval_batches=20),
}
# the fused LM head + cross-entropy alone (forward loss, backward dHidden and dW), bf16:
# hidden [8192, 768] ~ N(0, 1), tied weight [50304, 768] ~ N(0, 0.02), targets uniform in
# [0, 50257), all from seed 2
LMHEAD = {"lmhead-ce-8192": dict(M=8192, C=768, Vp=50304, V=50257)}
# schedule of the accumulation workload: max 6e-4, min 6e-5, 100 warmup steps; the decay
# length is the run's choice (its token budget), 10,000 optimizer steps here
LR_SCHEDULE = dict(max_lr=6e-4, min_lr=6e-5, warmup_steps=100, total_steps=10000)
METRIC = "GPT-2 124M training tokens/s (fwd+bwd+AdamW, T=1024, bf16) and MFU"
# the line's metric names the model the workload trains
METRICS = {"gpt2-124m": METRIC,
           "gpt2-124m-accum": METRIC,
           "lmhead-ce-8192": "fused LM-head + cross-entropy fwd+bwd TFLOP/s (8192x768x50304, bf16)",
           "gpt2-350m": "GPT-2 350M training tokens/s (fwd+bwd+AdamW, T=1024, bf16) and MFU"}
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HP = dict(lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, max_norm=1.0)


def n_params(w):
    C, L, V, Tm = w["n_embd"], w["n_layer"], w["padded_vocab"], w["max_T"]
    per_layer = 12 * C * C + 13 * C
    return V * C + Tm * C + L * per_layer + 2 * C


def flops_per_token(w):
    """Algorithmic: 6N (matmul fwd+bwd) + 6*L*C*T (causal attention)."""
    return 6 * n_params(w) + 6 * w["n_layer"] * w["n_embd"] * w["T"]


def stored_traffic(group, workload, launches_per_step):
    """DRAM bytes per launch of a kernel group from the committed ncu capture
    (profiles/gemm_dram_traffic_*.json: one block's GEMMs run standalone at the
    step's shapes, so bytes per launch carry over to the 12-block step), or None
    when that capture was taken on another workload or on kernel sources that
    have changed since."""
    path = os.path.join(ROOT, "profiles", "gemm_dram_traffic_gpt2_124m_layer_m16384.json")
    if workload != "gpt2-124m" or not os.path.exists(path):
        return None, None
    rec = json.load(open(path))
    if group not in rec:
        return None, None
    h = hashlib.sha256()
    for f in sorted(rec["kernel_sources"]):
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if h.hexdigest() != rec["kernel_sources_sha256"]:
        return None, "kernel sources changed since the capture"
    g = rec[group]
    per_launch = g["dram_bytes_per_step"] / max(1.0, launches_per_step)
    return per_launch, ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one block's "
                        f"{rec['per_layer']['launches']} GEMM launches captured standalone "
                        "(opbench layer_gemms at M=16384), per launch; "
                        "profiles/gemm_dram_traffic_gpt2_124m_layer_m16384.json")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle legs
def oracle_sample(w, stream, T_sample, with_adamw=True):
    """Times one oracle fwd+bwd of 1 x T_sample tokens (+ one clip/AdamW pass).

    Returns (seconds for the fwd+bwd, seconds for AdamW, threads)."""
    import oracle
    m = oracle.Model(w["n_layer"], w["n_embd"], w["n_head"], w["vocab_size"], w["padded_vocab"],
                     w["max_T"])
    named = synth.init_params(0, m.shapes())
    p = m.pack(named, np.float32)
    x, y = oracle.batch_from_stream(stream, 0, 1, T_sample)
    t0 = time.perf_counter()
    _, _, g, _ = m.fwd_bwd(p, x, y)
    t1 = time.perf_counter()
    ta = 0.0
    if with_adamw:
        mm, vv = np.zeros_like(p), np.zeros_like(p)
        t2 = time.perf_counter()
        m.clip_adamw(p, g, mm, vv, 1, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"],
                     HP["weight_decay"], HP["max_norm"])
        ta = time.perf_counter() - t2
    return t1 - t0, ta, oracle.num_threads()


def cpu_baseline(w, stream):
    """The oracle on a bounded sample: one 1 x T sequence fwd+bwd and one AdamW
    pass, scaled to one optimizer step (accum x B x T tokens)."""
    T, acc = w["T"], w.get("accum", 1)
    t_seq, t_adam, cores = oracle_sample(w, stream, T)
    step_s = acc * w["B"] * t_seq + t_adam
    return {"value": acc * w["B"] * T / step_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"oracle fp32: fwd+bwd of 1 x {T} tokens ({t_seq:.1f} s) + one clip+AdamW over "
                      f"all {n_params(w)} params ({t_adam:.2f} s), scaled to one {acc}x{w['B']}x{T} step"}


def run_reference(args, w, wname):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    T_s = 256
    stream = synth.token_stream(3, (args.warmup + args.steps + 1) * T_s + 1)
    import oracle
    m = oracle.Model(w["n_layer"], w["n_embd"], w["n_head"], w["vocab_size"], w["padded_vocab"],
                     w["max_T"])
    p = m.pack(synth.init_params(0, m.shapes()), np.float32)
    mm, vv = np.zeros_like(p), np.zeros_like(p)
    share = T_s / (w.get("accum", 1) * w["B"] * w["T"])  # one AdamW per optimizer step
    times = []
    for i in range(args.warmup + args.steps):
        x, y = oracle.batch_from_stream(stream, i * T_s, 1, T_s)
        t0 = time.perf_counter()
        _, _, g, _ = m.fwd_bwd(p, x, y)
        t1 = time.perf_counter()
        m.clip_adamw(p, g, mm, vv, i + 1, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"],
                     HP["weight_decay"], HP["max_norm"])
        t2 = time.perf_counter()
        if i >= args.warmup:
            times.append((t1 - t0) + share * (t2 - t1))
    total = sum(times)
    value = args.steps * T_s / total
    sample = (f"oracle fp32 on the host cores: each step = fwd+bwd of 1 x {T_s} tokens of the "
              f"{wname} workload + AdamW time x {share:.4f} "
              f"(one update per {w.get('accum', 1)}x{w['B']}x{w['T']} tokens)")
    line = {"impl": "reference", "metric": METRICS[wname], "value": value, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": wname, "global_batch": w["B"], "seq_len": w["T"],
                       "sample_tokens_per_step": T_s, "parallelism": "none (CPU)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- LM head alone
def lmhead_inputs(w):
    """The seed-2 inputs of the LM-head workload (float32 host arrays)."""
    M, Cc, Vp, V = w["M"], w["C"], w["Vp"], w["V"]
    h = synth.normal(synth.derive_key(2, 1), M * Cc, 1.0).reshape(M, Cc).astype(np.float32)
    W = synth.normal(synth.derive_key(2, 2), Vp * Cc, 0.02).reshape(Vp, Cc).astype(np.float32)
    y = synth.randint(synth.derive_key(2, 3), M, V).astype(np.int32)
    return h, W, y


def lmhead_cpu_baseline(w, h, W, y, rows=64):
    """The oracle (fp32) on the first `rows` rows, scaled to all M rows (the work
    per row does not depend on the other rows)."""
    import oracle
    t0 = time.perf_counter()
    oracle.lmhead_ce(h[:rows], W, y[:rows], w["V"])
    dt = (time.perf_counter() - t0) * w["M"] / rows
    fl = 3 * 2.0 * w["M"] * w["C"] * w["Vp"]
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"oracle fp32 forward + backward on {rows} of the {w['M']} rows "
                      f"({dt * rows / w['M']:.1f} s), scaled to all rows"}


def run_lmhead(args, w, wname):
    """Config 2: the tied head with mean cross-entropy alone, forward and backward,
    as one op-level call (gpt2_lmhead_ce) per step on device-resident inputs."""
    import ctypes
    import torch
    import decoder_only_lm_b200 as g
    M, Cc, Vp, V = w["M"], w["C"], w["Vp"], w["V"]
    h_np, W_np, y_np = lmhead_inputs(w)
    h = torch.from_numpy(h_np).cuda().bfloat16()
    W = torch.from_numpy(W_np).cuda().bfloat16()
    y = torch.from_numpy(y_np).cuda()
    ws_b = ctypes.c_size_t()
    g._check(g.lib.gpt2_lmhead_ce_workspace(M, Cc, Vp, g.BF16, ctypes.byref(ws_b)))
    ws = torch.empty(ws_b.value, dtype=torch.uint8, device="cuda")
    loss = torch.empty(1, device="cuda")
    lse = torch.empty(M, device="cuda")
    dh = torch.empty_like(h)
    dW = torch.zeros((Vp, Cc), device="cuda")  # accumulated into by every call
    st = torch.cuda.current_stream()

    def call(hh=h, yy=y):
        g._check(g.lib.gpt2_lmhead_ce(hh.data_ptr(), W.data_ptr(), yy.data_ptr(), M, Cc, Vp, V, g.BF16,
                                      1.0, loss.data_ptr(), lse.data_ptr(), dh.data_ptr(),
                                      dW.data_ptr(), ws.data_ptr(), ws_b.value, st.cuda_stream))

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = g.launch_count()
    e0.record(st)
    for _ in range(args.steps):
        call()
    e1.record(st)
    torch.cuda.synchronize()
    n1 = g.launch_count()
    clk = clocks.stop()
    assert g.device_error() == 0
    ms = e0.elapsed_time(e1) / args.steps
    fl = 3 * 2.0 * M * Cc * Vp  # forward, dHidden, dW (the recompute is extra work)
    tflops = fl / (ms / 1e3) / 1e12
    peaks, peak_src = load_peaks()
    # end to end: hidden and targets from pinned host memory, the loss read back
    hh = torch.from_numpy(h_np).bfloat16().pin_memory()
    yh = torch.from_numpy(y_np).pin_memory()
    hd, yd = torch.empty_like(h), torch.empty_like(y)
    times = []
    lh = torch.empty(1, pin_memory=True)
    for i in range(max(3, args.steps // 2) + 1):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        hd.copy_(hh, non_blocking=True)
        yd.copy_(yh, non_blocking=True)
        call(hd, yd)
        lh.copy_(loss, non_blocking=True)
        b.record(st)
        torch.cuda.synchronize()
        if i > 0:
            times.append(a.elapsed_time(b))
    e_ms = sum(times) / len(times)
    line = {
        "metric": METRICS[wname], "value": tflops, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (hidden N(0,1), weight N(0,0.02), targets uniform, seed 2)",
        "config": {"workload": wname, "rows": M, "hidden": Cc, "padded_vocab": Vp, "vocab": V,
                   "flops_per_step": fl, "flops": "algorithmic: 3 x 2 M C Vp (forward, dHidden, "
                   "dW); the backward's recompute of the logits is extra",
                   "l2": "working set (weights 77 MB, fp32 dW 155 MB, workspace 230 MB) > 126 MB L2;"
                         " no flush"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"], "traffic": None,
                     "kernel": "gpt2_lmhead_ce (LSE-partial GEMM, merge, per 2048-row chunk: "
                               "CE-gradient GEMM, dHidden GEMM + split reduction, dW GEMM)",
                     "peak_source": f"{peak_src} bf16 burst (op timed alone)",
                     "measured": "CUDA events around the timed calls on the launching stream"},
        "clocks": clk,
        "gpu_launches": n1 - n0,
        "e2e": {"value": fl / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * Cc * 2 + M * 4, "d2h_bytes_per_step": 4, "ms_per_step": e_ms,
                "api": "gpt2_lmhead_ce (host bf16 hidden + int32 targets in, loss out)"},
        "cpu_baseline": None if args.no_cpu_baseline else lmhead_cpu_baseline(w, h_np, W_np, y_np),
    }
    print(json.dumps(line), flush=True)


def run_lmhead_reference(args, w, wname):
    """The oracle on the LM-head workload, each step a 16-row sample scaled to
    all rows."""
    import oracle
    h, W, y = lmhead_inputs(w)
    rows = 16
    fl = 3 * 2.0 * w["M"] * w["C"] * w["Vp"]
    times = []
    for i in range(args.warmup + args.steps):
        r0 = (i * rows) % w["M"]
        t0 = time.perf_counter()
        oracle.lmhead_ce(h[r0:r0 + rows], W, y[r0:r0 + rows], w["V"])
        if i >= args.warmup:
            times.append((time.perf_counter() - t0) * w["M"] / rows)
    step_s = sum(times) / len(times)
    value = fl / step_s / 1e12
    sample = (f"oracle fp32 forward + backward on {rows} rows per step, scaled to all {w['M']} rows")
    print(json.dumps({
        "impl": "reference", "metric": METRICS[wname], "value": value, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seed 2)", "config": {"workload": wname, "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
        flush=True)


# ---------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default="gpt2-124m", choices=sorted(WORKLOADS) + sorted(LMHEAD))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in LMHEAD:
        if int(os.environ.get("RANK", "0")) != 0:
            return  # one GPU's op; further ranks have nothing to do
        if args.impl == "reference":
            return run_lmhead_reference(args, LMHEAD[args.workload], args.workload)
        return run_lmhead(args, LMHEAD[args.workload], args.workload)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w, args.workload)

    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import decoder_only_lm_b200 as g

    B, T = w["B"], w["T"]
    acc = w.get("accum", 1)  # micro-batches per optimizer step
    steps_total = args.warmup + args.steps
    # timed steps, then the e2e leg's windows at step index steps_total + 1
    n_tok = ((steps_total + 2) * acc * world + 2) * B * T + 1
    stream_np = synth.token_stream(3, n_tok)
    stream = torch.from_numpy(stream_np.view(np.int16)).cuda()
    model = g.GPT2(w["n_layer"], w["n_embd"], w["n_head"], w["vocab_size"], w["padded_vocab"],
                   w["max_T"], bf16=True, max_B=B, max_Tseq=T)
    model.set_params(synth.init_params(0, model.shapes()))
    # data parallel: the library averages each gradient bucket (NCCL all-reduce on
    # its communication stream) as the last micro-batch's backward finishes it
    if world > 1:
        from decoder_only_lm_b200.dp import init_library_exchange
        init_library_exchange(model)

    def hp_at(i):
        hp = dict(HP)
        if acc > 1:
            hp["lr"] = g.cosine_lr(i, **LR_SCHEDULE)
        return hp

    def step(i):
        # one optimizer step: acc micro-batches whose gradients add up (loss scaled
        # by 1/acc), consecutive windows of the stream (rank-offset for data parallel)
        model.zero_grad()
        for a in range(acc):
            off = ((i * acc + a) * world + rank) * B * T
            x, y = model.batch_from_stream(stream, off, B, T)
            model.forward_loss(x, y, loss=False)
            if world > 1:
                model.dp_sync(a == acc - 1)  # exchange after the last micro-batch only
            model.backward(1.0 / acc)
        model.clip_adamw_step(**hp_at(i), norm=False)

    # Each optimizer step is replayed from a CUDA graph recorded by
    # gpt2_stream_begin (windows cut at a device cursor that advances through
    # the stream: rank r starts at B*T*r and advances B*T*N; the learning rate is
    # set before each replay).  With N > 1 the graph holds the bucketed
    # gradient exchange too.
    lrs = [hp_at(i)["lr"] for i in range(steps_total)]
    model.stream_begin(stream, rank * B * T, world * B * T, B, T, accum=acc,
                       **{k: v for k, v in HP.items() if k != "lr"})
    kernels_per_step = model.stream_kernels()  # what each replay launches
    model.stream_steps(lrs[:args.warmup])
    model.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    # timed region: K steps back to back, no profiling
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(st)
    model.stream_steps(lrs[args.warmup:])
    e1.record(st)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    cursor = model.stream_end()  # also surfaces any device-side error of the timed steps
    assert cursor == (rank + steps_total * acc * world) * B * T, cursor
    if world > 1:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = t.item()
        dist.barrier()
    model.synchronize()  # surfaces any device-side error of the timed steps

    # the same K steps again with the library's per-kernel-group CUDA events on
    # (the events perturb the step slightly, so they stay out of the timed region)
    model.profile_reset()
    model.profile(True)
    for i in range(args.warmup, steps_total):
        step(i)
    model.profile(False)
    prof = model.profile_read()
    model.synchronize()

    ms_per_step = ms / args.steps
    tokens = args.steps * acc * B * T * world
    value = tokens / (ms / 1e3)
    fpt = flops_per_token(w)
    achieved_tflops = value * fpt / 1e12
    peaks, peak_src = load_peaks()

    # dominant kernel group, measured live over the timed region
    groups = {k: v for k, v in prof.items() if isinstance(v, dict)}
    dom = max(groups, key=lambda k: groups[k]["ms"])
    d = groups[dom]
    per_launch_ms = d["ms"] / max(1, d["launches"])
    traffic, traffic_src = stored_traffic(dom, args.workload, d["launches"] / max(1, args.steps))
    if d["flops"] > 0 and dom in ("gemm", "lmhead", "attn_fwd", "attn_bwd"):
        ach = d["flops"] / (d["ms"] / 1e3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "traffic": traffic, "traffic_source": traffic_src,
                "kernel": dom, "launches": d["launches"], "ms_per_launch": per_launch_ms,
                "peak_source": f"{peak_src} bf16 sustained",
                "measured": "CUDA events around every launch of the group, on the library's stream, "
                            "over a profiled repeat of the timed steps"}
    else:
        ach = d["bytes"] / (d["ms"] / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                "traffic": traffic, "traffic_source": traffic_src, "kernel": dom,
                "launches": d["launches"],
                "ms_per_launch": per_launch_ms, "peak_source": f"{peak_src} copy",
                "measured": "CUDA events around every launch of the group, on the library's stream, "
                            "over a profiled repeat of the timed steps"}

    # end to end through the public API: host tokens in, loss + norm out, every step
    e2e = None
    if not args.no_e2e:
        # one pinned host buffer pair per micro-batch, filled before the timed step
        xh = torch.empty((acc, B, T), dtype=torch.int32, pin_memory=True)
        yh = torch.empty((acc, B, T), dtype=torch.int32, pin_memory=True)
        k_e2e = max(3, args.steps // 2)
        times = []
        for i in range(k_e2e + 1):
            for m_ in range(acc):
                off = (((steps_total + 1) * acc + m_) * world + rank) * B * T
                win = stream_np[off:off + B * T + 1].astype(np.int32)
                xh.numpy()[m_] = win[:-1].reshape(B, T)
                yh.numpy()[m_] = win[1:].reshape(B, T)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            if world == 1 and acc == 1:
                model.train_step(xh.numpy()[0], yh.numpy()[0], **HP, read=True)
            else:
                model.zero_grad()
                for m_ in range(acc):
                    model.forward_loss(xh.numpy()[m_], yh.numpy()[m_], loss=(m_ == acc - 1))
                    if world > 1:
                        model.dp_sync(m_ == acc - 1)
                    model.backward(1.0 / acc)
                model.clip_adamw_step(**hp_at(steps_total + i), norm=True)
            b.record(st)
            torch.cuda.synchronize()
            if i > 0:
                times.append(a.elapsed_time(b))
        e_ms = sum(times) / len(times)
        if world > 1:
            t = torch.tensor([e_ms], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = t.item()
        e2e = {"value": acc * B * T * world / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": acc * 2 * B * T * 4, "d2h_bytes_per_step": 8,
               "ms_per_step": e_ms,
               "api": ("gpt2_train_step" if acc == 1 and world == 1 else
                       f"{acc} x (gpt2_forward_loss + gpt2_backward) + gpt2_clip_adamw_step")
                      + " (host int32 tokens, loss + norm read back)"}

    # evaluation pass (no activations kept, one loss read per batch), separate stream
    evaluation = None
    if w.get("eval_batches"):
        nb = w["eval_batches"]
        ev_np = synth.token_stream(4, nb * B * T + 1)
        ev = torch.from_numpy(ev_np.view(np.int16)).cuda()
        losses = []
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for k in range(nb):
            x, y = model.batch_from_stream(ev, k * B * T, B, T)
            losses.append(model.eval_loss(x, y))
        b.record(st)
        torch.cuda.synchronize()
        ev_ms = a.elapsed_time(b)
        evaluation = {"batches": nb, "tokens": nb * B * T, "ms": ev_ms,
                      "tokens_per_s": nb * B * T / (ev_ms / 1e3),
                      "mean_loss": sum(losses) / nb,
                      "data": "Zipf(1.1)/EOT stream seed 4, consecutive windows"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, stream_np)

    if rank == 0:
        line = {
            "metric": METRICS[args.workload], "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (Zipf(1.1)/EOT token stream seed 3, N(0,0.02) weights seed 0)",
            "config": {"workload": args.workload, "global_batch": acc * B * world, "seq_len": T,
                       "micro_batch_per_gpu": B, "accumulation": acc, "parallelism": f"dp{world}",
                       "step_launch": "CUDA graph of one optimizer step, replayed (gpt2_stream_steps)"
                                      + (", bucketed NCCL gradient exchange inside" if world > 1 else ""),
                       "l2": "working set (saved activations and weights + optimizer state, GBs) "
                             ">> 126 MB L2; no flush"},
            # MFU is against the dense bf16 datasheet peak (2250 TFLOP/s per GPU);
            # the ratios to this pool's measured cuBLAS peaks are context only
            "mfu": {"value": achieved_tflops / (DATASHEET_BF16_TFLOPS * world),
                    "peak_tflops": DATASHEET_BF16_TFLOPS * world,
                    "peak_source": "dense bf16 datasheet, per GPU x n_gpus",
                    "algorithmic_flops_per_step": fpt * acc * B * T * world,
                    "achieved_tflops": achieved_tflops,
                    "context": {"vs_measured_burst": achieved_tflops / (peaks["bf16_tflops"] * world),
                                "vs_measured_sustained":
                                    achieved_tflops / (peaks["bf16_tflops_sustained"] * world),
                                "measured_peak_source": peak_src}},
            "roofline": roof,
            "clocks": clk,
            # kernels launched in the timed region: the step graph's kernels, once per
            # replayed step (the per-call profiled repeat launches the same set)
            "gpu_launches": kernels_per_step * args.steps,
            "gpu_launches_per_step": kernels_per_step,
            "profiled_pass_launches": prof["total_launches"],
            "profiled_pass_ms_per_step": sum(v["ms"] for v in groups.values()) / args.steps,
            "kernel_groups_ms_per_step": {k: round(v["ms"] / args.steps, 4) for k, v in groups.items()},
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        if evaluation is not None:
            line["eval"] = evaluation
        print(json.dumps(line), flush=True)
    model.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
