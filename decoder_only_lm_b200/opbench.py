"""Time one op-level entry point of the library on synthetic bf16 inputs.

    python -m decoder_only_lm_b200.opbench matmul --M 16384 --N 3072 --K 768 [--a-mn] [--b-mn]
    python -m decoder_only_lm_b200.opbench lmhead --M 8192 --C 768 --Vp 50304 [--fwd-only]
    python -m decoder_only_lm_b200.opbench attention --B 16 --T 1024 --C 768 --H 12 [--bwd]
    python -m decoder_only_lm_b200.opbench layernorm --M 16384 --C 768 [--bwd]
    python -m decoder_only_lm_b200.opbench linear --M 16384 --N 3072 --K 768 --epi gelu [--graph]
    python -m decoder_only_lm_b200.opbench layer_gemms --M 16384 --C 768 (one block's linear layers)
    python -m decoder_only_lm_b200.opbench sample --B 16 --V 50257 [--temperature 0.8 --top-k 0 --top-p 0.9]
    python -m decoder_only_lm_b200.opbench generate --B 16 --T0 64 --new 64 [--cached] (GPT-2 124M, bf16)

Each call is timed with CUDA events on the current stream after warm-up and
reported as one JSON line (ms per call, and TFLOP/s or GB/s of algorithmic
work).  Small fixed cases of this script are what the ncu captures under
profiles/ run.
"""
from __future__ import annotations

import argparse
import json

import torch

import decoder_only_lm_b200 as g


def timed(fn, iters, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def timed_graph(fn, iters, warmup):
    """As timed(), but the iters calls are captured once as a CUDA graph and
    the replay is timed: no host (binding) time between the launches."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for _ in range(iters):
            fn()
    gr.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    gr.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


EPIS = {"bias": g.LINEAR_BIAS, "gelu": g.LINEAR_BIAS_GELU, "resid": g.LINEAR_RESIDUAL,
        "gelu_bwd": g.LINEAR_GELU_BWD}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["matmul", "lmhead", "attention", "layernorm", "linear",
                                   "sample", "generate", "layer_gemms"])
    ap.add_argument("--temperature", type=float, default=0.8)
    ap.add_argument("--top-k", type=int, default=0)
    ap.add_argument("--top-p", type=float, default=0.9)
    ap.add_argument("--T0", type=int, default=64)
    ap.add_argument("--new", type=int, default=64)
    ap.add_argument("--cached", action="store_true", help="generate with the key/value cache")
    ap.add_argument("--epi", choices=sorted(EPIS), default="bias")
    ap.add_argument("--graph", action="store_true",
                    help="time a CUDA-graph replay of the calls (no host time in between)")
    ap.add_argument("--M", type=int, default=16384)
    ap.add_argument("--N", type=int, default=3072)
    ap.add_argument("--K", type=int, default=768)
    ap.add_argument("--C", type=int, default=768)
    ap.add_argument("--Vp", type=int, default=50304)
    ap.add_argument("--V", type=int, default=50257)
    ap.add_argument("--B", type=int, default=16)
    ap.add_argument("--T", type=int, default=1024)
    ap.add_argument("--H", type=int, default=12)
    ap.add_argument("--a-mn", action="store_true")
    ap.add_argument("--b-mn", action="store_true")
    ap.add_argument("--accumulate", action="store_true")
    ap.add_argument("--bwd", action="store_true")
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args()
    if a.graph:
        global timed
        timed = timed_graph
    torch.manual_seed(0)
    dev = "cuda"
    out = {"op": a.op}
    if a.op == "matmul":
        A = torch.randn((a.K, a.M) if a.a_mn else (a.M, a.K), device=dev).bfloat16()
        B = torch.randn((a.K, a.N) if a.b_mn else (a.N, a.K), device=dev).bfloat16()
        D = torch.zeros((a.M, a.N), device=dev, dtype=torch.float32 if a.accumulate else torch.bfloat16)
        fn = lambda: g.matmul(A, B, a_kmajor=not a.a_mn, b_kmajor=not a.b_mn, M=a.M, N=a.N, K=a.K,
                              out=D, accumulate=a.accumulate)
        ms = timed(fn, a.iters, a.warmup)
        fl = 2.0 * a.M * a.N * a.K
        out.update(M=a.M, N=a.N, K=a.K, a_mn=a.a_mn, b_mn=a.b_mn, ms=ms, tflops=fl / ms / 1e9)
    elif a.op == "linear":
        # one linear layer of the block with its fused epilogue: x [M,K], W [N,K]
        # (GELU backward: W [K,N]), bf16
        x = torch.randn((a.M, a.K), device=dev).bfloat16()
        w_kn = a.epi == "gelu_bwd"
        w = (torch.randn((a.K, a.N) if w_kn else (a.N, a.K), device=dev) / a.K ** 0.5).bfloat16()
        bias = None if w_kn else torch.randn(a.N, device=dev)
        odt = torch.float32 if a.epi == "resid" else torch.bfloat16
        o = torch.empty((a.M, a.N), device=dev, dtype=odt)
        o2 = torch.empty((a.M, a.N), device=dev, dtype=torch.bfloat16) if a.epi == "gelu" else None
        inp = None
        if a.epi == "resid":
            inp = torch.randn((a.M, a.N), device=dev)
        elif a.epi == "gelu_bwd":
            inp = torch.randn((a.M, a.N), device=dev).bfloat16()
        fn = lambda: g.linear(EPIS[a.epi], x, w, bias=bias, inp=inp, w_kn=w_kn, out=o, out2=o2)
        ms = timed(fn, a.iters, a.warmup)
        fl = 2.0 * a.M * a.N * a.K
        out.update(M=a.M, N=a.N, K=a.K, epi=a.epi, ms=ms, tflops=fl / ms / 1e9)
    elif a.op == "layer_gemms":
        # the twelve contractions of one transformer block as the training step
        # issues them (M = B*T rows, C, F = 4C, bf16 operands): forward QKV + bias,
        # attention projection + residual, fc + bias + GELU, fc projection +
        # residual; backward per layer in reverse: fc projection dX with GELU',
        # its dW, fc dX, its dW, projection dX, its dW, QKV dX, its dW (fp32 dW
        # accumulated, split along the rows where the cost model picks it)
        M, Cc = a.M, a.C
        F = 4 * Cc
        bf = torch.bfloat16
        r = lambda *s_: torch.randn(*s_, device=dev).to(bf)
        x, att, g_, u = r(M, Cc), r(M, Cc), r(M, F), r(M, F)
        Wqkv, Wp, Wfc, Wfp = r(3 * Cc, Cc), r(Cc, Cc), r(F, Cc), r(Cc, F)
        bq, bp, bfc, bfp = (torch.randn(n, device=dev) for n in (3 * Cc, Cc, F, Cc))
        res = torch.randn(M, Cc, device=dev)
        res2 = torch.empty_like(res)
        qkv, fc_u, fc_g = torch.empty(M, 3 * Cc, device=dev, dtype=bf), torch.empty(M, F, device=dev, dtype=bf), torch.empty(M, F, device=dev, dtype=bf)
        dres, du, dln, dqkv = r(M, Cc), torch.empty(M, F, device=dev, dtype=bf), torch.empty(M, Cc, device=dev, dtype=bf), r(M, 3 * Cc)
        dWqkv, dWp, dWfc, dWfp = (torch.zeros(*w.shape, device=dev) for w in (Wqkv, Wp, Wfc, Wfp))

        def fn():
            g.linear(g.LINEAR_BIAS, x, Wqkv, bias=bq, out=qkv)
            g.linear(g.LINEAR_RESIDUAL, att, Wp, bias=bp, inp=res, out=res2)
            g.linear(g.LINEAR_BIAS_GELU, x, Wfc, bias=bfc, out=fc_g, out2=fc_u)
            g.linear(g.LINEAR_RESIDUAL, g_, Wfp, bias=bfp, inp=res2, out=res)
            g.linear(g.LINEAR_GELU_BWD, dres, Wfp, inp=u, w_kn=True, out=du)
            g.matmul(dres, g_, a_kmajor=False, b_kmajor=False, M=Cc, N=F, K=M, out=dWfp, accumulate=True)
            g.matmul(du, Wfc, a_kmajor=True, b_kmajor=False, M=M, N=Cc, K=F, out=dln)
            g.matmul(du, x, a_kmajor=False, b_kmajor=False, M=F, N=Cc, K=M, out=dWfc, accumulate=True)
            g.matmul(dres, Wp, a_kmajor=True, b_kmajor=False, M=M, N=Cc, K=Cc, out=dln)
            g.matmul(dres, att, a_kmajor=False, b_kmajor=False, M=Cc, N=Cc, K=M, out=dWp, accumulate=True)
            g.matmul(dqkv, Wqkv, a_kmajor=True, b_kmajor=False, M=M, N=Cc, K=3 * Cc, out=dln)
            g.matmul(dqkv, x, a_kmajor=False, b_kmajor=False, M=3 * Cc, N=Cc, K=M, out=dWqkv, accumulate=True)

        ms = timed(fn, a.iters, a.warmup)
        fl = 3 * 2.0 * M * 12 * Cc * Cc
        out.update(M=M, C=Cc, ms=ms, tflops=fl / ms / 1e9)
    elif a.op == "sample":
        # next-token choice over B rows of fp32 logits (the padded width, V drawn)
        z = 3.0 * torch.randn((a.B, a.Vp), device=dev)
        u = torch.rand(a.B, device=dev)
        o = torch.empty(a.B, dtype=torch.int32, device=dev)
        fn = lambda: g.sample(z, a.V, a.temperature, a.top_k, a.top_p, u, out=o)
        ms = timed(fn, a.iters, a.warmup)
        out.update(B=a.B, V=a.V, temperature=a.temperature, top_k=a.top_k, top_p=a.top_p, ms=ms,
                   gbs=a.B * a.V * 4 / ms / 1e6)
    elif a.op == "generate":
        # GPT-2 124M (bf16, N(0, 0.02) weights): a prompt of T0 ids, then `new`
        # tokens, each recomputing the whole window (no KV cache)
        import synth
        m = g.GPT2(12, 768, 12, 50257, 50304, 1024, bf16=True, max_B=a.B, max_Tseq=1024)
        m.set_params(synth.init_params(0, m.shapes()))
        prompt = torch.randint(0, 50257, (a.B, a.T0), dtype=torch.int32, device=dev)
        u = torch.rand((a.new, a.B), device=dev)
        for _ in range(a.warmup):
            m.generate(prompt, 2, a.temperature, a.top_k, a.top_p, u[:2], cached=a.cached)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        m.generate(prompt, a.new, a.temperature, a.top_k, a.top_p, u, cached=a.cached)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        out.update(B=a.B, T0=a.T0, new=a.new, cached=a.cached, temperature=a.temperature, top_k=a.top_k,
                   top_p=a.top_p, ms=ms, ms_per_token_step=ms / a.new,
                   tokens_per_s=a.B * a.new / ms * 1e3)
        m.close()
    elif a.op == "lmhead":
        h = torch.randn((a.M, a.C), device=dev).bfloat16()
        W = (0.02 * torch.randn((a.Vp, a.C), device=dev)).bfloat16()
        y = torch.randint(0, a.V, (a.M,), device=dev, dtype=torch.int32)
        fn = lambda: g.lmhead_ce(h, W, y, a.V, grads=not a.fwd_only)
        ms = timed(fn, a.iters, a.warmup)
        n_gemm = 1 if a.fwd_only else 3
        fl = n_gemm * 2.0 * a.M * a.C * a.Vp
        out.update(M=a.M, C=a.C, Vp=a.Vp, fwd_only=a.fwd_only, ms=ms, tflops_algorithmic=fl / ms / 1e9)
    elif a.op == "attention":
        qkv = torch.randn((a.B, a.T, 3 * a.C), device=dev).bfloat16()
        o, lse = g.attention_fwd(qkv, a.H)
        dout = torch.randn_like(o)
        if a.bwd:
            fn = lambda: g.attention_bwd(dout, qkv, o, lse, a.H)
            mult = 4.0
        else:
            fn = lambda: g.attention_fwd(qkv, a.H)
            mult = 2.0
        ms = timed(fn, a.iters, a.warmup)
        fl = mult * a.B * a.H * a.T * a.T * (a.C // a.H)  # causal half of 2 (4) full matmuls
        out.update(B=a.B, T=a.T, C=a.C, H=a.H, bwd=a.bwd, ms=ms, tflops_algorithmic=fl / ms / 1e9)
    else:
        x = torch.randn((a.M, a.C), device=dev)
        gam = torch.randn(a.C, device=dev)
        bet = torch.randn(a.C, device=dev)
        y, mean, rstd = g.layernorm_fwd(x, gam, bet, out_dtype=torch.bfloat16)
        if a.bwd:
            dy = torch.randn((a.M, a.C), device=dev).bfloat16()
            dx = torch.zeros_like(x)
            fn = lambda: g.layernorm_bwd(dy, x, mean, rstd, gam, dx=dx)
            by = a.M * a.C * (2 + 4 + 8)
        else:
            fn = lambda: g.layernorm_fwd(x, gam, bet, out_dtype=torch.bfloat16)
            by = a.M * a.C * (4 + 2)
        ms = timed(fn, a.iters, a.warmup)
        out.update(M=a.M, C=a.C, bwd=a.bwd, ms=ms, gbs=by / ms / 1e6)
    out["device_error"] = g.device_error()
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
