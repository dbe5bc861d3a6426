"""GPU path vs the oracle at the shapes the GPT-2 124M step runs at.

The small parity cases (test_gpu_parity, test_gpu_ops) fit in one or two
tiles per CTA pair.  These cases reach the paths that only the full-size
step takes:

* one whole 124M step (L=12, C=768, H=12, V=50257 padded to 50304) on one
  T=1024 sequence of the Zipf/end-of-text stream: loss, every gradient and
  the parameters after one clip + AdamW, with the bf16 bars;
* attention at T=1024, H=12, D=64 (16 key tiles per query tile), including
  scores large enough that the running row maximum keeps growing, so the
  output accumulator is rescaled while the key tiles stream by;
* each fused linear-layer epilogue at M=16384 rows with the layer's own N and
  K (several output tiles per CTA pair, both TMEM accumulators in turn), on
  sampled rows;
* the weight-gradient contraction (both operands MN-major, fp32 accumulate
  into existing values) at K=16384 rows, where the output is split along K.

Sources: the GPT-2 training step of the lecture summary and of the Zero
framework's "Transformer Block" and "Attention" sections (pre-LN block,
causal attention, tanh GELU, tied head); the B*T+1 window of chapter 28.3.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.parity_util import TOL, Shape, gpu_model, inputs, rel_l2
from tests.test_gpu_parity import check_step

pytestmark = pytest.mark.gpu

GPT2_124M_T1024 = Shape(12, 768, 12, 50257, 50304, 1024, 1, 1024)
# GPT-2 medium's layer shapes (C=1024, H=16, F=4096, padded vocabulary) with two
# of its 24 layers: a different number of tiles per row, K=1024 for the head
# and the fc layer, and LayerNorm rows of 1024 columns
GPT2_350M_2L_T1024 = Shape(2, 1024, 16, 50257, 50304, 1024, 1, 1024)
# the benchmarked configurations: 16 sequences of 1024 tokens per step
GPT2_124M_B16 = Shape(12, 768, 12, 50257, 50304, 1024, 16, 1024)
GPT2_350M_B16 = Shape(24, 1024, 16, 50257, 50304, 1024, 16, 1024)
# the micro-batch of the accumulation workload: 64 sequences (65536 rows)
GPT2_124M_B64 = Shape(12, 768, 12, 50257, 50304, 1024, 64, 1024)


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available()
    return torch


@pytest.fixture(scope="module")
def g(torch):
    import decoder_only_lm_b200 as g
    return g


@pytest.mark.parametrize("s", [GPT2_124M_T1024, GPT2_350M_2L_T1024], ids=["124m", "350m_2layers"])
def test_step_t1024_zipf(torch, s):
    """One bf16 training step on the first 1024-token window of the seed-3
    Zipf/end-of-text stream, against the float64 oracle: GPT-2 124M whole, and
    two layers of GPT-2 medium."""
    om, named, stream, x, y = inputs(s, seed=0, stream_seed=3, uniform=False)
    assert (x == synth.EOT).any() and np.mean(x == 0) > 0.05  # the stream's skew is present
    flat = om.pack(named)
    lo, rlo, go, _ = om.fwd_bwd(flat, x, y, row_loss=True)
    gm = gpu_model(s, True)
    gm.set_params(named)
    rl = torch.empty(s.B * s.T, dtype=torch.float32, device="cuda")
    gm.zero_grad()
    lg = gm.forward_loss(torch.from_numpy(x).cuda(), torch.from_numpy(y).cuda(), row_loss=rl)
    gm.backward()
    gm.synchronize()
    check_step(om, gm, named, flat, go, lo, rlo, lg, rl.cpu().numpy(), True)
    gm.close()


@pytest.mark.parametrize("s,sampled", [(GPT2_124M_B16, (0, 9, 15)), (GPT2_350M_B16, (5,)),
                                       (GPT2_124M_B64, (63,))],
                         ids=["124m_b16", "350m_b16", "124m_b64"])
def test_step_as_benchmarked(torch, s, sampled):
    """GPT-2 124M and 350M at B=16, T=1024, and the 124M micro-batch of 64
    sequences of the accumulation workload: the launch configurations of the
    benchmark (16384 or 65536 rows: 8 or 32 LM-head chunks of 2048 rows, 1536
    or 6144 CTAs per attention kernel, the GEMM tilings and split counts).  Forward: nothing couples the
    sequences of a batch, so the row losses of sampled sequences must match the
    oracle run on each of those sequences alone.  Backward: the mean loss is
    linear in the sequences' losses, so the gradient must equal the mean of
    the B single-sequence gradients, accumulated here at B=1 (the path that
    test_step_t1024_zipf checks against the oracle) with grad_scale = 1/B."""
    om, named, stream, x, y = inputs(s, seed=0, stream_seed=3, uniform=False)
    tol = TOL[True]
    gm = gpu_model(s, True)
    gm.set_params(named)
    rl = torch.empty(s.B * s.T, dtype=torch.float32, device="cuda")
    gm.zero_grad()
    lg = gm.forward_loss(torch.from_numpy(x).cuda(), torch.from_numpy(y).cuda(), row_loss=rl)
    gm.backward()
    gm.synchronize()
    rows = rl.cpu().numpy().reshape(s.B, s.T)
    assert abs(lg - rows.mean()) <= 1e-4
    flat = om.pack(named)
    for b in sampled:
        lo_b, rlo_b, _, _ = om.fwd_bwd(flat, x[b:b + 1], y[b:b + 1], grads=False, row_loss=True)
        assert abs(rows[b].mean() - lo_b) <= tol["loss"], (b, rows[b].mean(), lo_b)
        assert np.max(np.abs(rows[b] - rlo_b)) <= 10 * tol["loss"], b
    g16 = {n: gm.get_tensor(n, which=1) for n, _ in om.shapes()}
    gm.close()
    one = Shape(s.n_layer, s.n_embd, s.n_head, s.vocab_size, s.padded_vocab, s.max_T, 1, s.T)
    g1 = gpu_model(one, True)
    g1.set_params(named)
    g1.zero_grad()
    for b in range(s.B):
        g1.forward_loss(torch.from_numpy(x[b:b + 1]).cuda(), torch.from_numpy(y[b:b + 1]).cuda(),
                        loss=False)
        g1.backward(1.0 / s.B)
    g1.synchronize()
    for name, _ in om.shapes():
        r = rel_l2(g16[name], g1.get_tensor(name, which=1))
        assert r <= tol["grad"], (name, r)
    g1.close()


@pytest.mark.parametrize("scale", [1.0, 6.0], ids=["qkv_x1", "qkv_x6"])
@pytest.mark.parametrize("bf16", [True, False], ids=["bf16", "fp32"])
def test_attention_t1024_h12(g, torch, scale, bf16):
    """Causal attention forward and backward at B=2, T=1024, C=768, H=12.
    With q, k, v ~ N(0, 36) the scores have a standard deviation near 36, so
    the row maximum rises by far more than the 2^8 factor after which the
    kernel rescales its output accumulator, many times along each row."""
    B, T, C, H = 2, 1024, 768, 12
    key = synth.derive_key(11, int(scale))
    qkv = (synth.normal(key, B * T * 3 * C) * scale).reshape(B, T, 3 * C).astype(np.float32)
    dout = synth.normal(synth.derive_key(12, int(scale)), B * T * C).reshape(B, T, C)
    dt = torch.bfloat16 if bf16 else torch.float32
    q = torch.from_numpy(qkv).cuda().to(dt)
    d = torch.from_numpy(dout.astype(np.float32)).cuda().to(dt)
    qr = q.float().cpu().numpy().astype(np.float64)
    out, lse = g.attention_fwd(q, H)
    oo = oracle.attention(qr, H)
    tol = 3e-2 if bf16 else 1e-4
    assert rel_l2(out.float().cpu().numpy(), oo) <= tol
    dq = g.attention_bwd(d, q, out, lse, H)
    do = oracle.attention_bwd(d.float().cpu().numpy().astype(np.float64), qr, H)
    assert rel_l2(dq.float().cpu().numpy(), do) <= tol
    # per head-block of the gradient (dq, dk, dv separately), not only overall
    for part in range(3):
        sl = slice(part * C, (part + 1) * C)
        assert rel_l2(dq.float().cpu().numpy()[..., sl], do[..., sl]) <= tol, part
    assert g.device_error() == 0


def sampled_rows(M, n=64, key=21):
    rows = synth.randint(synth.derive_key(key, M), n, M)
    return np.unique(np.concatenate([rows, [0, 1, 255, 256, M - 1]]))


# (epilogue, N, K) of the 124M layer: QKV + bias, fc + bias + GELU, attention
# projection + residual, fc projection + residual, GELU backward of the fc input
# gradient.
FULL_LINEAR = [("bias", 2304, 768), ("bias_gelu", 3072, 768), ("residual", 768, 768),
               ("residual", 768, 3072), ("gelu_bwd", 3072, 768)]


@pytest.mark.parametrize("epi,N,K", FULL_LINEAR,
                         ids=[f"{e}_{n}x{k}" for e, n, k in FULL_LINEAR])
def test_linear_epilogues_m16384(g, torch, epi, N, K):
    """The fused linear layer at M=16384 (64 row tiles of 256; 3-12 column
    tiles): sampled rows against the oracle's epilogue on the float64
    contraction of the same bf16 operands."""
    M = 16384
    rng = np.random.default_rng(N + K)
    w_kn = epi == "gelu_bwd"
    x = torch.from_numpy(rng.standard_normal((M, K), dtype=np.float32)).cuda().bfloat16()
    w = torch.from_numpy((rng.standard_normal((K, N) if w_kn else (N, K), dtype=np.float32)
                          / np.sqrt(K)).astype(np.float32)).cuda().bfloat16()
    bias = torch.from_numpy(rng.standard_normal(N, dtype=np.float32)).cuda()
    rows = sampled_rows(M)
    xr = x[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    wr = w.float().cpu().numpy().astype(np.float64)
    y = xr @ (wr if w_kn else wr.T)
    b = bias.cpu().numpy().astype(np.float64)
    tol = 1e-2
    if epi == "bias":
        out = g.linear(g.LINEAR_BIAS, x, w, bias=bias)
        ref = y + b
    elif epi == "bias_gelu":
        out, pre = g.linear(g.LINEAR_BIAS_GELU, x, w, bias=bias)
        pre_r = pre.float().cpu().numpy()[rows].astype(np.float64)
        assert rel_l2(pre_r, y + b) <= tol
        ref = oracle.gelu(pre_r)
    elif epi == "residual":
        res = torch.from_numpy(rng.standard_normal((M, N), dtype=np.float32)).cuda()
        out = g.linear(g.LINEAR_RESIDUAL, x, w, bias=bias, inp=res)
        ref = res.cpu().numpy()[rows] + y + b
    else:
        u = torch.from_numpy(rng.standard_normal((M, N), dtype=np.float32)).cuda().bfloat16()
        out = g.linear(g.LINEAR_GELU_BWD, x, w, inp=u, w_kn=True)
        ref = oracle.gelu_bwd(y, u.float().cpu().numpy()[rows].astype(np.float64))
    got = out.float().cpu().numpy()[rows]
    assert rel_l2(got, ref) <= tol
    # element-wise as well: every sampled element within a few bf16 steps of
    # the reference (the contraction is exact up to fp32 accumulation)
    scale = np.abs(ref).max()
    assert np.max(np.abs(got - ref)) <= 2e-2 * scale
    assert g.device_error() == 0


# dW = dY^T X of the 124M layers at B*T = 16384 rows: (out features, in features)
DW_SHAPES = [(2304, 768), (768, 768), (3072, 768), (768, 3072)]


@pytest.mark.parametrize("M,N", DW_SHAPES, ids=[f"{m}x{n}" for m, n in DW_SHAPES])
def test_weight_gradient_k16384(g, torch, M, N):
    """dW (+)= dY^T X with K = 16384 rows: both operands MN-major (the
    activations as stored), bf16 in, fp32 accumulated into existing values;
    the output has at most 36 tiles of 256 x 256, so K is split across CTA
    pairs and the partial sums are added in a fixed order."""
    K = 16384
    rng = np.random.default_rng(M * 7 + N)
    dy = torch.from_numpy(rng.standard_normal((K, M), dtype=np.float32)).cuda().bfloat16()
    xa = torch.from_numpy(rng.standard_normal((K, N), dtype=np.float32)).cuda().bfloat16()
    prev = torch.from_numpy(rng.standard_normal((M, N), dtype=np.float32)).cuda()
    out = g.matmul(dy, xa, a_kmajor=False, b_kmajor=False, M=M, N=N, K=K, out=prev.clone(),
                   accumulate=True)
    ref = prev.cpu().numpy().astype(np.float64) + (
        dy.float().cpu().numpy().astype(np.float64).T @ xa.float().cpu().numpy().astype(np.float64))
    assert rel_l2(out.cpu().numpy(), ref) <= 1e-5
    # deterministic: the same call gives the same bits
    out2 = g.matmul(dy, xa, a_kmajor=False, b_kmajor=False, M=M, N=N, K=K, out=prev.clone(),
                    accumulate=True)
    assert torch.equal(out, out2)
    assert g.device_error() == 0
