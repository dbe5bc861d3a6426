"""Op-level entry points vs the oracle's functions: LayerNorm, attention, the
tied LM head + cross-entropy (including the full 8192 x 768 x 50304 workload
on sampled rows), and the dense contraction in every operand layout."""
import numpy as np
import pytest

import oracle
import synth
from tests.parity_util import rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    assert torch.cuda.is_available()
    import decoder_only_lm_b200 as g
    return g


def bf16_round(a):
    import torch
    return torch.from_numpy(np.asarray(a, np.float32)).bfloat16().float().numpy().astype(np.float64)


@pytest.mark.parametrize("M,C", [(1, 64), (301, 768), (64, 1024), (20011, 768)])
@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16"])
def test_layernorm(g, M, C, bf16):
    import torch
    rng = np.random.default_rng(M + C)
    x = (rng.normal(size=(M, C)) * 3 + 1).astype(np.float32)
    gam = rng.normal(size=C).astype(np.float32)
    bet = rng.normal(size=C).astype(np.float32)
    dt = torch.bfloat16 if bf16 else torch.float32
    y, mean, rstd = g.layernorm_fwd(torch.from_numpy(x).cuda(), torch.from_numpy(gam).cuda(),
                                    torch.from_numpy(bet).cuda(), out_dtype=dt)
    yo, mo, ro = oracle.layernorm(x.astype(np.float64), gam, bet)
    tol = 8e-3 if bf16 else 1e-5
    assert np.max(np.abs(y.float().cpu().numpy() - yo)) <= tol * max(1, np.abs(yo).max())
    np.testing.assert_allclose(mean.cpu().numpy(), mo, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(rstd.cpu().numpy(), ro, rtol=1e-4)
    dy = rng.normal(size=(M, C)).astype(np.float32)
    dyt = torch.from_numpy(dy).cuda().to(dt)
    dyr = dyt.float().cpu().numpy().astype(np.float64)
    dx, dgam, dbet = g.layernorm_bwd(dyt, torch.from_numpy(x).cuda(), mean, rstd,
                                     torch.from_numpy(gam).cuda())
    dxo, dgo, dbo = oracle.layernorm_bwd(dyr, x.astype(np.float64), mo, ro, gam)
    assert rel_l2(dx.cpu().numpy(), dxo) <= 1e-4
    assert rel_l2(dgam.cpu().numpy(), dgo) <= 1e-4
    assert rel_l2(dbet.cpu().numpy(), dbo) <= 1e-4


def test_layernorm_unaligned_view(g):
    """Rows that do not start on a 16-byte boundary (a view 4 bytes into its
    buffer) take the element-wise kernels and give the same values."""
    import torch
    rng = np.random.default_rng(5)
    M, C = 97, 768
    x = (rng.normal(size=(M, C)) * 2).astype(np.float32)
    gam = rng.normal(size=C).astype(np.float32)
    bet = rng.normal(size=C).astype(np.float32)
    dy = rng.normal(size=(M, C)).astype(np.float32)
    buf = torch.zeros(M * C + 1, device="cuda")
    xv = buf[1:].view(M, C)
    xv.copy_(torch.from_numpy(x))
    assert xv.data_ptr() % 16 != 0
    gt, bt = torch.from_numpy(gam).cuda(), torch.from_numpy(bet).cuda()
    y0, m0, r0 = g.layernorm_fwd(torch.from_numpy(x).cuda(), gt, bt)
    y1, m1, r1 = g.layernorm_fwd(xv, gt, bt)
    yo, mo, ro = oracle.layernorm(x.astype(np.float64), gam, bet)
    for y in (y0, y1):
        assert np.max(np.abs(y.cpu().numpy() - yo)) <= 1e-5 * max(1, np.abs(yo).max())
    dyt = torch.from_numpy(dy).cuda()
    dx0, dg0, db0 = g.layernorm_bwd(dyt, torch.from_numpy(x).cuda(), m0, r0, gt)
    dx1, dg1, db1 = g.layernorm_bwd(dyt, xv, m1, r1, gt)
    dxo, dgo, dbo = oracle.layernorm_bwd(dy.astype(np.float64), x.astype(np.float64), mo, ro, gam)
    for dx, dgm, dbt in ((dx0, dg0, db0), (dx1, dg1, db1)):
        assert rel_l2(dx.cpu().numpy(), dxo) <= 1e-4
        assert rel_l2(dgm.cpu().numpy(), dgo) <= 1e-4
        assert rel_l2(dbt.cpu().numpy(), dbo) <= 1e-4


# head size 64 (bf16: the tcgen05 kernels) at T = 130 and 320 ends in a query
# block whose second 64-query half lies wholly past T: the kept score
# gradients there are never written and must not reach any stored row;
# T = 2048 runs 16 key blocks per (batch, head), 136 score-gradient tiles;
# T = 1: one key, the diagonal tile only
@pytest.mark.parametrize("B,T,C,H", [(2, 37, 64, 4), (1, 200, 128, 2), (2, 64, 96, 3),
                                     (1, 130, 128, 2), (2, 320, 128, 2), (1, 2048, 128, 2),
                                     (3, 1, 128, 2)])
@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16"])
def test_attention(g, B, T, C, H, bf16):
    import torch
    rng = np.random.default_rng(T)
    qkv = rng.normal(size=(B, T, 3 * C)).astype(np.float32)
    dt = torch.bfloat16 if bf16 else torch.float32
    q = torch.from_numpy(qkv).cuda().to(dt)
    qr = q.float().cpu().numpy().astype(np.float64)
    out, lse = g.attention_fwd(q, H)
    oo = oracle.attention(qr, H)
    tol = 3e-2 if bf16 else 1e-4
    assert rel_l2(out.float().cpu().numpy(), oo) <= tol
    dout = torch.from_numpy(rng.normal(size=(B, T, C)).astype(np.float32)).cuda().to(dt)
    dq = g.attention_bwd(dout, q, out, lse, H)
    do = oracle.attention_bwd(dout.float().cpu().numpy().astype(np.float64), qr, H)
    assert rel_l2(dq.float().cpu().numpy(), do) <= tol


def test_attention_items_across_rounds(g):
    """bf16, B=32, T=1024, C=256, H=4: 1024 (query block, head, batch) items,
    more than the forward kernel's persistent CTAs (two per SM) take at once,
    so every CTA runs several items in turn, on alternating Q and output
    buffers with its barrier phases carried from item to item.  Three batch
    elements, whose items fall in different rounds, against the oracle; the
    backward (which reads the forward's log-sum-exp) as well."""
    import torch
    B, T, C, H = 32, 1024, 256, 4
    rng = np.random.default_rng(1024)
    q = torch.from_numpy(rng.normal(size=(B, T, 3 * C)).astype(np.float32)).cuda().bfloat16()
    dout = torch.from_numpy(rng.normal(size=(B, T, C)).astype(np.float32)).cuda().bfloat16()
    out, lse = g.attention_fwd(q, H)
    dq = g.attention_bwd(dout, q, out, lse, H)
    qr = q.float().cpu().numpy().astype(np.float64)
    dr = dout.float().cpu().numpy().astype(np.float64)
    for b in (0, 13, 31):
        qb = np.ascontiguousarray(qr[b:b + 1])
        assert rel_l2(out[b:b + 1].float().cpu().numpy(), oracle.attention(qb, H)) <= 3e-2, b
        do = oracle.attention_bwd(np.ascontiguousarray(dr[b:b + 1]), qb, H)
        assert rel_l2(dq[b:b + 1].float().cpu().numpy(), do) <= 3e-2, b
    assert g.device_error() == 0


@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16"])
def test_lmhead_ce_midsize(g, bf16):
    import torch
    M, C, Vp, V = 600, 128, 2064, 2050
    rng = np.random.default_rng(2)
    h = rng.normal(size=(M, C)).astype(np.float32)
    W = (rng.normal(size=(Vp, C)) * 0.02).astype(np.float32)
    y = rng.integers(0, V, M).astype(np.int32)
    dt = torch.bfloat16 if bf16 else torch.float32
    ht, Wt = torch.from_numpy(h).cuda().to(dt), torch.from_numpy(W).cuda().to(dt)
    loss, lse, dh, dW = g.lmhead_ce(ht, Wt, torch.from_numpy(y).cuda(), V, grad_scale=1.0)
    hr, Wr = ht.float().cpu().numpy().astype(np.float64), Wt.float().cpu().numpy().astype(np.float64)
    lo, rlo, dho, dWo = oracle.lmhead_ce(hr, Wr, y, V)
    tol = 2e-2 if bf16 else 1e-4
    assert abs(loss.item() - lo) <= tol
    assert rel_l2(dh.float().cpu().numpy(), dho) <= (3e-2 if bf16 else 1e-3)
    assert rel_l2(dW.cpu().numpy(), dWo) <= (3e-2 if bf16 else 1e-3)


def test_lmhead_ce_full_size_sampled_rows(g):
    """The 8192 x 768 x 50304 bf16 workload: per-row results on sampled rows
    against the oracle, and dW by linearity over two halves of the rows."""
    import torch
    M, C, Vp, V = 8192, 768, 50304, 50257
    h = synth.normal(synth.derive_key(2, 1), M * C, 1.0).reshape(M, C).astype(np.float32)
    W = synth.normal(synth.derive_key(2, 2), Vp * C, 0.02).reshape(Vp, C).astype(np.float32)
    y = synth.randint(synth.derive_key(2, 3), M, V).astype(np.int32)
    ht = torch.from_numpy(h).cuda().bfloat16()
    Wt = torch.from_numpy(W).cuda().bfloat16()
    yt = torch.from_numpy(y).cuda()
    loss, lse, dh, dW = g.lmhead_ce(ht, Wt, yt, V)
    rows = np.sort(synth.randint(synth.derive_key(2, 4), 48, M))
    rows = np.unique(np.concatenate([rows, [0, M - 1]]))
    hr = ht.float().cpu().numpy().astype(np.float64)
    Wr = Wt.float().cpu().numpy().astype(np.float64)
    _, rlo, dho, _ = oracle.lmhead_ce(hr[rows], Wr, y[rows], V, grad_scale=len(rows) / M)
    lse_g = lse.cpu().numpy()[rows]
    lse_o = rlo + np.einsum("mc,mc->m", hr[rows], Wr[y[rows]])  # loss + z_y = lse
    assert np.max(np.abs(lse_g - lse_o)) <= 2e-2
    assert rel_l2(dh.float().cpu().numpy()[rows], dho) <= 3e-2
    # linearity: dW of all rows = dW(first half) + dW(second half), each scaled by its share
    _, _, _, dW1 = g.lmhead_ce(ht[: M // 2], Wt, yt[: M // 2], V, grad_scale=0.5)
    _, _, _, dW2 = g.lmhead_ce(ht[M // 2:], Wt, yt[M // 2:], V, grad_scale=0.5)
    assert rel_l2((dW1 + dW2).cpu().numpy(), dW.cpu().numpy()) <= 1e-3
    # mean loss of the full batch near ln(V) at this init (logits ~ N(0, 0.02^2 * 768))
    assert abs(loss.item() - np.log(Vp)) < 0.5


@pytest.mark.parametrize("ak,bk", [(1, 1), (1, 0), (0, 1), (0, 0)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 200, 136), (1024, 768, 768), (16, 520, 256),
                                   (3, 50304, 768)])
@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16"])
def test_matmul_layouts(g, ak, bk, M, N, K, bf16):
    import torch
    rng = np.random.default_rng(M * N + K + 3 * ak + bk)
    A = rng.normal(size=(M, K)).astype(np.float32)
    B = rng.normal(size=(N, K)).astype(np.float32)
    dt = torch.bfloat16 if bf16 else torch.float32
    At = torch.from_numpy(A if ak else np.ascontiguousarray(A.T)).cuda().to(dt)
    Bt = torch.from_numpy(B if bk else np.ascontiguousarray(B.T)).cuda().to(dt)
    out = g.matmul(At, Bt, a_kmajor=bool(ak), b_kmajor=bool(bk), M=M, N=N, K=K)
    Ar = At.float().cpu().numpy().astype(np.float64)
    Br = Bt.float().cpu().numpy().astype(np.float64)
    ref = (Ar if ak else Ar.T) @ (Br if bk else Br.T).T
    assert rel_l2(out.cpu().numpy(), ref) <= 1e-5
    # accumulate mode adds alpha * A B^T to what is there
    out2 = g.matmul(At, Bt, a_kmajor=bool(ak), b_kmajor=bool(bk), M=M, N=N, K=K, alpha=0.5,
                    out=out.clone(), accumulate=True)
    assert rel_l2(out2.cpu().numpy(), 1.5 * ref) <= 1e-5


@pytest.mark.parametrize("epi", ["bias", "bias_gelu", "residual", "gelu_bwd"])
@pytest.mark.parametrize("M,N,K", [(300, 520, 136), (1, 64, 64), (2050, 768, 3072), (4, 2304, 768),
                                   (3, 384, 3072), (16, 384, 3072)])
@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16"])
def test_linear_epilogues(g, epi, M, N, K, bf16):
    """The fused linear layer against the oracle: the contraction in fp64 from
    the same (rounded) operands, then the epilogue of the block it fuses."""
    import torch
    rng = np.random.default_rng(M + 7 * N + K)
    dt = torch.bfloat16 if bf16 else torch.float32
    w_kn = epi == "gelu_bwd"  # the backward contraction reads W as [K, N]
    x = torch.from_numpy(rng.normal(size=(M, K)).astype(np.float32)).cuda().to(dt)
    w = torch.from_numpy((rng.normal(size=(K, N) if w_kn else (N, K)) / np.sqrt(K))
                         .astype(np.float32)).cuda().to(dt)
    bias = torch.from_numpy(rng.normal(size=N).astype(np.float32)).cuda()
    xr = x.float().cpu().numpy().astype(np.float64)
    wr = w.float().cpu().numpy().astype(np.float64)
    y = xr @ (wr if w_kn else wr.T)
    tol = 1e-2 if bf16 else 1e-5
    if epi == "bias":
        out = g.linear(g.LINEAR_BIAS, x, w, bias=bias)
        ref = y + bias.cpu().numpy()
    elif epi == "bias_gelu":
        out, pre = g.linear(g.LINEAR_BIAS_GELU, x, w, bias=bias)
        pre_ref = y + bias.cpu().numpy()
        assert rel_l2(pre.float().cpu().numpy(), pre_ref) <= tol
        # the activation is taken of the stored (rounded) pre-activation
        ref = oracle.gelu(pre.float().cpu().numpy().astype(np.float64))
    elif epi == "residual":
        res = torch.from_numpy(rng.normal(size=(M, N)).astype(np.float32)).cuda()
        out = g.linear(g.LINEAR_RESIDUAL, x, w, bias=bias, inp=res)
        assert out.dtype == torch.float32
        ref = res.cpu().numpy() + y + bias.cpu().numpy()
    else:
        u = torch.from_numpy(rng.normal(size=(M, N)).astype(np.float32)).cuda().to(dt)
        out = g.linear(g.LINEAR_GELU_BWD, x, w, inp=u, w_kn=True)
        ref = oracle.gelu_bwd(y, u.float().cpu().numpy().astype(np.float64))
    assert rel_l2(out.float().cpu().numpy(), ref) <= tol
    assert g.device_error() == 0
