"""Pins of the CPU oracle to things other than itself.

Each test fixes a part of the oracle against what the pages print (worked
values under tests/golden/), closed forms, invariants, float64 PyTorch library
routines (an independent implementation) or central finite differences, so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth
from tests import torch_ref

TINY = dict(n_layer=2, n_embd=64, n_head=4, vocab_size=512, padded_vocab=512, max_T=64)


def tiny_model(**kw):
    cfg = dict(TINY)
    cfg.update(kw)
    return oracle.Model(**cfg)


def tiny_inputs(m, seed=0, B=4, T=32, stream_seed=1):
    named = synth.init_params(seed, m.shapes())
    s = synth.uniform_stream(stream_seed, B * T + 1, m.cfg.vocab_size)
    x, y = oracle.batch_from_stream(s, 0, B, T)
    return named, x, y


# --------------------------------------------------------------------------- slicing

def test_slicing_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "slicing_ch28.json")))["single"]
    x, y = oracle.batch_from_stream(np.array(g["stream"], np.uint16), 0, g["B"], g["T"])
    assert x.tolist() == g["x"] and y.tolist() == g["y"]


def test_slicing_rank_offsets(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "slicing_ch28.json")))["ranks"]
    B, T, R = g["B"], g["T"], g["R"]
    s = np.arange(64, dtype=np.uint16)
    for r in range(R):
        x, _ = oracle.batch_from_stream(s, B * T * r, B, T)
        assert x.reshape(-1).tolist() == g["first_inputs"][str(r)]
        x2, _ = oracle.batch_from_stream(s, B * T * r + B * T * R, B, T)
        assert int(x2[0, 0]) == g["next_start"][str(r)]


def test_slicing_rejects_short_stream():
    with pytest.raises(oracle.OracleError):
        oracle.batch_from_stream(np.arange(6, dtype=np.uint16), 0, 2, 3)


# --------------------------------------------------------------------------- cross-entropy

def test_ce_printed_values(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "ce_cs336.json")))
    tol = g["printed_tolerance"]
    # p = 0.1: ten equal logits.  p = 0.8: two logits [ln 4, 0].
    for dt in (np.float32, np.float64):
        l1, _ = oracle.cross_entropy(np.zeros((1, 10), dt), [3])
        l2, _ = oracle.cross_entropy(np.array([[math.log(4.0), 0.0]], dt), [0])
        assert abs(l1 - g["ce"][0]["loss"]) <= tol and abs(l2 - g["ce"][1]["loss"]) <= tol
        assert abs(l1 + math.log(0.1)) < 1e-6 and abs(l2 + math.log(0.8)) < 1e-6


def test_perplexity_printed_value(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "ce_cs336.json")))
    # logits [a, 0] with target 0 give p = e^-2, so the mean loss is 2.
    a = -2.0 - math.log1p(-math.exp(-2.0))
    loss, _ = oracle.cross_entropy(np.array([[a, 0.0]] * 3), [0, 0, 0])
    assert abs(loss - 2.0) < 1e-12
    assert abs(math.exp(loss) - g["ppl"][0]["ppl"]) <= g["printed_tolerance"]


def test_ce_matches_library_and_shift_invariance():
    rng = np.random.default_rng(0)
    z = rng.normal(size=(37, 211)) * 3
    y = rng.integers(0, 211, 37)
    loss, rl = oracle.cross_entropy(z, y)
    ref = F.cross_entropy(torch.tensor(z), torch.tensor(y), reduction="none").numpy()
    np.testing.assert_allclose(rl, ref, rtol=0, atol=1e-12)
    # subtracting the row maximum is exact: a huge common shift changes nothing
    _, rl2 = oracle.cross_entropy(z + 1e4, y)
    np.testing.assert_allclose(rl2, ref, atol=1e-9)


# --------------------------------------------------------------------------- parameter counts

def test_param_counts(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "param_counts.json")))
    c = g["gpt2_124m"]
    m = oracle.Model(c["n_layer"], c["n_embd"], c["n_head"], c["vocab_size"], c["vocab_size"], c["max_T"])
    assert m.n_params == 124_439_808
    assert round(m.n_params / 1e6) == c["printed_millions"]
    wte = dict((n, s) for n, s, _ in m.tensors)["wte"]
    assert wte[0] * wte[1] == 38_597_376 and round(wte[0] * wte[1] / 1e6, -1) == c["wte_printed_millions"]
    t = oracle.Model(2, 16, 2, g["tiny"]["vocab_size"], g["tiny"]["vocab_size"], 12)
    assert t.n_params == g["tiny"]["printed"]
    # padded vocabulary (50,304 rows) used by the benchmark workloads
    assert oracle.Model(12, 768, 12, 50257, 50304, 1024).n_params == 124_475_904


# --------------------------------------------------------------------------- single ops vs library

@pytest.mark.parametrize("M,C", [(7, 64), (33, 768)])
def test_layernorm_matches_library(M, C):
    rng = np.random.default_rng(1)
    x = rng.normal(size=(M, C)) * 2 + 0.5
    g = rng.normal(size=C)
    b = rng.normal(size=C)
    y, mean, rstd = oracle.layernorm(x, g, b, 1e-5)
    ref = F.layer_norm(torch.tensor(x), (C,), torch.tensor(g), torch.tensor(b), 1e-5).numpy()
    np.testing.assert_allclose(y, ref, atol=1e-12)
    # backward against autograd
    xt = torch.tensor(x, requires_grad=True)
    gt = torch.tensor(g, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    dy = rng.normal(size=(M, C))
    F.layer_norm(xt, (C,), gt, bt, 1e-5).backward(torch.tensor(dy))
    dx, dg, db = oracle.layernorm_bwd(dy, x, mean, rstd, g)
    np.testing.assert_allclose(dx, xt.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dg, gt.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(db, bt.grad.numpy(), atol=1e-11)


def test_gelu_matches_library():
    u = np.linspace(-8, 8, 1001)
    g = oracle.gelu(u)
    ut = torch.tensor(u, requires_grad=True)
    ref = F.gelu(ut, approximate="tanh")
    np.testing.assert_allclose(g, ref.detach().numpy(), atol=1e-14)
    dg = np.cos(u)
    ref.backward(torch.tensor(dg))
    np.testing.assert_allclose(oracle.gelu_bwd(dg, u), ut.grad.numpy(), atol=1e-13)
    # the tanh form differs from the exact erf GELU (a wrong constant would not)
    assert np.max(np.abs(g - F.gelu(torch.tensor(u)).numpy())) > 1e-5


@pytest.mark.parametrize("B,T,C,H", [(2, 17, 32, 4), (1, 64, 64, 2)])
def test_attention_matches_library(B, T, C, H):
    rng = np.random.default_rng(2)
    qkv = rng.normal(size=(B, T, 3 * C))
    out = oracle.attention(qkv, H)
    t = torch.tensor(qkv, requires_grad=True)
    q, k, v = t.split(C, dim=2)
    sh = lambda z: z.view(B, T, H, C // H).transpose(1, 2)
    ref = F.scaled_dot_product_attention(sh(q), sh(k), sh(v), is_causal=True)
    ref = ref.transpose(1, 2).reshape(B, T, C)
    np.testing.assert_allclose(out, ref.detach().numpy(), atol=1e-12)
    dout = rng.normal(size=(B, T, C))
    ref.backward(torch.tensor(dout))
    np.testing.assert_allclose(oracle.attention_bwd(dout, qkv, H), t.grad.numpy(), atol=1e-11)


def test_lmhead_ce_matches_library():
    rng = np.random.default_rng(3)
    M, C, Vp, V = 70, 24, 131, 120
    h = rng.normal(size=(M, C))
    W = rng.normal(size=(Vp, C)) * 0.3
    y = rng.integers(0, V, M)
    loss, rl, dh, dW = oracle.lmhead_ce(h, W, y, V, grad_scale=0.5)
    ht = torch.tensor(h, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    ref = F.cross_entropy(F.linear(ht, Wt), torch.tensor(y))
    (0.5 * ref).backward()
    assert abs(loss - ref.item()) < 1e-12
    np.testing.assert_allclose(dh, ht.grad.numpy(), atol=1e-13)
    np.testing.assert_allclose(dW, Wt.grad.numpy(), atol=1e-13)
    # targets beyond the real vocabulary are refused
    with pytest.raises(oracle.OracleError):
        oracle.lmhead_ce(h, W, np.full(M, V), V)


# --------------------------------------------------------------------------- full model

@pytest.mark.parametrize("B,T", [(4, 32), (3, 7)])
def test_full_model_matches_library_autograd(B, T):
    m = tiny_model()
    named, x, y = tiny_inputs(m, B=B, T=T)
    # non-trivial LayerNorm parameters and biases so that every term is exercised
    rng = np.random.default_rng(4)
    for k in named:
        if named[k].ndim == 1:
            named[k] = named[k] + rng.normal(size=named[k].shape).astype(np.float32) * 0.1
    flat = m.pack(named)
    loss, rl, g, logits = m.fwd_bwd(flat, x, y, row_loss=True, logits=True)
    P = torch_ref.to_torch(named)
    ref, ref_logits = torch_ref.forward(P, x, y, m.cfg.n_layer, m.cfg.n_head)
    ref.backward()
    assert abs(loss - ref.item()) < 1e-12
    np.testing.assert_allclose(logits, ref_logits.detach().numpy().reshape(B * T, -1), atol=1e-12)
    G = m.unpack(g)
    for n, _ in m.shapes():
        np.testing.assert_allclose(G[n], P[n].grad.numpy(), atol=1e-12, rtol=1e-9, err_msg=n)


def test_tied_gradient_is_sum_of_both_uses():
    m = tiny_model()
    named, x, y = tiny_inputs(m)
    _, _, g, _ = m.fwd_bwd(m.pack(named), x, y)
    P = torch_ref.to_torch(named)
    head = torch.tensor(np.asarray(named["wte"], np.float64), requires_grad=True)
    loss, _ = torch_ref.forward(P, x, y, m.cfg.n_layer, m.cfg.n_head, untied_head=head)
    loss.backward()
    emb_part, head_part = P["wte"].grad.numpy(), head.grad.numpy()
    assert np.abs(emb_part).max() > 0 and np.abs(head_part).max() > 0
    np.testing.assert_allclose(m.unpack(g)["wte"], emb_part + head_part, atol=1e-13)


def test_finite_differences():
    m = tiny_model(n_layer=1, n_embd=32, n_head=2, vocab_size=64, padded_vocab=72, max_T=16)
    B, T = 2, 8
    named, x, y = tiny_inputs(m, B=B, T=T)
    rng = np.random.default_rng(5)
    for k in named:  # move away from the symmetric init so every path carries gradient
        named[k] = named[k] + rng.normal(size=named[k].shape) * 0.05
    flat = m.pack(named)
    _, _, g, _ = m.fwd_bwd(flat, x, y)
    h = 1e-5
    for name, shape, off in m.tensors:
        n = int(np.prod(shape))
        idx = rng.choice(n, size=min(n, 24), replace=False) + off
        gmax = np.abs(g[off:off + n]).max()
        for i in idx:
            p = flat.copy()
            p[i] += h
            lp = m.fwd_bwd(p, x, y, grads=False)[0]
            p[i] -= 2 * h
            lm = m.fwd_bwd(p, x, y, grads=False)[0]
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[i]) <= 1e-6 * max(abs(g[i]), 1e-3 * gmax) + 1e-10, (name, i, fd, g[i])


def test_uniform_logits_give_log_vocab():
    # wte = 0 makes every logit 0: the loss is ln(Vp) exactly, at any input.
    for kw in (dict(), dict(padded_vocab=640)):
        m = tiny_model(**kw)
        named, x, y = tiny_inputs(m)
        named["wte"][:] = 0
        loss = m.fwd_bwd(m.pack(named), x, y, grads=False)[0]
        assert abs(loss - math.log(m.cfg.padded_vocab)) < 1e-12


def test_uniform_logits_log_vocab_at_gpt2_width():
    m = oracle.Model(12, 768, 12, 50257, 50304, 1024)
    named = {n: np.zeros(s, np.float32) for n, s in m.shapes()}
    for n, s in m.shapes():
        if n.endswith(".w") and len(s) == 1:
            named[n][:] = 1
    named["wpe"] = synth.normal(7, 1024 * 768, 0.02).reshape(1024, 768).astype(np.float32)
    x = np.array([[50256, 10, 20, 30]], np.int32)
    loss = m.fwd_bwd(m.pack(named, np.float32), x, x, grads=False)[0]
    assert abs(loss - math.log(50304)) < 1e-5  # 10.825840


def test_initial_loss_near_log_vocab():
    m = tiny_model()
    named, x, y = tiny_inputs(m)
    loss = m.fwd_bwd(m.pack(named), x, y, grads=False)[0]
    assert abs(loss - math.log(512)) < 0.1


@pytest.mark.parametrize("dt", [np.float32, np.float64])
def test_causal_invariance(dt):
    m = tiny_model()
    named, x, y = tiny_inputs(m)
    flat = m.pack(named, dt)
    _, rl, _, lg = m.fwd_bwd(flat, x, y, grads=False, row_loss=True, logits=True)
    t0 = 11
    x2, y2 = x.copy(), y.copy()
    rng = np.random.default_rng(6)
    x2[:, t0 + 1:] = rng.integers(0, 512, x2[:, t0 + 1:].shape)
    y2[:, t0 + 1:] = rng.integers(0, 512, y2[:, t0 + 1:].shape)
    _, rl2, _, lg2 = m.fwd_bwd(flat, x2, y2, grads=False, row_loss=True, logits=True)
    B, T = x.shape
    keep = (np.arange(B * T) % T) <= t0
    assert np.array_equal(rl[keep], rl2[keep]) and np.array_equal(lg[keep], lg2[keep])
    assert not np.array_equal(lg[~keep], lg2[~keep])


def test_out_of_range_token_refused():
    m = tiny_model()
    named, x, y = tiny_inputs(m)
    x[1, 3] = 512
    with pytest.raises(oracle.OracleError) as e:
        m.fwd_bwd(m.pack(named), x, y)
    assert e.value.code == 2


@pytest.mark.parametrize("dt,tol", [(np.float64, 1e-12), (np.float32, 2e-6)])
def test_gradient_accumulation_identity(dt, tol):
    m = tiny_model()
    named, x, y = tiny_inputs(m)
    flat = m.pack(named, dt)
    _, _, full, _ = m.fwd_bwd(flat, x, y)
    acc = np.zeros_like(full)
    m.fwd_bwd(flat, x[:2], y[:2], grad_scale=0.5, grads_in=acc)
    m.fwd_bwd(flat, x[2:], y[2:], grad_scale=0.5, grads_in=acc)
    assert np.linalg.norm(acc - full) <= tol * np.linalg.norm(full)


# --------------------------------------------------------------------------- clip + AdamW

def _state(m, seed=0, scale=1.0):
    named, x, y = tiny_inputs(m, seed=seed)
    p = m.pack(named)
    _, _, g, _ = m.fwd_bwd(p, x, y)
    return p, g * scale


def test_adamw_first_step_closed_form():
    m = tiny_model()
    p, g = _state(m, scale=1e-3)  # norm well below 1: no clipping
    lr, b1, b2, eps, wd = 6e-4, 0.9, 0.95, 1e-8, 0.1
    p1, mm, vv = p.copy(), np.zeros_like(p), np.zeros_like(p)
    n = m.clip_adamw(p1, g, mm, vv, 1, lr, b1, b2, eps, wd, 1.0)
    assert abs(n - np.linalg.norm(g)) < 1e-12 * n
    decay = np.zeros_like(p)
    for name, shape, off in m.tensors:
        decay[off:off + int(np.prod(shape))] = 1.0 if len(shape) == 2 else 0.0
    expect = p * (1 - lr * wd * decay) - lr * g / (np.abs(g) + eps / math.sqrt(1 - b2))
    np.testing.assert_allclose(p1, expect, rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(mm, (1 - b1) * g, rtol=1e-15)
    np.testing.assert_allclose(vv, (1 - b2) * g * g, rtol=1e-15)


def test_clip_scale():
    m = tiny_model()
    p, g = _state(m, scale=50.0)
    n_true = np.linalg.norm(g)
    assert n_true > 1
    mm, vv = np.zeros_like(p), np.zeros_like(p)
    n = m.clip_adamw(p.copy(), g, mm, vv, 1, 6e-4, 0.9, 0.95, 1e-8, 0.1, 1.0)
    assert abs(n - n_true) < 1e-12 * n_true
    s = 1.0 / (n_true + 1e-6)
    np.testing.assert_allclose(mm, 0.1 * s * g, rtol=1e-12)
    # the clipped gradient has norm 1 / (1 + 1e-6 / n)
    assert abs(np.linalg.norm(mm / 0.1) - 1 / (1 + 1e-6 / n_true)) < 1e-12
    # below the threshold the scale is exactly 1
    p2, g2 = _state(m, scale=1e-3)
    mm2 = np.zeros_like(p2)
    m.clip_adamw(p2.copy(), g2, mm2, np.zeros_like(p2), 1, 6e-4, 0.9, 0.95, 1e-8, 0.1, 1.0)
    np.testing.assert_array_equal(mm2, (1 - 0.9) * g2)


def test_nonfinite_gradient_leaves_state_untouched():
    m = tiny_model()
    p, g = _state(m)
    g[5] = np.nan
    p0, mm, vv = p.copy(), np.ones_like(p), np.ones_like(p)
    with pytest.raises(oracle.OracleError) as e:
        m.clip_adamw(p, g, mm, vv, 1)
    assert e.value.code == 3
    assert np.array_equal(p, p0) and (mm == 1).all() and (vv == 1).all()


def test_adamw_matches_torch_with_eps_rescaling():
    """Three steps against torch.optim.AdamW.

    The pages fold bias correction into the step size and add eps to the
    uncorrected sqrt(v); torch adds eps to sqrt(v_hat).  The two agree exactly
    when torch is given eps_t = eps / sqrt(1 - b2^t) at step t.
    """
    m = tiny_model()
    lr, b1, b2, eps, wd = 1e-3, 0.9, 0.95, 1e-6, 0.1
    p, _ = _state(m)
    mm, vv = np.zeros_like(p), np.zeros_like(p)
    named = m.unpack(p.copy())
    tp = {k: torch.tensor(v.copy(), requires_grad=True) for k, v in named.items()}
    decay = [tp[n] for n, s in m.shapes() if len(s) == 2]
    nodecay = [tp[n] for n, s in m.shapes() if len(s) != 2]
    opt = torch.optim.AdamW([{"params": decay, "weight_decay": wd},
                             {"params": nodecay, "weight_decay": 0.0}], lr=lr, betas=(b1, b2), eps=eps)
    rng = np.random.default_rng(7)
    for t in (1, 2, 3):
        g = rng.normal(size=p.size) * 1e-3  # norm < 1: no clipping on either side
        m.clip_adamw(p, g, mm, vv, t, lr, b1, b2, eps, wd, 1.0)
        G = m.unpack(g)
        for k in tp:
            tp[k].grad = torch.tensor(G[k].copy())
        for grp in opt.param_groups:
            grp["eps"] = eps / math.sqrt(1 - b2 ** t)
        opt.step()
    P = m.unpack(p)
    for k in tp:
        np.testing.assert_allclose(P[k], tp[k].detach().numpy(), rtol=1e-12, atol=1e-15, err_msg=k)


# --------------------------------------------------------------------------- learning works

def test_overfit_one_batch():
    m = tiny_model()
    named, x, y = tiny_inputs(m)
    p = m.pack(named)
    mm, vv = np.zeros_like(p), np.zeros_like(p)
    first = None
    for t in range(1, 31):
        loss, _, g, _ = m.fwd_bwd(p, x, y)
        first = first if first is not None else loss
        m.clip_adamw(p, g, mm, vv, t, lr=3e-3)
    assert loss < 0.5 * first


def test_tiny_mod17_task_learns():
    """The 7,056-parameter task of chapter 28 section 28.7: predict (t+1) mod 17.

    Only "the loss falls" is pinned: the page prints the start and end losses
    of its own run but not the learning rate, batch or seed (trajectory parity
    unpinned).
    """
    m = oracle.Model(2, 16, 2, 17, 17, 12)
    named = synth.init_params(0, m.shapes())
    p = m.pack(named)
    B, T = 8, 12
    starts = synth.randint(synth.derive_key(11), 100 * B, 17).reshape(100, B)
    mm, vv = np.zeros_like(p), np.zeros_like(p)
    losses = []
    for t in range(100):
        seq = (starts[t][:, None] + np.arange(T + 1)[None]) % 17
        loss, _, g, _ = m.fwd_bwd(p, seq[:, :-1], seq[:, 1:])
        losses.append(loss)
        m.clip_adamw(p, g, mm, vv, t + 1, lr=1e-2, wd=0.0)
    assert losses[0] > 2.5 and losses[-1] < 0.5 * losses[0]


_NORM_CHILD = r"""
import sys, numpy as np
sys.path.insert(0, sys.argv[1])
import oracle, synth
m = oracle.Model(2, 64, 4, 512, 512, 64)
p = m.pack(synth.init_params(0, m.shapes()))
g = synth.normal(synth.derive_key(31), p.size, 1.0).astype(np.float64)
mm, vv = np.zeros_like(p), np.zeros_like(p)
n = m.clip_adamw(p, g, mm, vv, 1)
sys.stdout.write(repr(n) + " " + str(oracle.num_threads()) + " " + p.tobytes().hex()[:0])
np.save(sys.argv[2], p)
"""


def test_clip_adamw_identical_for_any_thread_count(tmp_path):
    """The gradient norm is one sum of squares over every element, taken in a
    fixed order, so that data-parallel ranks (each applying the same averaged
    gradient) end with bit-identical parameters: the same update computed in
    two processes with 1 and 5 OpenMP threads must agree bit for bit."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = []
    for nt in (1, 5):
        f = tmp_path / f"p{nt}.npy"
        env = dict(os.environ, OMP_NUM_THREADS=str(nt))
        r = subprocess.run([sys.executable, "-c", _NORM_CHILD, root, str(f)], env=env,
                           capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stderr
        norm, threads = r.stdout.split()[:2]
        assert int(threads) == nt
        out.append((norm, np.load(f)))
    assert out[0][0] == out[1][0]
    assert np.array_equal(out[0][1], out[1][1])
