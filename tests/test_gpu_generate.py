"""Next-token sampling, last-position logits and generation on the GPU against
the oracle: the same fp32 logits give the same ids; the logits match the
oracle's forward; generation equals its definition step by step."""
import numpy as np
import pytest

import oracle
import synth
from tests.parity_util import rel_l2

pytestmark = pytest.mark.gpu

SETTINGS = [  # temperature, top_k, top_p
    (0.0, 0, 1.0), (1.0, 0, 1.0), (0.8, 0, 0.9), (1.0, 50, 1.0), (1.3, 40, 0.7),
    (0.5, 1, 0.9), (0.7, 0, 0.05), (2.0, 3000, 0.95),
]


@pytest.fixture(scope="module")
def g():
    import torch
    assert torch.cuda.is_available()
    import decoder_only_lm_b200 as g
    return g


@pytest.mark.parametrize("V,pad", [(50257, 47), (1000, 0), (37, 3)])
@pytest.mark.parametrize("setting", SETTINGS)
def test_sample_matches_oracle(g, V, pad, setting):
    import torch
    T, k, p = setting
    rng = np.random.default_rng(V + int(100 * T) + k)
    B = 6
    z = (rng.normal(size=(B, V + pad)) * 3).astype(np.float32)
    z[0, 5] = z[0, 9] = z[0].max() + 2.0  # a tie at the top: the smaller id first
    z[1, : V // 2] = z[1, V // 2]         # many equal logits
    z[:, V:] = 100.0                       # padding columns are never drawn
    u = rng.random(B).astype(np.float32)
    zt = torch.from_numpy(z).cuda()
    got = g.sample(zt, V, T, k, p, torch.from_numpy(u).cuda()).cpu().numpy()
    ref = oracle.sample(z, V, T, k, p, u)
    np.testing.assert_array_equal(got, ref)
    again = g.sample(zt, V, T, k, p, torch.from_numpy(u).cuda()).cpu().numpy()
    np.testing.assert_array_equal(again, got)  # deterministic
    assert g.device_error() == 0


def test_sample_edge_uniforms_and_stride(g):
    """u = 0 and u just below 1 pick the first and the last kept id in id order;
    out_stride writes every other entry."""
    import torch
    rng = np.random.default_rng(7)
    V, B = 500, 4
    z = rng.normal(size=(B, V)).astype(np.float32)
    for u0 in (0.0, np.nextafter(np.float32(1), np.float32(0))):
        u = np.full(B, u0, np.float32)
        got = g.sample(torch.from_numpy(z).cuda(), V, 1.0, 20, 0.8, torch.from_numpy(u).cuda())
        np.testing.assert_array_equal(got.cpu().numpy(), oracle.sample(z, V, 1.0, 20, 0.8, u))
    out = torch.full((B, 2), -1, dtype=torch.int32, device="cuda")
    g.sample(torch.from_numpy(z).cuda(), V, 0.0, 0, 1.0, None, out=out)
    np.testing.assert_array_equal(out[:, 0].cpu().numpy(), np.argmax(z, axis=1))
    assert (out[:, 1].cpu().numpy() == -1).all()


def tiny(g, bf16, max_T=64, max_B=4):
    om = oracle.Model(2, 64, 4, 512, 512, max_T)
    named = synth.init_params(0, om.shapes())
    gm = g.GPT2(2, 64, 4, 512, 512, max_T, bf16=bf16, max_B=max_B, max_Tseq=max_T)
    gm.set_params(named)
    return om, om.pack(named), gm


def oracle_last_logits(om, params, x):
    B, T = x.shape
    _, _, _, lg = om.fwd_bwd(params, x, x, grads=False, logits=True)
    return lg.reshape(B, T, -1)[:, -1, :]


@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16"])
@pytest.mark.parametrize("B,T", [(1, 1), (3, 37), (4, 64)])
def test_logits_last_matches_oracle(g, bf16, B, T):
    om, params, gm = tiny(g, bf16)
    rng = np.random.default_rng(B * 100 + T)
    x = rng.integers(0, 512, size=(B, T)).astype(np.int32)
    got = gm.logits_last(x).cpu().numpy()
    ref = oracle_last_logits(om, params, x)
    assert got.shape == (B, 512)
    assert rel_l2(got, ref) <= (3e-2 if bf16 else 1e-4)
    gm.close()


@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16"])
@pytest.mark.parametrize("setting", [(0.0, 0, 1.0), (0.8, 0, 0.9), (1.0, 20, 1.0)])
def test_generate_is_logits_last_then_sample(g, bf16, setting):
    """Each generated token is the sample of the last-position logits of the
    window before it; the window slides once the context (64) is full."""
    import torch
    T, k, p = setting
    om, params, gm = tiny(g, bf16)
    rng = np.random.default_rng(11)
    B, T0, n = 3, 58, 12  # 58 + 12 > 64: the last steps see a sliding window
    prompt = torch.from_numpy(rng.integers(0, 512, size=(B, T0)).astype(np.int32)).cuda()
    u = torch.from_numpy(rng.random((n, B)).astype(np.float32)).cuda()
    out = gm.generate(prompt, n, T, k, p, None if T == 0 else u)
    assert out.shape == (B, T0 + n)
    np.testing.assert_array_equal(out[:, :T0].cpu().numpy(), prompt.cpu().numpy())
    seq = prompt.clone()
    for s in range(n):
        w = seq[:, -64:]
        lg = gm.logits_last(w)
        nxt = g.sample(lg, 512, T, k, p, u[s])
        seq = torch.cat([seq, nxt[:, None]], dim=1)
    np.testing.assert_array_equal(out.cpu().numpy(), seq.cpu().numpy())
    gm.close()


def test_generate_fp32_matches_oracle_loop(g):
    """fp32 mode: the oracle's own loop (its forward's last logits, its sample)
    gives the same tokens."""
    import torch
    om, params, gm = tiny(g, False)
    rng = np.random.default_rng(12)
    B, T0, n = 2, 20, 10
    prompt = rng.integers(0, 512, size=(B, T0)).astype(np.int32)
    u = rng.random((n, B)).astype(np.float32)
    out = gm.generate(torch.from_numpy(prompt).cuda(), n, 0.9, 0, 0.95,
                      torch.from_numpy(u).cuda()).cpu().numpy()
    seq = prompt.copy()
    for s in range(n):
        lg = oracle_last_logits(om, params, seq[:, -64:]).astype(np.float32)
        nxt = oracle.sample(lg, 512, 0.9, 0, 0.95, u[s])
        seq = np.concatenate([seq, nxt[:, None]], axis=1)
    np.testing.assert_array_equal(out, seq)
    gm.close()


@pytest.mark.parametrize("setting", [(0.0, 0, 1.0), (0.8, 0, 0.9), (1.0, 20, 1.0)])
def test_cached_generation_fp32_equals_recompute_and_oracle(g, setting):
    """fp32 mode: the KV-cache path gives the tokens of the recompute path and
    of the oracle's own loop (prompt + new tokens within the context)."""
    import torch
    T, k, p = setting
    om, params, gm = tiny(g, False)
    rng = np.random.default_rng(21)
    B, T0, n = 3, 17, 30
    prompt = rng.integers(0, 512, size=(B, T0)).astype(np.int32)
    u = rng.random((n, B)).astype(np.float32)
    ut = None if T == 0 else torch.from_numpy(u).cuda()
    pt = torch.from_numpy(prompt).cuda()
    cached = gm.generate(pt, n, T, k, p, ut, cached=True).cpu().numpy()
    full = gm.generate(pt, n, T, k, p, ut).cpu().numpy()
    np.testing.assert_array_equal(cached, full)
    seq = prompt.copy()
    for s in range(n):
        lg = oracle_last_logits(om, params, seq).astype(np.float32)
        seq = np.concatenate([seq, oracle.sample(lg, 512, T, k, p, u[s])[:, None]], axis=1)
    np.testing.assert_array_equal(cached, seq)
    gm.close()


def test_cached_generation_bf16_tracks_recompute(g):
    """bf16 mode: greedy tokens of the cached and the recompute path agree (the
    two paths group the same bf16 computation differently, so a near-tie may
    flip a late token), and the cached path is deterministic."""
    import torch
    om, params, gm = tiny(g, True)
    rng = np.random.default_rng(22)
    B, T0, n = 4, 9, 40
    pt = torch.from_numpy(rng.integers(0, 512, size=(B, T0)).astype(np.int32)).cuda()
    a = gm.generate(pt, n, 0.0, 0, 1.0, None, cached=True).cpu().numpy()
    b = gm.generate(pt, n, 0.0, 0, 1.0, None, cached=True).cpu().numpy()
    np.testing.assert_array_equal(a, b)
    full = gm.generate(pt, n, 0.0, 0, 1.0, None).cpu().numpy()
    # the first generated token comes from the same prefill forward
    np.testing.assert_array_equal(a[:, T0], full[:, T0])
    first_diff = [next((t for t in range(T0, T0 + n) if a[r, t] != full[r, t]), T0 + n)
                  for r in range(B)]
    assert np.mean(first_diff) >= T0 + n / 2, first_diff
    gm.close()


def test_cached_generation_refuses_a_sliding_window(g):
    import torch
    _, _, gm = tiny(g, False)
    pt = torch.zeros((1, 60), dtype=torch.int32, device="cuda")
    with pytest.raises(g.GPT2Error):
        gm.generate(pt, 10, 0.0, 0, 1.0, None, cached=True)  # 70 > context 64
    gm.close()
