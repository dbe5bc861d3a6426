"""The C ABI without a GPU: the library loads, exports every symbol that
include/gpt2.h declares, the binding covers them, and host-side validation
rejects bad configurations before any device call."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gpt2.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt2_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def g():
    import decoder_only_lm_b200 as g
    return g


def test_header_declares_the_step_entry_points():
    names = declared_functions()
    for n in ("gpt2_create", "gpt2_forward_loss", "gpt2_backward", "gpt2_clip_adamw_step",
              "gpt2_eval_loss", "gpt2_batch_from_stream", "gpt2_lmhead_ce"):
        assert n in names


def test_library_exports_every_declared_symbol(g):
    out = subprocess.run(["nm", "-D", "--defined-only", g.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (gpt2_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    # and nothing with C linkage beyond the header
    assert exported <= set(declared_functions())


def test_binding_covers_the_header(g):
    assert set(g.SIGNATURES) == set(declared_functions())
    for n in declared_functions():
        assert callable(getattr(g, n))


def _cfg(g, **kw):
    base = dict(n_layer=2, n_embd=64, n_head=4, vocab_size=512, padded_vocab=512, max_T=64, bf16=0,
                ln_eps=1e-5, max_B=4, max_Tseq=32, resid_init_scale=0, stream=None)
    base.update(kw)
    c = g.Config()
    for k, v in base.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("bad", [dict(n_embd=66), dict(n_head=5), dict(padded_vocab=500),
                                 dict(max_Tseq=128), dict(ln_eps=0.0), dict(n_layer=0),
                                 dict(n_embd=256, n_head=2), dict(resid_init_scale=1)])
def test_create_rejects_bad_config_on_the_host(g, bad):
    h = C.c_void_p()
    rc = g.lib.gpt2_create(C.byref(_cfg(g, **bad)), C.byref(h))
    assert rc == g.ERR_ARG and not h.value
    assert g.lib.gpt2_last_error(None)


def test_null_arguments_are_refused(g):
    assert g.lib.gpt2_create(None, None) == g.ERR_ARG
    assert g.lib.gpt2_backward(None, 1.0) == g.ERR_ARG
    assert g.lib.gpt2_zero_grad(None) == g.ERR_ARG
    ws = C.c_size_t()
    assert g.lib.gpt2_lmhead_ce_workspace(0, 64, 64, g.BF16, C.byref(ws)) == g.ERR_ARG
    assert g.lib.gpt2_lmhead_ce_workspace(128, 768, 50304, g.BF16, C.byref(ws)) == g.OK
    assert ws.value >= 128 * 50304 * 2  # holds the rows' dz (bf16)
    assert ws.value < 8192 * 50304 * 2  # ... and less than the full [8192, 50304] bf16 logits
    # the live dz is one 2048-row chunk whatever M is: at the GPT-2
    # 124M batch (16 x 1024 rows) the whole workspace stays within 256 MB, and
    # from there on it grows only by the per-row partials of the forward
    # (197 column tiles x 2 x 4 B) and the per-row target logit
    sizes = {}
    for M in (2048, 16384, 65536):
        assert g.lib.gpt2_lmhead_ce_workspace(M, 768, 50304, g.BF16, C.byref(ws)) == g.OK
        sizes[M] = ws.value
    assert sizes[16384] <= 256 * 2 ** 20
    assert sizes[16384] < 16384 * 50304 * 2 // 6
    per_row = (sizes[65536] - sizes[16384]) / (65536 - 16384)
    assert per_row <= 197 * 2 * 4 + 4 + 8 + 1  # (two lse/loss words of the op-level call)
    assert sizes[2048] >= 2048 * 50304 * 2
    # fused linear layer: missing inputs and unknown epilogues are refused on the host
    buf = C.c_void_p(16)  # never dereferenced: the arguments are rejected first
    L = g.lib.gpt2_linear
    assert L(g.LINEAR_BIAS, None, buf, 0, None, None, buf, None, 8, 8, 8, g.BF16, None, 0,
             None) == g.ERR_ARG
    assert L(g.LINEAR_BIAS_GELU, buf, buf, 0, None, None, buf, buf, 8, 8, 8, g.BF16, None, 0,
             None) == g.ERR_ARG  # no bias
    assert L(g.LINEAR_RESIDUAL, buf, buf, 0, None, None, buf, None, 8, 8, 8, g.BF16, None, 0,
             None) == g.ERR_ARG  # no residual input
    assert L(g.LINEAR_GELU_BWD, buf, buf, 1, buf, buf, buf, None, 8, 8, 8, g.BF16, None, 0,
             None) == g.ERR_ARG  # a bias given
    assert L(7, buf, buf, 0, None, None, buf, None, 8, 8, 8, g.BF16, None, 0, None) == g.ERR_ARG
    assert L(g.LINEAR_BIAS, buf, buf, 0, None, None, buf, None, 0, 8, 8, g.BF16, None, 0,
             None) == g.ERR_ARG
    # sampling: sizes and settings are checked on the host before any launch
    S = g.lib.gpt2_sample
    assert S(buf, 16, 1, 0, 1.0, 0, 0.9, buf, buf, 1, None) == g.ERR_ARG  # V = 0
    assert S(buf, 16, 1, 53249, 1.0, 0, 0.9, buf, buf, 1, None) == g.ERR_ARG  # V too large
    assert S(buf, 8, 1, 16, 1.0, 0, 0.9, buf, buf, 1, None) == g.ERR_ARG  # ld < V
    assert S(buf, 16, 1, 16, -0.5, 0, 0.9, buf, buf, 1, None) == g.ERR_ARG  # temperature < 0
    assert S(buf, 16, 1, 16, 1.0, -1, 0.9, buf, buf, 1, None) == g.ERR_ARG  # top_k < 0
    assert S(buf, 16, 1, 16, 1.0, 0, 0.0, buf, buf, 1, None) == g.ERR_ARG  # top_p = 0
    assert S(buf, 16, 1, 16, 1.0, 0, 1.5, buf, buf, 1, None) == g.ERR_ARG  # top_p > 1
    assert S(buf, 16, 1, 16, 1.0, 0, 0.9, None, buf, 1, None) == g.ERR_ARG  # no uniforms
    assert g.lib.gpt2_generate(None, buf, 1, 4, 4, 0.0, 0, 1.0, None, buf) == g.ERR_ARG
    assert g.lib.gpt2_generate_cached(None, buf, 1, 4, 4, 0.0, 0, 1.0, None, buf) == g.ERR_ARG
    assert g.lib.gpt2_logits_last(None, buf, 1, 4, 1, buf, 64) == g.ERR_ARG


def test_attention_bwd_workspace_layout(g):
    """gpt2_attention_bwd_workspace as the header states it: one float of Delta
    per (batch, head, position); for bf16 with head size 64, after Delta at a
    1 KB boundary, the causal half of the score gradients in bf16, B*H*n(n+1)/2
    tiles of 128 x 128 with n = ceil(T/128) (226 MB at B=16, T=1024, H=12)."""
    ws = C.c_size_t()

    def size(B, T, Cc, H, dt):
        assert g.lib.gpt2_attention_bwd_workspace(B, T, Cc, H, dt, C.byref(ws)) == g.OK
        return ws.value

    for B, T, Cc, H in [(16, 1024, 768, 12), (2, 130, 128, 2), (3, 1, 128, 2), (1, 2048, 1024, 16)]:
        delta = B * H * T * 4
        n = -(-T // 128)
        assert size(B, T, Cc, H, g.F32) == delta
        assert size(B, T, Cc, H, g.BF16) == -(-delta // 1024) * 1024 + B * H * n * (n + 1) // 2 * 128 * 128 * 2
    assert size(16, 1024, 768, 12, g.BF16) - 16 * 12 * 1024 * 4 == 226_492_416
    # other head sizes (the CUDA-core kernels) keep only Delta
    assert size(2, 100, 64, 2, g.BF16) == 2 * 2 * 100 * 4
    assert size(2, 100, 64, 4, g.BF16) == 2 * 4 * 100 * 4
    # sizes are checked on the host
    assert g.lib.gpt2_attention_bwd_workspace(0, 8, 128, 2, g.BF16, C.byref(ws)) == g.ERR_ARG
    assert g.lib.gpt2_attention_bwd_workspace(1, 8, 128, 2, g.BF16, None) == g.ERR_ARG
