"""An independent float64 PyTorch (CPU) GPT-2, used only to pin the oracle.

It is built from library routines (F.layer_norm, F.linear, F.gelu with the
tanh approximation, F.scaled_dot_product_attention with is_causal, and
F.cross_entropy) and takes its gradients from autograd, so it shares neither
code nor closed-form derivatives with the oracle.
"""
import numpy as np
import torch
import torch.nn.functional as F


def to_torch(named, dtype=torch.float64, requires_grad=True):
    return {k: torch.tensor(np.asarray(v), dtype=dtype, requires_grad=requires_grad)
            for k, v in named.items()}


def forward(P, x, y, n_layer, n_head, eps=1e-5, untied_head=None, reduction="mean"):
    x = torch.as_tensor(np.asarray(x), dtype=torch.long)
    y = torch.as_tensor(np.asarray(y), dtype=torch.long)
    B, T = x.shape
    C = P["wte"].shape[1]
    h = F.embedding(x, P["wte"]) + P["wpe"][:T][None]
    for l in range(n_layer):
        p = lambda n: P[f"h.{l}.{n}"]
        a = F.layer_norm(h, (C,), p("ln1.w"), p("ln1.b"), eps)
        qkv = F.linear(a, p("attn.qkv.w"), p("attn.qkv.b"))
        q, k, v = qkv.split(C, dim=2)
        sh = lambda t: t.view(B, T, n_head, C // n_head).transpose(1, 2)
        o = F.scaled_dot_product_attention(sh(q), sh(k), sh(v), is_causal=True)
        o = o.transpose(1, 2).reshape(B, T, C)
        h = h + F.linear(o, p("attn.proj.w"), p("attn.proj.b"))
        a = F.layer_norm(h, (C,), p("ln2.w"), p("ln2.b"), eps)
        u = F.linear(a, p("mlp.fc.w"), p("mlp.fc.b"))
        h = h + F.linear(F.gelu(u, approximate="tanh"), p("mlp.proj.w"), p("mlp.proj.b"))
    hf = F.layer_norm(h, (C,), P["lnf.w"], P["lnf.b"], eps)
    head = P["wte"] if untied_head is None else untied_head
    logits = F.linear(hf, head)
    loss = F.cross_entropy(logits.view(B * T, -1), y.view(-1), reduction=reduction)
    return loss, logits
