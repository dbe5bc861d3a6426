"""ctypes front-end of the CPU oracle — TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The oracle (``oracle.cpp``) is a plain
CPU implementation of the GPT-2 training step written from the pages'
definitions; it shares no code with the CUDA library.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


class Cfg(C.Structure):
    _fields_ = [("n_layer", C.c_int), ("n_embd", C.c_int), ("n_head", C.c_int),
                ("vocab_size", C.c_int), ("padded_vocab", C.c_int), ("max_T", C.c_int),
                ("ln_eps", C.c_double)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = C.CDLL(path)
        _declare(_lib)
    return _lib


_P = C.c_void_p


def _declare(L):
    i64, i32, dbl = C.c_int64, C.c_int, C.c_double
    L.oracle_num_threads.restype = i32
    L.oracle_num_tensors.argtypes = [C.POINTER(Cfg)]
    L.oracle_tensor_info.argtypes = [C.POINTER(Cfg), i32, C.c_char_p, i32, C.POINTER(i64),
                                     C.POINTER(i64), C.POINTER(i32), C.POINTER(i64)]
    L.oracle_param_count.argtypes = [C.POINTER(Cfg)]
    L.oracle_param_count.restype = i64
    L.oracle_batch_from_stream.argtypes = [_P, i64, i64, i32, i32, _P, _P]
    for suf in ("f32", "f64"):
        getattr(L, f"oracle_fwd_bwd_{suf}").argtypes = [C.POINTER(Cfg), _P, _P, _P, i32, i32, dbl,
                                                        C.POINTER(dbl), _P, _P, _P]
        getattr(L, f"oracle_clip_adamw_{suf}").argtypes = [C.POINTER(Cfg), _P, _P, _P, _P, i32, dbl,
                                                           dbl, dbl, dbl, dbl, dbl, C.POINTER(dbl)]
        getattr(L, f"oracle_layernorm_{suf}").argtypes = [_P, _P, _P, i64, i64, dbl, _P, _P, _P]
        getattr(L, f"oracle_layernorm_bwd_{suf}").argtypes = [_P, _P, _P, _P, _P, i64, i64, _P, _P, _P]
        getattr(L, f"oracle_gelu_{suf}").argtypes = [_P, i64, _P]
        getattr(L, f"oracle_gelu_bwd_{suf}").argtypes = [_P, _P, i64, _P]
        getattr(L, f"oracle_attention_{suf}").argtypes = [_P, i32, i32, i32, i32, _P]
        getattr(L, f"oracle_attention_bwd_{suf}").argtypes = [_P, _P, i32, i32, i32, i32, _P]
        getattr(L, f"oracle_ce_{suf}").argtypes = [_P, _P, i64, i64, _P, C.POINTER(dbl)]
        getattr(L, f"oracle_lmhead_ce_{suf}").argtypes = [_P, _P, _P, i64, i64, i64, i64, dbl,
                                                          C.POINTER(dbl), _P, _P, _P]


ERRORS = {1: "bad argument", 2: "token id out of range", 3: "non-finite gradient norm"}


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle error {code}: {ERRORS.get(code, '?')}")
        self.code = code


def _chk(rc):
    if rc != 0:
        raise OracleError(rc)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _arr(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def _suf(dtype):
    return {np.dtype(np.float32): "f32", np.dtype(np.float64): "f64"}[np.dtype(dtype)]


def num_threads() -> int:
    return lib().oracle_num_threads()


class Model:
    """The oracle's view of one GPT-2 configuration."""

    def __init__(self, n_layer, n_embd, n_head, vocab_size, padded_vocab=None, max_T=1024,
                 ln_eps=1e-5):
        self.cfg = Cfg(n_layer, n_embd, n_head, vocab_size, padded_vocab or vocab_size, max_T,
                       ln_eps)
        n = lib().oracle_num_tensors(C.byref(self.cfg))
        if n < 0:
            raise OracleError(1)
        self.tensors = []
        buf = C.create_string_buffer(128)
        for i in range(n):
            r, c, nd, off = C.c_int64(), C.c_int64(), C.c_int(), C.c_int64()
            _chk(lib().oracle_tensor_info(C.byref(self.cfg), i, buf, 128, C.byref(r), C.byref(c),
                                          C.byref(nd), C.byref(off)))
            shape = (r.value, c.value) if nd.value == 2 else (r.value,)
            self.tensors.append((buf.value.decode(), shape, off.value))
        self.n_params = lib().oracle_param_count(C.byref(self.cfg))

    def shapes(self):
        return [(n, s) for n, s, _ in self.tensors]

    def pack(self, named, dtype=np.float64):
        flat = np.empty(self.n_params, dtype=dtype)
        for n, s, off in self.tensors:
            flat[off:off + int(np.prod(s))] = np.asarray(named[n], dtype=dtype).reshape(-1)
        return flat

    def unpack(self, flat):
        return {n: flat[off:off + int(np.prod(s))].reshape(s) for n, s, off in self.tensors}

    def fwd_bwd(self, params, x, y, grads=True, grad_scale=1.0, row_loss=False, logits=False,
                grads_in=None):
        """Returns (loss, row_loss or None, grads or None, logits or None)."""
        dt = params.dtype
        x = _arr(x, np.int32)
        y = _arr(y, np.int32)
        B, T = x.shape
        loss = C.c_double()
        rl = np.zeros(B * T, dtype=dt) if row_loss else None
        g = None
        if grads:
            g = np.zeros(self.n_params, dtype=dt) if grads_in is None else grads_in
        lg = np.zeros((B * T, self.cfg.padded_vocab), dtype=dt) if logits else None
        fn = getattr(lib(), f"oracle_fwd_bwd_{_suf(dt)}")
        _chk(fn(C.byref(self.cfg), _ptr(params), _ptr(x), _ptr(y), B, T, grad_scale, C.byref(loss),
                _ptr(rl), _ptr(g), _ptr(lg)))
        return loss.value, rl, g, lg

    def clip_adamw(self, params, grads, m, v, t, lr=6e-4, b1=0.9, b2=0.95, eps=1e-8, wd=0.1,
                   max_norm=1.0):
        """Updates params, m, v in place; returns the pre-clip gradient norm."""
        nrm = C.c_double()
        fn = getattr(lib(), f"oracle_clip_adamw_{_suf(params.dtype)}")
        _chk(fn(C.byref(self.cfg), _ptr(params), _ptr(grads), _ptr(m), _ptr(v), t, lr, b1, b2,
                eps, wd, max_norm, C.byref(nrm)))
        return nrm.value


def batch_from_stream(stream, offset, B, T):
    s = _arr(stream, np.uint16)
    x = np.empty((B, T), dtype=np.int32)
    y = np.empty((B, T), dtype=np.int32)
    _chk(lib().oracle_batch_from_stream(_ptr(s), s.size, offset, B, T, _ptr(x), _ptr(y)))
    return x, y


def layernorm(x, g, b, eps=1e-5):
    dt = x.dtype
    M, Cc = x.shape
    y = np.empty_like(x)
    mean = np.empty(M, dtype=dt)
    rstd = np.empty(M, dtype=dt)
    _chk(getattr(lib(), f"oracle_layernorm_{_suf(dt)}")(_ptr(x), _ptr(_arr(g, dt)), _ptr(_arr(b, dt)),
                                                        M, Cc, eps, _ptr(y), _ptr(mean), _ptr(rstd)))
    return y, mean, rstd


def layernorm_bwd(dy, x, mean, rstd, g):
    dt = x.dtype
    M, Cc = x.shape
    dx = np.zeros_like(x)
    dg = np.zeros(Cc, dtype=dt)
    db = np.zeros(Cc, dtype=dt)
    _chk(getattr(lib(), f"oracle_layernorm_bwd_{_suf(dt)}")(_ptr(_arr(dy, dt)), _ptr(x), _ptr(mean),
                                                            _ptr(rstd), _ptr(_arr(g, dt)), M, Cc,
                                                            _ptr(dx), _ptr(dg), _ptr(db)))
    return dx, dg, db


def gelu(u):
    g = np.empty_like(u)
    _chk(getattr(lib(), f"oracle_gelu_{_suf(u.dtype)}")(_ptr(u), u.size, _ptr(g)))
    return g


def gelu_bwd(dg, u):
    du = np.empty_like(u)
    _chk(getattr(lib(), f"oracle_gelu_bwd_{_suf(u.dtype)}")(_ptr(_arr(dg, u.dtype)), _ptr(u), u.size,
                                                            _ptr(du)))
    return du


def attention(qkv, H):
    """qkv [B, T, 3C] -> out [B, T, C]."""
    B, T, C3 = qkv.shape
    out = np.empty((B, T, C3 // 3), dtype=qkv.dtype)
    _chk(getattr(lib(), f"oracle_attention_{_suf(qkv.dtype)}")(_ptr(qkv), B, T, C3 // 3, H, _ptr(out)))
    return out


def attention_bwd(dout, qkv, H):
    B, T, C3 = qkv.shape
    d = np.empty_like(qkv)
    _chk(getattr(lib(), f"oracle_attention_bwd_{_suf(qkv.dtype)}")(_ptr(_arr(dout, qkv.dtype)), _ptr(qkv),
                                                                    B, T, C3 // 3, H, _ptr(d)))
    return d


def cross_entropy(z, y):
    """z [M, V] logits, y [M] -> (mean loss, row losses)."""
    M, V = z.shape
    rl = np.empty(M, dtype=z.dtype)
    mean = C.c_double()
    _chk(getattr(lib(), f"oracle_ce_{_suf(z.dtype)}")(_ptr(z), _ptr(_arr(y, np.int32)), M, V, _ptr(rl),
                                                      C.byref(mean)))
    return mean.value, rl


def lmhead_ce(h, W, y, vocab_size=None, grad_scale=1.0, grads=True):
    """Tied head + mean CE: returns (loss, row_loss, dh, dW)."""
    dt = h.dtype
    M, Cc = h.shape
    Vp = W.shape[0]
    rl = np.empty(M, dtype=dt)
    dh = np.zeros_like(h) if grads else None
    dW = np.zeros_like(W) if grads else None
    loss = C.c_double()
    _chk(getattr(lib(), f"oracle_lmhead_ce_{_suf(dt)}")(_ptr(h), _ptr(_arr(W, dt)), _ptr(_arr(y, np.int32)),
                                                        M, Cc, Vp, vocab_size or Vp, grad_scale,
                                                        C.byref(loss), _ptr(rl), _ptr(dh), _ptr(dW)))
    return loss.value, rl, dh, dW


# weights of the draw: probabilities as integers in units of 2^-36 (exact sums)
SAMPLE_WEIGHT_SCALE = 2.0 ** 36


def sample(logits, vocab, temperature, top_k, top_p, u):
    """Next-token choice for each row of ``logits`` [B, >= vocab] (fp32), following
    the text-generation section of the CS336 pre-training page (§5: temperature,
    top-p) and the lecture's top-k, step by step:

    - temperature == 0 (or top_k == 1): the highest logit, the first such id on
      ties (greedy decoding);
    - else p_i = exp((z_i - max z) / temperature) in fp32 over the first
      ``vocab`` columns (the real vocabulary; padding columns are never drawn),
      and the weight of id i is w_i = rint(p_i * 2^36) (an integer: every
      cumulative probability below is an exact integer sum);
    - order the ids by probability, highest first, the smaller id first among
      equal probabilities;
    - top_k > 0: keep the first top_k of that order;
    - top_p < 1: keep, in that order, the shortest prefix whose weight reaches
      top_p times the kept weight (the crossing id included);
    - draw with u[b] in [0, 1): walk the kept ids in increasing id order,
      accumulating w, and return the first id at which the sum exceeds
      u[b] times the kept weight (the last kept id if none does).

    Returns int32 [B].
    """
    z_all = np.asarray(logits, dtype=np.float32)
    B = z_all.shape[0]
    u = np.asarray(u, dtype=np.float32).reshape(-1) if u is not None else None
    out = np.empty(B, dtype=np.int32)
    for b in range(B):
        z = z_all[b, :vocab]
        if temperature == 0 or top_k == 1:
            out[b] = int(np.argmax(z))
            continue
        p = np.exp((z - z.max()) / np.float32(temperature)).astype(np.float32)
        w = np.rint(p.astype(np.float64) * SAMPLE_WEIGHT_SCALE).astype(np.int64)
        ids = np.arange(vocab)
        order = np.lexsort((ids, -p))  # probability descending, then id ascending
        if 0 < top_k < vocab:
            order = order[:top_k]
        if top_p < 1:
            cum = np.cumsum(w[order])
            need = np.float64(np.float32(top_p)) * np.float64(cum[-1])
            cut = int(np.argmax(cum.astype(np.float64) >= need)) + 1
            order = order[:cut]
        kept = np.sort(order)
        wk = w[kept]
        target = np.float64(u[b]) * np.float64(wk.sum())
        cum = np.cumsum(wk).astype(np.float64)
        hit = np.nonzero(cum > target)[0]
        out[b] = kept[hit[0]] if hit.size else kept[-1]
    return out
