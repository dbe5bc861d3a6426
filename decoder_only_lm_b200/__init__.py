"""Python binding of libgpt2_b200.so, the B200 GPT-2 training-step library.

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  The raw C entry points are available under their C
names (``gpt2_create``, ``gpt2_forward_loss`` ...) through :data:`lib`;
:class:`GPT2` wraps one handle with PyTorch tensors for device memory and
streams.  Importing this package raises if the compiled library is missing:
there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgpt2_b200.so")

PROF_NAMES = ["gemm", "lmhead", "attn_fwd", "attn_bwd", "ln_fwd", "ln_bwd", "embed", "optim",
              "other"]

OK, ERR_ARG, ERR_TOKEN, ERR_NONFINITE, ERR_CUDA, ERR_OOM, ERR_TIMEOUT, ERR_STATE = range(8)
PARAM, GRAD, ADAM_M, ADAM_V = range(4)
F32, BF16 = 0, 1

ALLOC_FN = C.CFUNCTYPE(C.c_void_p, C.c_size_t, C.c_void_p)
FREE_FN = C.CFUNCTYPE(None, C.c_void_p, C.c_void_p)
BUCKET_FN = C.CFUNCTYPE(None, C.c_void_p, C.c_int)


class Config(C.Structure):
    _fields_ = [("n_layer", C.c_int), ("n_embd", C.c_int), ("n_head", C.c_int),
                ("vocab_size", C.c_int), ("padded_vocab", C.c_int), ("max_T", C.c_int),
                ("bf16", C.c_int), ("ln_eps", C.c_float), ("max_B", C.c_int), ("max_Tseq", C.c_int),
                ("resid_init_scale", C.c_int), ("stream", C.c_void_p), ("alloc", ALLOC_FN),
                ("free", FREE_FN), ("alloc_ctx", C.c_void_p)]


_P = C.c_void_p
_i, _i64, _f, _sz = C.c_int, C.c_int64, C.c_float, C.c_size_t

# name -> (restype, argtypes); names are the C ABI's (include/gpt2.h)
SIGNATURES = {
    "gpt2_create": (_i, [C.POINTER(Config), C.POINTER(_P)]),
    "gpt2_destroy": (_i, [_P]),
    "gpt2_last_error": (C.c_char_p, [_P]),
    "gpt2_num_tensors": (_i, [_P, C.POINTER(_i)]),
    "gpt2_tensor_info": (_i, [_P, _i, C.POINTER(C.c_char_p), C.POINTER(_i), C.POINTER(_i64),
                              C.POINTER(_i)]),
    "gpt2_param_count": (_i, [_P, C.POINTER(_i64)]),
    "gpt2_set_tensor": (_i, [_P, _i, _i, _P, _i]),
    "gpt2_get_tensor": (_i, [_P, _i, _i, _P, _i]),
    "gpt2_get_step": (_i, [_P, C.POINTER(_i)]),
    "gpt2_set_step": (_i, [_P, _i]),
    "gpt2_batch_from_stream": (_i, [_P, _P, _i64, _i64, _i, _i, _P, _P]),
    "gpt2_forward_loss": (_i, [_P, _P, _P, _i, _i, _i, C.POINTER(_f), _P]),
    "gpt2_backward": (_i, [_P, _f]),
    "gpt2_zero_grad": (_i, [_P]),
    "gpt2_clip_adamw_step": (_i, [_P, _f, _f, _f, _f, _f, _f, C.POINTER(_f)]),
    "gpt2_train_step": (_i, [_P, _P, _P, _i, _i, _i, _f, _f, _f, _f, _f, _f, C.POINTER(_f),
                             C.POINTER(_f)]),
    "gpt2_eval_loss": (_i, [_P, _P, _P, _i, _i, _i, C.POINTER(_f)]),
    "gpt2_logits_last": (_i, [_P, _P, _i, _i, _i, _P, _i64]),
    "gpt2_sample": (_i, [_P, _i64, _i, _i, _f, _i, _f, _P, _P, _i64, _P]),
    "gpt2_generate": (_i, [_P, _P, _i, _i, _i, _f, _i, _f, _P, _P]),
    "gpt2_generate_cached": (_i, [_P, _P, _i, _i, _i, _f, _i, _f, _P, _P]),
    "gpt2_stream_begin": (_i, [_P, _P, _i64, _i64, _i64, _i, _i, _i, _f, _f, _f, _f, _f]),
    "gpt2_stream_steps": (_i, [_P, _i, C.POINTER(_f)]),
    "gpt2_stream_end": (_i, [_P, C.POINTER(_i64)]),
    "gpt2_stream_kernels": (_i, [_P, C.POINTER(_i64)]),
    "gpt2_synchronize": (_i, [_P]),
    "gpt2_arena": (_i, [_P, _i, C.POINTER(C.POINTER(_f)), C.POINTER(_i64)]),
    "gpt2_arena_layout": (_i, [C.POINTER(Config), _i, C.c_char_p, _i, C.POINTER(_i64),
                               C.POINTER(_i64), C.POINTER(_i)]),
    "gpt2_grad_buckets": (_i, [C.POINTER(Config), _i, C.POINTER(_i), C.POINTER(_i64),
                               C.POINTER(_i64), C.POINTER(_i)]),
    "gpt2_set_bucket_callback": (_i, [_P, BUCKET_FN, _P]),
    "gpt2_dp_unique_id": (_i, [C.c_char_p]),
    "gpt2_dp_init": (_i, [_P, C.c_char_p, _i, _i]),
    "gpt2_dp_sync": (_i, [_P, _i]),
    "gpt2_profile_enable": (_i, [_P, _i]),
    "gpt2_profile_reset": (_i, [_P]),
    "gpt2_profile_read": (_i, [_P, _i, C.POINTER(_i64), C.POINTER(C.c_double), C.POINTER(C.c_double),
                               C.POINTER(C.c_double)]),
    "gpt2_lmhead_ce_workspace": (_i, [_i, _i, _i, _i, C.POINTER(_sz)]),
    "gpt2_lmhead_ce": (_i, [_P, _P, _P, _i, _i, _i, _i, _i, _f, _P, _P, _P, _P, _P, _sz, _P]),
    "gpt2_layernorm_fwd": (_i, [_P, _P, _P, _i64, _i, _f, _P, _i, _P, _P, _P]),
    "gpt2_layernorm_bwd_workspace": (_i, [_i64, _i, C.POINTER(_sz)]),
    "gpt2_layernorm_bwd": (_i, [_P, _i, _P, _P, _P, _P, _i64, _i, _P, _P, _P, _P, _sz, _P]),
    "gpt2_attention_fwd": (_i, [_P, _i, _i, _i, _i, _i, _P, _P, _P]),
    "gpt2_attention_bwd_workspace": (_i, [_i, _i, _i, _i, _i, C.POINTER(_sz)]),
    "gpt2_attention_bwd": (_i, [_P, _P, _P, _P, _i, _i, _i, _i, _i, _P, _P, _sz, _P]),
    "gpt2_attention_bwd_noalloc": (_i, [_P, _P, _P, _P, _i, _i, _i, _i, _i, _P, _P]),
    "gpt2_matmul_workspace": (_i, [_i, _i, _i, C.POINTER(_sz)]),
    "gpt2_matmul": (_i, [_P, _i, _i64, _P, _i, _i64, _i, _i, _i, _i, _f, _i, _P, _i, _i64, _P,
                         _sz, _P]),
    "gpt2_linear": (_i, [_i, _P, _P, _i, _P, _P, _P, _P, _i, _i, _i, _i, _P, _sz, _P]),
    "gpt2_device_error": (_i, [C.POINTER(_i)]),
    "gpt2_launch_count": (_i, [C.POINTER(_i64)]),
    "gpt2_wait_selfcheck": (_i, [C.POINTER(_i)]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python decoder_only_lm_b200/build.py`"
                          " (this package has no CPU fallback)")
    L = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()
globals().update({name: getattr(lib, name) for name in SIGNATURES})


class GPT2Error(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"gpt2 error {code}: {msg}")
        self.code = code


def _check(rc, handle=None):
    if rc != OK:
        msg = lib.gpt2_last_error(handle)
        raise GPT2Error(rc, msg.decode() if msg else "")


def _ptr(t):
    """Device or host address of a torch tensor / numpy array (None stays NULL)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def make_config(n_layer, n_embd, n_head, vocab_size, padded_vocab=None, max_T=1024, bf16=True,
                max_B=1, max_Tseq=None, ln_eps=1e-5):
    """A gpt2_config without stream or allocator (for the host-only calls)."""
    return Config(n_layer, n_embd, n_head, vocab_size, padded_vocab or vocab_size, max_T,
                  1 if bf16 else 0, ln_eps, max_B, max_Tseq or max_T, 0, None, ALLOC_FN(),
                  FREE_FN(), None)


def arena_layout(cfg):
    """[(name, offset, n_elems)] of every tensor in the arenas (gpt2_arena_layout;
    host only)."""
    n = C.c_int()
    _check(lib.gpt2_arena_layout(C.byref(cfg), -1, None, 0, None, None, C.byref(n)))
    out = []
    buf = C.create_string_buffer(128)
    for i in range(n.value):
        off, cnt = C.c_int64(), C.c_int64()
        _check(lib.gpt2_arena_layout(C.byref(cfg), i, buf, 128, C.byref(off), C.byref(cnt), None))
        out.append((buf.value.decode(), off.value, cnt.value))
    return out


DP_ID_BYTES = 128


def dp_unique_id():
    """gpt2_dp_unique_id: the bytes every rank passes to GPT2.dp_init (made on
    one rank, sent to the others)."""
    import torch  # noqa: F401  (NCCL: the process's own copy, as PyTorch loads it)
    buf = C.create_string_buffer(DP_ID_BYTES)
    _check(lib.gpt2_dp_unique_id(buf))
    return buf.raw


def grad_buckets(cfg):
    """[(bucket, offset, count)] of the gradient arena in the order the
    backward finishes the buckets (gpt2_grad_buckets; host only)."""
    n = C.c_int()
    _check(lib.gpt2_grad_buckets(C.byref(cfg), 0, C.byref(n), None, None, None))
    off, cnt, b = (C.c_int64 * n.value)(), (C.c_int64 * n.value)(), (C.c_int * n.value)()
    _check(lib.gpt2_grad_buckets(C.byref(cfg), n.value, C.byref(n), off, cnt, b))
    return [(b[k], off[k], cnt[k]) for k in range(n.value)]


class GPT2:
    """One model handle: parameters, gradients, AdamW state and activations."""

    def __init__(self, n_layer, n_embd, n_head, vocab_size, padded_vocab=None, max_T=1024,
                 bf16=True, max_B=1, max_Tseq=None, ln_eps=1e-5, stream=None,
                 torch_allocator=True):
        import torch
        self.torch = torch
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self._keep = []
        alloc = ALLOC_FN()
        free = FREE_FN()
        if torch_allocator:
            st = self.stream

            def _alloc(nbytes, ctx):
                try:
                    return torch.cuda.caching_allocator_alloc(int(nbytes), stream=st)
                except Exception:  # out of memory: the library reports GPT2_ERR_OOM
                    return None

            def _free(p, ctx):
                torch.cuda.caching_allocator_delete(p)

            alloc, free = ALLOC_FN(_alloc), FREE_FN(_free)
            self._keep += [alloc, free]
        cfg = Config(n_layer, n_embd, n_head, vocab_size, padded_vocab or vocab_size, max_T,
                     1 if bf16 else 0, ln_eps, max_B, max_Tseq or max_T, 0,
                     self.stream.cuda_stream, alloc, free, None)
        self.cfg = cfg
        h = C.c_void_p()
        _check(lib.gpt2_create(C.byref(cfg), C.byref(h)))
        self.h = h
        n = C.c_int()
        _check(lib.gpt2_num_tensors(h, C.byref(n)), h)
        self.tensors = []
        for i in range(n.value):
            name, nd, dec = C.c_char_p(), C.c_int(), C.c_int()
            shape = (C.c_int64 * 2)()
            _check(lib.gpt2_tensor_info(h, i, C.byref(name), C.byref(nd), shape, C.byref(dec)), h)
            shp = (shape[0], shape[1]) if nd.value == 2 else (shape[0],)
            self.tensors.append((name.value.decode(), shp, dec.value))
        self.index = {n: i for i, (n, _, _) in enumerate(self.tensors)}
        cnt = C.c_int64()
        _check(lib.gpt2_param_count(h, C.byref(cnt)), h)
        self.n_params = cnt.value

    # ------------------------------------------------------------- state
    def shapes(self):
        return [(n, s) for n, s, _ in self.tensors]

    def set_tensor(self, name, value, which=PARAM):
        t = self.torch.as_tensor(value, dtype=self.torch.float32)
        t = t.contiguous()
        on_dev = 1 if t.is_cuda else 0
        _check(lib.gpt2_set_tensor(self.h, self.index[name], which, _ptr(t), on_dev), self.h)

    def set_params(self, named):
        for n, _, _ in self.tensors:
            self.set_tensor(n, named[n])

    def get_tensor(self, name, which=PARAM, device=False):
        shape = self.tensors[self.index[name]][1]
        if device:
            out = self.torch.empty(shape, dtype=self.torch.float32, device="cuda")
        else:
            out = np.empty(shape, dtype=np.float32)
        _check(lib.gpt2_get_tensor(self.h, self.index[name], which, _ptr(out), 1 if device else 0),
               self.h)
        return out

    def get_all(self, which=PARAM):
        return {n: self.get_tensor(n, which) for n, _, _ in self.tensors}

    @property
    def step(self):
        t = C.c_int()
        _check(lib.gpt2_get_step(self.h, C.byref(t)), self.h)
        return t.value

    @step.setter
    def step(self, t):
        _check(lib.gpt2_set_step(self.h, int(t)), self.h)

    # ------------------------------------------------------------- step
    @staticmethod
    def _tok(t):
        return t if isinstance(t, np.ndarray) else t.contiguous()

    def batch_from_stream(self, stream_u16, offset, B, T):
        torch = self.torch
        x = torch.empty(B * T, dtype=torch.int32, device="cuda")
        y = torch.empty(B * T, dtype=torch.int32, device="cuda")
        _check(lib.gpt2_batch_from_stream(self.h, _ptr(stream_u16), stream_u16.numel(), offset, B, T,
                                          _ptr(x), _ptr(y)), self.h)
        return x.view(B, T), y.view(B, T)

    def _xy(self, x, y):
        x, y = self._tok(x), self._tok(y)
        on_dev = 0 if isinstance(x, np.ndarray) else int(x.is_cuda)
        if on_dev == 0:
            x = np.ascontiguousarray(np.asarray(x.cpu() if hasattr(x, "cpu") else x, dtype=np.int32))
            y = np.ascontiguousarray(np.asarray(y.cpu() if hasattr(y, "cpu") else y, dtype=np.int32))
        B, T = x.shape
        return x, y, B, T, on_dev

    def forward_loss(self, x, y, loss=True, row_loss=None):
        x, y, B, T, dev = self._xy(x, y)
        out = C.c_float()
        _check(lib.gpt2_forward_loss(self.h, _ptr(x), _ptr(y), B, T, dev,
                                     C.byref(out) if loss else None, _ptr(row_loss)), self.h)
        return out.value if loss else None

    def backward(self, grad_scale=1.0):
        _check(lib.gpt2_backward(self.h, grad_scale), self.h)

    def zero_grad(self):
        _check(lib.gpt2_zero_grad(self.h), self.h)

    def clip_adamw_step(self, lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1,
                        max_norm=1.0, norm=True):
        out = C.c_float()
        _check(lib.gpt2_clip_adamw_step(self.h, lr, beta1, beta2, eps, weight_decay, max_norm,
                                        C.byref(out) if norm else None), self.h)
        return out.value if norm else None

    def train_step(self, x, y, lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1,
                   max_norm=1.0, read=True):
        x, y, B, T, dev = self._xy(x, y)
        loss, norm = C.c_float(), C.c_float()
        _check(lib.gpt2_train_step(self.h, _ptr(x), _ptr(y), B, T, dev, lr, beta1, beta2, eps,
                                   weight_decay, max_norm, C.byref(loss) if read else None,
                                   C.byref(norm) if read else None), self.h)
        return (loss.value, norm.value) if read else None

    def stream_begin(self, stream_u16, start, stride, B, T, accum=1, beta1=0.9, beta2=0.95,
                     eps=1e-8, weight_decay=0.1, max_norm=1.0):
        """gpt2_stream_begin: record one optimizer step over windows of a device
        token stream (kept referenced until stream_end) as a CUDA graph."""
        self._stream_ref = stream_u16
        _check(lib.gpt2_stream_begin(self.h, _ptr(stream_u16), stream_u16.numel(), start, stride,
                                     B, T, accum, beta1, beta2, eps, weight_decay, max_norm),
               self.h)

    def stream_steps(self, lrs):
        """gpt2_stream_steps: one replayed optimizer step per learning rate in lrs."""
        arr = (C.c_float * len(lrs))(*[float(v) for v in lrs])
        _check(lib.gpt2_stream_steps(self.h, len(lrs), arr), self.h)

    def stream_kernels(self):
        """gpt2_stream_kernels: kernels one replay of the recorded step runs."""
        n = C.c_int64()
        _check(lib.gpt2_stream_kernels(self.h, C.byref(n)), self.h)
        return n.value

    def stream_end(self):
        """gpt2_stream_end: returns the cursor (offset of the next window)."""
        cur = C.c_int64()
        rc = lib.gpt2_stream_end(self.h, C.byref(cur))
        self._stream_ref = None
        _check(rc, self.h)
        return cur.value

    def eval_loss(self, x, y):
        x, y, B, T, dev = self._xy(x, y)
        out = C.c_float()
        _check(lib.gpt2_eval_loss(self.h, _ptr(x), _ptr(y), B, T, dev, C.byref(out)), self.h)
        return out.value

    def logits_last(self, x):
        """fp32 logits [B, padded_vocab] of the last position of each row of x [B, T]."""
        torch = self.torch
        x, _, B, T, dev = self._xy(x, x)
        out = torch.empty((B, self.cfg.padded_vocab), dtype=torch.float32, device="cuda")
        _check(lib.gpt2_logits_last(self.h, _ptr(x), B, T, dev, _ptr(out), out.stride(0)), self.h)
        return out

    def generate(self, prompt, n_new, temperature=0.8, top_k=0, top_p=0.9, uniform=None,
                 cached=False):
        """prompt: int32 cuda [B, T0]; uniform: fp32 cuda [n_new, B] in [0, 1) (None
        for greedy settings).  cached: keep a key/value cache (gpt2_generate_cached)
        instead of recomputing the window every step.  Returns int32 cuda
        [B, T0 + n_new]."""
        torch = self.torch
        prompt = prompt.to(device="cuda", dtype=torch.int32).contiguous()
        B, T0 = prompt.shape
        out = torch.empty((B, T0 + n_new), dtype=torch.int32, device="cuda")
        u = None if uniform is None else uniform.to(device="cuda", dtype=torch.float32).contiguous()
        fn = lib.gpt2_generate_cached if cached else lib.gpt2_generate
        _check(fn(self.h, _ptr(prompt), B, T0, n_new, temperature, top_k, top_p, _ptr(u), _ptr(out)),
               self.h)
        return out

    def synchronize(self):
        _check(lib.gpt2_synchronize(self.h), self.h)

    def arena(self, which=GRAD):
        """Zero-copy torch view of one fp32 arena (all tensors, aligned)."""
        ptr, n = C.POINTER(C.c_float)(), C.c_int64()
        _check(lib.gpt2_arena(self.h, which, C.byref(ptr), C.byref(n)), self.h)
        addr = C.cast(ptr, C.c_void_p).value

        class _View:
            __cuda_array_interface__ = {"shape": (n.value,), "typestr": "<f4",
                                        "data": (addr, False), "version": 2}
        return self.torch.as_tensor(_View(), device="cuda")

    def dp_init(self, unique_id, rank, world):
        """gpt2_dp_init: average the gradient buckets over `world` ranks (NCCL)
        inside every backward from now on."""
        if len(unique_id) != DP_ID_BYTES:
            raise ValueError("unique_id must be the bytes of dp_unique_id()")
        _check(lib.gpt2_dp_init(self.h, C.c_char_p(bytes(unique_id)), int(rank), int(world)),
               self.h)

    def dp_sync(self, on=True):
        """gpt2_dp_sync: whether the backward calls that follow exchange."""
        _check(lib.gpt2_dp_sync(self.h, int(bool(on))), self.h)

    def set_bucket_callback(self, fn):
        """gpt2_set_bucket_callback: fn(bucket) is called as the backward makes
        each gradient bucket final (None clears it)."""
        if fn is None:
            self._bucket_cb = None
            _check(lib.gpt2_set_bucket_callback(self.h, BUCKET_FN(), None), self.h)
            return
        self._bucket_cb = BUCKET_FN(lambda user, b: fn(b))
        _check(lib.gpt2_set_bucket_callback(self.h, self._bucket_cb, None), self.h)

    def profile(self, enable=True):
        _check(lib.gpt2_profile_enable(self.h, int(enable)), self.h)

    def profile_reset(self):
        _check(lib.gpt2_profile_reset(self.h), self.h)

    def profile_read(self):
        """{group: dict(launches, ms, flops, bytes)} plus 'total_launches'."""
        out = {}
        for i, name in enumerate(PROF_NAMES):
            n, ms, fl, by = C.c_int64(), C.c_double(), C.c_double(), C.c_double()
            _check(lib.gpt2_profile_read(self.h, i, C.byref(n), C.byref(ms), C.byref(fl), C.byref(by)),
                   self.h)
            out[name] = dict(launches=n.value, ms=ms.value, flops=fl.value, bytes=by.value)
        n = C.c_int64()
        _check(lib.gpt2_profile_read(self.h, -1, C.byref(n), None, None, None), self.h)
        out["total_launches"] = n.value
        return out

    def close(self):
        if getattr(self, "h", None):
            lib.gpt2_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ----------------------------------------------------------------- op-level calls
def _dtype_code(t):
    import torch
    return BF16 if t.dtype == torch.bfloat16 else F32


def lmhead_ce(hidden, W, y, vocab_size, grad_scale=1.0, grads=True, stream=None):
    """Tied head + mean CE on device tensors: returns (loss, lse, dh, dW)."""
    import torch
    M, Cc = hidden.shape
    Vp = W.shape[0]
    dt = _dtype_code(hidden)
    ws_b = C.c_size_t()
    _check(lib.gpt2_lmhead_ce_workspace(M, Cc, Vp, dt, C.byref(ws_b)))
    ws = torch.empty(ws_b.value, dtype=torch.uint8, device=hidden.device)
    loss = torch.empty(1, dtype=torch.float32, device=hidden.device)
    lse = torch.empty(M, dtype=torch.float32, device=hidden.device)
    dh = torch.empty_like(hidden) if grads else None
    dW = torch.zeros(W.shape, dtype=torch.float32, device=hidden.device) if grads else None
    _check(lib.gpt2_lmhead_ce(_ptr(hidden), _ptr(W), _ptr(y), M, Cc, Vp, vocab_size, dt, grad_scale,
                              _ptr(loss), _ptr(lse), _ptr(dh), _ptr(dW), _ptr(ws), ws_b.value,
                              _stream_ptr(stream)))
    return loss, lse, dh, dW


def layernorm_fwd(x, gamma, beta, eps=1e-5, out_dtype=None, stream=None):
    import torch
    M, Cc = x.shape
    out_dtype = out_dtype or torch.float32
    y = torch.empty((M, Cc), dtype=out_dtype, device=x.device)
    mean = torch.empty(M, dtype=torch.float32, device=x.device)
    rstd = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.gpt2_layernorm_fwd(_ptr(x), _ptr(gamma), _ptr(beta), M, Cc, eps, _ptr(y),
                                  _dtype_code(y), _ptr(mean), _ptr(rstd), _stream_ptr(stream)))
    return y, mean, rstd


def layernorm_bwd(dy, x, mean, rstd, gamma, dx=None, dgamma=None, dbeta=None, stream=None):
    import torch
    M, Cc = x.shape
    dx = torch.zeros_like(x) if dx is None else dx
    dgamma = torch.zeros(Cc, dtype=torch.float32, device=x.device) if dgamma is None else dgamma
    dbeta = torch.zeros(Cc, dtype=torch.float32, device=x.device) if dbeta is None else dbeta
    ws_b = C.c_size_t()
    _check(lib.gpt2_layernorm_bwd_workspace(M, Cc, C.byref(ws_b)))
    ws = torch.empty(ws_b.value, dtype=torch.uint8, device=x.device)
    _check(lib.gpt2_layernorm_bwd(_ptr(dy), _dtype_code(dy), _ptr(x), _ptr(mean), _ptr(rstd),
                                  _ptr(gamma), M, Cc, _ptr(dx), _ptr(dgamma), _ptr(dbeta), _ptr(ws),
                                  ws_b.value, _stream_ptr(stream)))
    return dx, dgamma, dbeta


def attention_fwd(qkv, n_head, stream=None):
    import torch
    B, T, C3 = qkv.shape
    out = torch.empty((B, T, C3 // 3), dtype=qkv.dtype, device=qkv.device)
    lse = torch.empty((B, n_head, T), dtype=torch.float32, device=qkv.device)
    _check(lib.gpt2_attention_fwd(_ptr(qkv), _dtype_code(qkv), B, T, C3 // 3, n_head, _ptr(out),
                                  _ptr(lse), _stream_ptr(stream)))
    return out, lse


def attention_bwd(dout, qkv, out, lse, n_head, stream=None):
    import torch
    B, T, C3 = qkv.shape
    dqkv = torch.empty_like(qkv)
    ws_b = C.c_size_t()
    _check(lib.gpt2_attention_bwd_workspace(B, T, C3 // 3, n_head, _dtype_code(qkv), C.byref(ws_b)))
    ws = torch.empty(max(ws_b.value, 1), dtype=torch.uint8, device=qkv.device)
    _check(lib.gpt2_attention_bwd(_ptr(dout), _ptr(qkv), _ptr(out), _ptr(lse), _dtype_code(qkv), B, T,
                                  C3 // 3, n_head, _ptr(dqkv), _ptr(ws), ws_b.value,
                                  _stream_ptr(stream)))
    return dqkv


def attention_bwd_noalloc(dout, qkv, out, lse, n_head, dqkv=None, stream=None):
    """gpt2_attention_bwd_noalloc: no workspace, the scratch is the library's own."""
    import torch
    B, T, C3 = qkv.shape
    dqkv = torch.empty_like(qkv) if dqkv is None else dqkv
    _check(lib.gpt2_attention_bwd_noalloc(_ptr(dout), _ptr(qkv), _ptr(out), _ptr(lse),
                                          _dtype_code(qkv), B, T, C3 // 3, n_head, _ptr(dqkv),
                                          _stream_ptr(stream)))
    return dqkv


def matmul(A, B, a_kmajor=True, b_kmajor=True, M=None, N=None, K=None, alpha=1.0, out=None,
           accumulate=False, stream=None):
    """D[m,n] = alpha * sum_k A(m,k) B(n,k) with the layouts of gpt2_matmul."""
    import torch
    if a_kmajor:
        M_, K_ = A.shape
    else:
        K_, M_ = A.shape
    N_ = B.shape[0] if b_kmajor else B.shape[1]
    M, N, K = M or M_, N or N_, K or K_
    if out is None:
        out = torch.zeros((M, N), dtype=torch.float32, device=A.device)
    ws_b = C.c_size_t()
    _check(lib.gpt2_matmul_workspace(M, N, K, C.byref(ws_b)))
    ws = torch.empty(max(ws_b.value, 1), dtype=torch.uint8, device=A.device)
    _check(lib.gpt2_matmul(_ptr(A), int(a_kmajor), A.stride(0), _ptr(B), int(b_kmajor), B.stride(0),
                           _dtype_code(A), M, N, K, alpha, int(accumulate), _ptr(out),
                           _dtype_code(out), out.stride(0), _ptr(ws), ws_b.value,
                           _stream_ptr(stream)))
    return out


LINEAR_BIAS, LINEAR_BIAS_GELU, LINEAR_RESIDUAL, LINEAR_GELU_BWD = 0, 1, 2, 3


def linear(epi, x, w, bias=None, inp=None, w_kn=False, out=None, out2=None, stream=None):
    """One linear layer with its fused epilogue (gpt2_linear): y = x W^T (W [N,K])
    or x W (w_kn, W [K,N]), then bias / bias+GELU / residual add / GELU backward.
    Returns out, or (out, pre-activation) for LINEAR_BIAS_GELU."""
    import torch
    M, K = x.shape
    N = w.shape[1] if w_kn else w.shape[0]
    if out is None:
        dt = torch.float32 if epi == LINEAR_RESIDUAL else x.dtype
        out = torch.empty((M, N), dtype=dt, device=x.device)
    if epi == LINEAR_BIAS_GELU and out2 is None:
        out2 = torch.empty((M, N), dtype=x.dtype, device=x.device)
    ws_b = C.c_size_t()
    _check(lib.gpt2_matmul_workspace(M, N, K, C.byref(ws_b)))
    ws = torch.empty(max(ws_b.value, 1), dtype=torch.uint8, device=x.device)
    _check(lib.gpt2_linear(epi, _ptr(x), _ptr(w), int(w_kn), _ptr(bias), _ptr(inp), _ptr(out),
                           _ptr(out2), M, N, K, _dtype_code(x), _ptr(ws), ws_b.value,
                           _stream_ptr(stream)))
    return (out, out2) if epi == LINEAR_BIAS_GELU else out


def sample(logits, vocab, temperature=0.8, top_k=0, top_p=0.9, uniform=None, out=None,
           stream=None):
    """Next token of each row of fp32 cuda logits [B, >= vocab] (gpt2_sample);
    uniform: fp32 cuda [B] in [0, 1) (None for greedy settings)."""
    import torch
    B = logits.shape[0]
    if out is None:
        out = torch.empty(B, dtype=torch.int32, device=logits.device)
    u = None if uniform is None else uniform.to(device=logits.device, dtype=torch.float32).contiguous()
    _check(lib.gpt2_sample(_ptr(logits), logits.stride(0), B, vocab, temperature, top_k, top_p,
                           _ptr(u), _ptr(out), out.stride(0) if out.dim() > 1 else 1,
                           _stream_ptr(stream)))
    return out


def cosine_lr(t, max_lr, min_lr, warmup_steps, total_steps):
    """Learning rate for schedule step t, counted from 0 [CS336 §2, learning-rate
    schedule: linear warmup from 0 to max_lr over warmup_steps, then half a
    cosine period down to min_lr at total_steps, min_lr from there on; LECTURE:
    max 6e-4 with a minimum of 10% of it].  Host-side: the value is passed to
    clip_adamw_step as lr.  The optimizer's own step count (bias correction)
    starts at 1 and is kept by the library."""
    import math
    if warmup_steps < 0 or warmup_steps >= total_steps:
        raise ValueError("cosine_lr needs 0 <= warmup_steps < total_steps")
    if t >= total_steps:
        return min_lr
    if t < warmup_steps:
        return max_lr * (t / warmup_steps)
    phase = math.pi * (t - warmup_steps) / (total_steps - warmup_steps)
    return min_lr + (max_lr - min_lr) * (1.0 + math.cos(phase)) / 2.0


def launch_count():
    """Kernel launches issued by the library from this thread so far."""
    n = C.c_int64()
    _check(lib.gpt2_launch_count(C.byref(n)))
    return n.value


def wait_selfcheck():
    """gpt2_wait_selfcheck: True when a deliberately unmet device wait gave up
    (after its 2 s budget) and was recorded."""
    e = C.c_int()
    _check(lib.gpt2_wait_selfcheck(C.byref(e)))
    return bool(e.value)


def device_error():
    c = C.c_int()
    _check(lib.gpt2_device_error(C.byref(c)))
    return c.value
