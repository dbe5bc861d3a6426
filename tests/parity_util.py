"""Shared set-up of the GPU-vs-oracle parity tests: one configuration, the
same seeded inputs on both sides, and the tolerance metrics."""
from dataclasses import dataclass

import numpy as np

import oracle
import synth

# Tolerances of the comparison (GPU path vs the float64 oracle):
#   fp32 mode: |loss| <= 1e-4 nats, per-tensor gradient relative L2 <= 1e-3
#   bf16 mode: |loss| <= 2e-2 nats, per-tensor gradient relative L2 <= 3e-2
TOL = {False: dict(loss=1e-4, grad=1e-3), True: dict(loss=2e-2, grad=3e-2)}


@dataclass
class Shape:
    n_layer: int
    n_embd: int
    n_head: int
    vocab_size: int
    padded_vocab: int
    max_T: int
    B: int
    T: int


# The tiny fp32 workload (L=2, C=64, H=4, F=256, V=512, T_max=64; B=4, T=32).
TINY = Shape(2, 64, 4, 512, 512, 64, 4, 32)
# Several tiles plus ragged tails: B*T = 300 rows, T = 100 (not a multiple of
# any tile), padded vocabulary with 24 pad rows, head size 64.
RAGGED = Shape(2, 128, 2, 1000, 1024, 128, 3, 100)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    n = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (n if n > 0 else 1.0)


def oracle_model(s: Shape):
    return oracle.Model(s.n_layer, s.n_embd, s.n_head, s.vocab_size, s.padded_vocab, s.max_T)


def gpu_model(s: Shape, bf16: bool, max_B=None, max_Tseq=None):
    import decoder_only_lm_b200 as g
    return g.GPT2(s.n_layer, s.n_embd, s.n_head, s.vocab_size, s.padded_vocab, s.max_T, bf16=bf16,
                  max_B=max_B or s.B, max_Tseq=max_Tseq or s.T)


def inputs(s: Shape, seed=0, stream_seed=1, uniform=True):
    """Seeded weights and a B*T+1 token stream cut into x, y.  uniform=False
    draws the web-text stand-in instead: Zipf(1.1) ids with the last id of the
    vocabulary as the end-of-text separator before every document (id 0 is
    then about 14% of the tokens at V = 50257, more at small V)."""
    om = oracle_model(s)
    named = synth.init_params(seed, om.shapes())
    n = s.B * s.T + 1
    if uniform:
        stream = synth.uniform_stream(stream_seed, n, s.vocab_size)
    else:
        stream = synth.token_stream(stream_seed, n, eot=s.vocab_size - 1)
    x, y = oracle.batch_from_stream(stream, 0, s.B, s.T)
    return om, named, stream, x, y
