"""Seeded synthetic inputs shared by the CUDA path and the CPU oracle.

This module only makes inputs: random numbers, weights at their initial
values, and token streams.  It holds none of the model's arithmetic, so both
sides of every parity test can draw from it without sharing any of the method.

Generator
---------
Every stream of random 64-bit words is the counter-based form of splitmix64
(Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014): word ``i`` (0-based) of the stream keyed by ``key`` is
``mix(key + (i + 1) * 0x9E3779B97F4A7C15)`` with the published finaliser
``mix``.  Being counter based, any slice of a stream can be produced
directly and in vectorised numpy.

* uniform in [0, 1): the top 53 bits of a word times 2**-53;
* normal: Box-Muller on two uniforms of one pair of words (2k, 2k+1);
* integer in [0, n): floor(u * n);
* Zipf(s) over ranks 1..R: inverse CDF on the normalised table of r**-s;
* geometric on {1, 2, ...} with success probability p: inverse CDF.

Workload recipes (token streams, initial weights) follow the pages' GPT-2
training setups: ids are uint16 in a headerless stream, every document is
preceded by the end-of-text id, weights are N(0, 0.02) for matrices with
zero biases and unit LayerNorm gains.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "GOLDEN", "mix64", "derive_key", "words", "uniform", "normal", "randint",
    "zipf_ids", "geometric", "token_stream", "uniform_stream", "init_tensor",
    "init_params", "EOT",
]

GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1

#: GPT-2's end-of-text id (the last of its 50,257 vocabulary entries).
EOT = 50256


def _mix_scalar(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def mix64(z: int) -> int:
    """splitmix64 finaliser on one Python integer (used to derive keys)."""
    return _mix_scalar(z)


def derive_key(seed: int, *tags: int) -> int:
    """A stream key from a seed and integer tags (tensor index, purpose ...)."""
    k = _mix_scalar(seed + GOLDEN)
    for t in tags:
        k = _mix_scalar(k ^ _mix_scalar((t + 1) * GOLDEN))
    return k


def words(key: int, n: int, offset: int = 0) -> np.ndarray:
    """Words offset .. offset+n-1 of the splitmix64 stream keyed by ``key``."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        z = np.uint64(key & _MASK) + i * np.uint64(GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
        z = z ^ (z >> np.uint64(31))
    return z


def uniform(key: int, n: int, offset: int = 0) -> np.ndarray:
    """n doubles in [0, 1)."""
    return (words(key, n, offset) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(key: int, n: int, std: float = 1.0) -> np.ndarray:
    """n N(0, std^2) doubles by Box-Muller (both outputs of each pair are used)."""
    npair = (n + 1) // 2
    w = words(key, 2 * npair)
    u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)  # (0, 1]
    u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)          # [0, 1)
    r = np.sqrt(-2.0 * np.log(u1))
    z = np.empty(2 * npair, dtype=np.float64)
    z[0::2] = r * np.cos(2.0 * np.pi * u2)
    z[1::2] = r * np.sin(2.0 * np.pi * u2)
    return z[:n] * std


def randint(key: int, n: int, high: int) -> np.ndarray:
    """n integers uniform in [0, high)."""
    return np.minimum(np.floor(uniform(key, n) * high), high - 1).astype(np.int64)


def zipf_ids(key: int, n: int, s: float = 1.1, ranks: int = 50256) -> np.ndarray:
    """n ids in [0, ranks): id = rank - 1 with P(rank r) proportional to r**-s."""
    r = np.arange(1, ranks + 1, dtype=np.float64)
    cdf = np.cumsum(r ** -s)
    cdf /= cdf[-1]
    u = uniform(key, n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), ranks - 1).astype(np.int64)


def geometric(key: int, n: int, p: float) -> np.ndarray:
    """n draws of a geometric law on {1, 2, ...} with success probability p."""
    u = 1.0 - uniform(key, n)  # (0, 1]
    return (np.floor(np.log(u) / np.log1p(-p)) + 1).astype(np.int64)


def token_stream(seed: int, n_tokens: int, zipf_s: float = 1.1, mean_doc: float = 600.0,
                 eot: int = EOT) -> np.ndarray:
    """A uint16 stream standing in for a tokenised web corpus.

    Each document is preceded by ``eot``; document lengths are geometric with
    mean ``mean_doc``; ids inside documents are Zipf(``zipf_s``) over the
    ``eot`` ordinary ids 0 .. eot-1.
    """
    ids = zipf_ids(derive_key(seed, 1), n_tokens, zipf_s, eot)
    n_docs = int(n_tokens / mean_doc * 2) + 16
    while True:
        lens = geometric(derive_key(seed, 2), n_docs, 1.0 / mean_doc)
        starts = np.concatenate([[0], np.cumsum(lens + 1)[:-1]])
        if starts[-1] + lens[-1] + 1 >= n_tokens:
            break
        n_docs *= 2
    starts = starts[starts < n_tokens]
    ids[starts] = eot
    return ids.astype(np.uint16)


def uniform_stream(seed: int, n_tokens: int, vocab: int) -> np.ndarray:
    """A uint16 stream of ids uniform in [0, vocab)."""
    return randint(derive_key(seed, 3), n_tokens, vocab).astype(np.uint16)


def init_tensor(seed: int, index: int, name: str, shape, std: float = 0.02) -> np.ndarray:
    """Initial value of one parameter tensor, as float32.

    Matrices (2-D) are N(0, std^2) from the stream keyed by (seed, index);
    LayerNorm gains (names ending in ``.w`` with one dimension) are 1 and every
    other vector (biases, LayerNorm shifts) is 0.
    """
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape))
    if len(shape) == 2:
        return normal(derive_key(seed, 100, index), n, std).astype(np.float32).reshape(shape)
    if name.endswith(".w"):
        return np.ones(shape, dtype=np.float32)
    return np.zeros(shape, dtype=np.float32)


def init_params(seed: int, tensors, std: float = 0.02, scale_names=None, scale: float = 1.0):
    """Initial values for a list of (name, shape) in order: {name: float32 array}.

    ``scale_names`` (optional) lists tensors whose std is multiplied by ``scale``
    (used for the 1/sqrt(2L) residual-projection scaling, off by default).
    """
    out = {}
    for i, (name, shape) in enumerate(tensors):
        s = std * (scale if scale_names and name in scale_names else 1.0)
        out[name] = init_tensor(seed, i, name, shape, s)
    return out
