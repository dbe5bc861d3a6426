"""Pins of the oracle's next-token sampling (temperature, top-k, top-p, the draw)
against the pages' worked example, library routines and closed forms."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def draws(z, V, T, k, p, n=4000):
    """Ids drawn for n evenly spaced u in [0, 1) (one row)."""
    u = (np.arange(n) + 0.5) / n
    zz = np.repeat(np.asarray(z, np.float32)[None, :], n, axis=0)
    return oracle.sample(zz, V, T, k, p, u)


def test_top_p_worked_example():
    """The page's example: sorted probabilities 0.50, 0.25, 0.15, 0.10 with
    p = 0.8 keep three tokens; the draw renormalises over them."""
    g = json.load(open(os.path.join(GOLDEN, "top_p_cs336.json")))
    probs = np.array(g["sorted_probs"])
    perm = np.array([2, 0, 3, 1])  # place the sorted tokens at shuffled ids
    z = np.zeros(4, np.float32)
    z[perm] = np.log(probs).astype(np.float32)
    ids = draws(z, 4, 1.0, 0, g["top_p"])
    kept = set(np.unique(ids).tolist())
    assert len(kept) == g["kept"] and kept == set(perm[: g["kept"]].tolist())
    freq = np.array([np.mean(ids == perm[i]) for i in range(g["kept"])])
    np.testing.assert_allclose(freq, probs[: g["kept"]] / probs[: g["kept"]].sum(), atol=1e-3)


def test_greedy_is_first_argmax():
    rng = np.random.default_rng(0)
    z = rng.normal(size=(5, 300)).astype(np.float32)
    z[1, 7] = z[1, 200] = z[1].max() + 1  # a tie: the smaller id wins
    for T, k in ((0.0, 0), (0.7, 1), (2.0, 1)):
        got = oracle.sample(z, 300, T, k, 0.9, np.full(5, 0.999))
        np.testing.assert_array_equal(got, np.argmax(z, axis=1))
    assert oracle.sample(z, 300, 0.0, 0, 1.0, np.zeros(5))[1] == 7


@pytest.mark.parametrize("T", [0.5, 1.0, 1.7])
def test_full_distribution_matches_softmax(T):
    """No filtering: the draw over evenly spaced u reproduces softmax(z / T)
    (scipy) to within the grid's resolution."""
    from scipy.special import softmax
    rng = np.random.default_rng(1)
    V = 40
    z = (rng.normal(size=V) * 2).astype(np.float32)
    n = 20000
    ids = draws(z, V, T, 0, 1.0, n)
    freq = np.bincount(ids, minlength=V) / n
    np.testing.assert_allclose(freq, softmax(z.astype(np.float64) / T), atol=2.0 / n)


def test_top_k_set_and_weights():
    """top-k keeps exactly the k largest logits (torch.topk) with weights
    proportional to their probabilities; k >= V keeps everything."""
    import torch
    rng = np.random.default_rng(2)
    V, k, n = 64, 5, 20000
    z = rng.normal(size=V).astype(np.float32)
    ids = draws(z, V, 1.0, k, 1.0, n)
    top = set(torch.topk(torch.from_numpy(z), k).indices.tolist())
    assert set(np.unique(ids).tolist()) == top
    sel = np.array(sorted(top))
    w = np.exp(z[sel].astype(np.float64) - z.max())
    freq = np.array([np.mean(ids == i) for i in sel])
    np.testing.assert_allclose(freq, w / w.sum(), atol=2.0 / n)
    np.testing.assert_array_equal(draws(z, V, 1.0, V + 3, 1.0, 500), draws(z, V, 1.0, 0, 1.0, 500))


def test_top_p_is_shortest_prefix_reaching_p():
    """The kept set is the smallest set of most probable tokens whose mass
    reaches p (checked by brute force over prefix sizes)."""
    from scipy.special import softmax
    rng = np.random.default_rng(3)
    V = 30
    for trial in range(20):
        z = (rng.normal(size=V) * 1.5).astype(np.float32)
        p = float(rng.uniform(0.05, 0.99))
        prob = softmax(z.astype(np.float64))
        srt = np.argsort(-prob, kind="stable")
        need = next(n for n in range(1, V + 1) if prob[srt[:n]].sum() >= p - 1e-12)
        kept = set(np.unique(draws(z, V, 1.0, 0, p, 8000)).tolist())
        # every kept token has non-negligible mass here, so all of them are drawn
        assert kept == set(srt[:need].tolist()), (trial, p)


def test_padding_columns_are_never_drawn():
    z = np.zeros((1, 16), np.float32)
    z[0, 12:] = 50.0  # huge logits in the padding columns 12..15
    ids = draws(z[0], 12, 1.0, 0, 1.0, 300)
    assert ids.max() < 12


def test_edge_cases():
    """One-token vocabulary; all logits equal (the tie order decides the
    nucleus); a tiny top-p keeps only the most probable token; u at the ends."""
    z1 = np.array([[3.0]], np.float32)
    for T, k, p in ((0.0, 0, 1.0), (1.0, 0, 0.5), (0.7, 5, 1.0)):
        assert oracle.sample(z1, 1, T, k, p, [0.99])[0] == 0
    V = 10
    flat = np.zeros((1, V), np.float32)
    # equal probabilities: ids enter the order smallest first, so top-p = 0.25
    # keeps ids 0, 1, 2 (3 x 0.1 >= 0.25) and the draw is uniform over them
    ids = draws(flat[0], V, 1.0, 0, 0.25, 3000)
    assert set(np.unique(ids).tolist()) == {0, 1, 2}
    np.testing.assert_allclose(np.bincount(ids, minlength=3)[:3] / 3000, [1 / 3] * 3, atol=2e-3)
    # top-k on equal logits keeps the k smallest ids
    assert set(np.unique(draws(flat[0], V, 1.0, 4, 1.0, 2000)).tolist()) == {0, 1, 2, 3}
    rng = np.random.default_rng(4)
    z = rng.normal(size=(3, 200)).astype(np.float32)
    np.testing.assert_array_equal(oracle.sample(z, 200, 1.0, 0, 1e-6, [0.5, 0.9, 0.0]),
                                  np.argmax(z, axis=1))
    # u = 0 gives the smallest kept id, u just below 1 the largest
    lo = oracle.sample(z, 200, 1.0, 10, 1.0, np.zeros(3))
    hi = oracle.sample(z, 200, 1.0, 10, 1.0, np.full(3, np.nextafter(np.float32(1), np.float32(0))))
    top10 = np.argsort(-z, axis=1)[:, :10]
    np.testing.assert_array_equal(lo, top10.min(axis=1))
    np.testing.assert_array_equal(hi, top10.max(axis=1))


def test_weights_are_exact_integers():
    """The weights of the draw are rint(p * 2^36): their sum is exact in
    float64 for any vocabulary up to 2^16 ids, so cumulative comparisons do not
    depend on the order of summation."""
    rng = np.random.default_rng(5)
    z = (rng.normal(size=50257) * 4).astype(np.float32)
    p = np.exp(z - z.max()).astype(np.float32)
    w = np.rint(p.astype(np.float64) * oracle.SAMPLE_WEIGHT_SCALE).astype(np.int64)
    assert w.max() == 2 ** 36 and w.sum() < 2 ** 53
    perm = rng.permutation(w.size)
    assert float(np.cumsum(w)[-1]) == float(np.cumsum(w[perm])[-1])
