"""The bucket reports of the data-parallel exchange on one GPU.

gpt2_backward reports each gradient bucket as soon as the last work writing
it has been enqueued.  Here the "exchange" copies each bucket on a side
stream at the moment it is reported (behind an event on the model's stream,
as the NCCL exchange does); after the backward has finished, every copy must
equal the final gradient bit for bit, so no bucket is reported before its
writers are done.  The buckets must arrive in order 0 .. L, once each, and not
at all while a step is being recorded as a graph.
"""
import numpy as np
import pytest

import synth
from tests.parity_util import RAGGED, gpu_model, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available()
    return torch


@pytest.mark.parametrize("bf16", [True, False], ids=["bf16", "fp32"])
def test_buckets_are_final_when_reported(torch, bf16):
    import decoder_only_lm_b200 as g
    from decoder_only_lm_b200.dp import CudaGradExchange
    om, named, stream, x, y = inputs(RAGGED)
    gm = gpu_model(RAGGED, bf16)
    gm.set_params(named)
    snaps, order = {}, []

    def copy(view):  # runs on the side stream, behind the report's event
        snaps.setdefault(order[-1], []).append(view.clone())

    ex = CudaGradExchange(gm, copy)
    seen = ex.ready

    def ready(b):
        order.append(b)
        seen(b)

    ex.ready = ready
    gm.zero_grad()
    gm.forward_loss(torch.from_numpy(x).cuda(), torch.from_numpy(y).cuda(), loss=False)
    ex.arm()
    gm.backward()
    ex.finish()
    torch.cuda.synchronize()
    L = RAGGED.n_layer
    assert order == list(range(L + 1))
    grad = gm.arena(g.GRAD)
    for b in order:
        ranges = ex.ranges[b]
        assert len(snaps[b]) == len(ranges)
        for (off, cnt), got in zip(ranges, snaps[b]):
            assert torch.equal(got, grad[off:off + cnt]), (b, off)
    # cleared: a second backward reports nothing
    order.clear()
    gm.forward_loss(torch.from_numpy(x).cuda(), torch.from_numpy(y).cuda(), loss=False)
    gm.backward()
    gm.synchronize()
    assert order == []
    gm.close()


def test_no_reports_while_a_step_is_recorded(torch):
    from tests.parity_util import TINY
    om, named, stream, x, y = inputs(TINY)
    gm = gpu_model(TINY, True)
    gm.set_params(named)
    seen = []
    gm.set_bucket_callback(seen.append)
    s = synth.uniform_stream(1, 8 * TINY.B * TINY.T + 1, TINY.vocab_size)
    ds = torch.from_numpy(s.astype(np.int16).view(np.int16)).cuda()
    gm.stream_begin(ds, 0, TINY.B * TINY.T, TINY.B, TINY.T)
    gm.stream_steps([6e-4])
    gm.stream_end()
    assert seen == []
    gm.forward_loss(x, y, loss=False)
    gm.backward()
    gm.synchronize()
    assert seen == list(range(TINY.n_layer + 1))
    gm.set_bucket_callback(None)
    gm.close()


def test_library_exchange_one_rank_is_exact(torch):
    """gpt2_dp_init over one rank (NCCL): every bucket's all-reduce (average)
    is an identity, so the exchanging backward, and steps recorded as a graph
    with the exchange inside, must give bit for bit what the same calls give
    without it; and dp_sync(0) must leave the exchange out."""
    import decoder_only_lm_b200 as g
    om, named, stream, x, y = inputs(RAGGED)
    xs, ys = torch.from_numpy(x).cuda(), torch.from_numpy(y).cuda()

    def grads(model):
        model.zero_grad()
        model.forward_loss(xs, ys, loss=False)
        model.backward()
        model.synchronize()
        return model.arena(g.GRAD).clone()

    ref = gpu_model(RAGGED, True)
    ref.set_params(named)
    gm = gpu_model(RAGGED, True)
    gm.set_params(named)
    gm.dp_init(g.dp_unique_id(), 0, 1)
    assert torch.equal(grads(gm), grads(ref))
    gm.dp_sync(False)
    assert torch.equal(grads(gm), grads(ref))
    gm.dp_sync(True)
    # two optimizer steps of two micro-batches each, replayed from the graph
    bt = RAGGED.B * RAGGED.T
    s = synth.uniform_stream(7, 6 * bt + 1, RAGGED.vocab_size)
    ds = torch.from_numpy(s.astype(np.int16).view(np.int16)).cuda()
    for m in (ref, gm):
        m.stream_begin(ds, 0, bt, RAGGED.B, RAGGED.T, accum=2)
        m.stream_steps([6e-4, 5e-4])
        assert m.stream_end() == 4 * bt
    for name in ("wte", "h.0.attn.qkv.w", "h.1.mlp.proj.b", "lnf.w"):
        assert np.array_equal(gm.get_tensor(name), ref.get_tensor(name)), name
    assert gm.step == ref.step == 2
    gm.close()
    ref.close()
