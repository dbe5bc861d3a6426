"""Stream training replayed from a CUDA graph (gpt2_stream_begin / _steps /
_end) against the same steps issued one call at a time.

Every kernel of the step is deterministic, so after the same optimizer steps
on the same windows (cut from a device stream at a device cursor, gradient
accumulation over micro-batches, a per-step learning rate) the parameters, the
gradients and the AdamW step count must be bit-identical.  A window past the
end of the stream must not be read: its update is skipped and reported.
"""
import numpy as np
import pytest

import synth
from tests.parity_util import RAGGED, TINY, gpu_model, inputs

pytestmark = pytest.mark.gpu

HP = dict(beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, max_norm=1.0)


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available()
    return torch


def eager_steps(gm, stream, bt, accum, lrs, start=0, shape=TINY):
    off = start
    for lr in lrs:
        gm.zero_grad()
        for _ in range(accum):
            x, y = gm.batch_from_stream(stream, off, shape.B, shape.T)
            gm.forward_loss(x, y, loss=False)
            gm.backward(1.0 / accum)
            off += bt
        gm.clip_adamw_step(lr=lr, **HP)
    gm.synchronize()
    return off


# TINY has head size 16 (CUDA-core attention); RAGGED head size 64, so in bf16
# the tcgen05 attention kernels, with the kept score gradients and the qkv bias
# column sums, are recorded into the graph
@pytest.mark.parametrize("shape", [TINY, RAGGED], ids=["tiny", "ragged"])
@pytest.mark.parametrize("bf16", [False, True], ids=["fp32", "bf16"])
def test_graph_steps_equal_eager_steps(bf16, shape, torch):
    om, named, _, _, _ = inputs(shape)
    bt, accum, lrs = shape.B * shape.T, 2, [6e-4, 3e-4, 1e-4]
    s_np = synth.uniform_stream(5, accum * len(lrs) * bt + 1, shape.vocab_size)
    stream = torch.from_numpy(s_np.astype(np.uint16).view(np.int16)).cuda()
    ge, gg = gpu_model(shape, bf16), gpu_model(shape, bf16)
    ge.set_params(named)
    gg.set_params(named)
    import decoder_only_lm_b200 as g
    end = eager_steps(ge, stream, bt, accum, lrs, shape=shape)
    n0 = g.launch_count()
    gg.stream_begin(stream, 0, bt, shape.B, shape.T, accum=accum, **HP)
    recorded = g.launch_count() - n0
    # every kernel issued while recording is in the graph (the bf16 weight
    # mirror is refreshed once before recording)
    assert gg.stream_kernels() == recorded - (1 if bf16 else 0) and gg.stream_kernels() > 50
    gg.stream_steps(lrs)
    assert gg.stream_end() == end
    assert gg.step == ge.step == len(lrs)
    for n, _ in om.shapes():
        for which in (0, 1):  # parameters, gradients
            assert np.array_equal(gg.get_tensor(n, which=which), ge.get_tensor(n, which=which)), n


def test_window_past_the_stream_is_refused(torch):
    import decoder_only_lm_b200 as g
    om, named, _, _, _ = inputs(TINY)
    bt = TINY.B * TINY.T
    s_np = synth.uniform_stream(6, 2 * bt + 1, TINY.vocab_size)  # two windows
    stream = torch.from_numpy(s_np.astype(np.uint16).view(np.int16)).cuda()
    ge, gg = gpu_model(TINY, True), gpu_model(TINY, True)
    ge.set_params(named)
    gg.set_params(named)
    eager_steps(ge, stream, bt, 1, [6e-4, 6e-4])
    gg.stream_begin(stream, 0, bt, TINY.B, TINY.T, accum=1, **HP)
    gg.stream_steps([6e-4, 6e-4, 6e-4])  # the third window does not fit
    with pytest.raises(g.GPT2Error) as e:
        gg.stream_end()
    assert e.value.code == g.ERR_ARG
    assert gg.step == 2  # the third update was skipped
    for n, _ in om.shapes():
        assert np.array_equal(gg.get_tensor(n), ge.get_tensor(n)), n
