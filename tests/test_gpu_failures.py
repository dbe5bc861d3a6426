"""Failure handling on the device without a fault: a bounded wait that runs
out reports a timeout through the error word, the kernel ends, and the
context stays usable (no trap, no hang, nothing injected into the GPU)."""
import time

import numpy as np
import pytest

from tests.parity_util import TINY, gpu_model, inputs

pytestmark = pytest.mark.gpu


def test_unmet_wait_gives_up_and_is_reported():
    import torch

    import decoder_only_lm_b200 as g
    assert torch.cuda.is_available()
    assert g.device_error() == 0
    t0 = time.time()
    assert g.wait_selfcheck()
    took = time.time() - t0
    assert 1.5 < took < 30, took  # the 2 s budget of a device wait
    assert g.device_error() == 0  # the record was cleared
    # the device and the library still work: one step against its own repeat
    om, named, stream, x, y = inputs(TINY)
    gm = gpu_model(TINY, True)
    gm.set_params(named)
    a = gm.forward_loss(x, y)
    b = gm.forward_loss(x, y)
    assert np.isfinite(a) and a == b
    gm.close()
