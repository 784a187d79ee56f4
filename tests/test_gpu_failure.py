"""Failure path on the GPU without a fault: a bounded wait that is made to run out.

The self-test kernel waits on a barrier nothing arrives at, with the same bounded wait
every kernel uses; it must record its site in the device error word and return, and the
context must stay usable for the next call.
"""
import numpy as np
import pytest
import torch

import oracle as O
from bit_w4a4_quantized_group_b200 import binding as B
from bit_w4a4_quantized_group_b200 import build as BUILD
from bit_w4a4_quantized_group_b200 import inputs as I

from gpu_helpers import run_prologue

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    BUILD.build()
    B.load()


def test_bounded_wait_times_out_and_the_context_survives():
    torch.cuda.synchronize()
    assert B.svdq_get_last_device_error(None) == (B.SVDQ_OK, 0)
    assert B.svdq_selftest_bounded_wait(2_000_000, None) == B.SVDQ_OK      # 2 ms limit
    st, site = B.svdq_get_last_device_error(None)
    assert (st, site) == (B.SVDQ_ERR_TIMEOUT, 90)
    # the word was cleared on read
    assert B.svdq_get_last_device_error(None) == (B.SVDQ_OK, 0)
    # and the next real call runs and is exact
    cfg = I.LayerConfig(name="t", b=64, m=256, n=256, rank=16, seed=3, outlier_count=2)
    layer = I.make_layer(cfg)
    rng = np.random.default_rng(1)
    L1 = O.bf16_rn(rng.standard_normal((16, 256)) * 0.05)
    got = run_prologue("nvfp4", layer.X, None, 1.0, L1)
    ref = O.prologue("nvfp4", layer.X, None, 1.0, L1)
    np.testing.assert_array_equal(got["codes"], ref["q"]["codes"])
