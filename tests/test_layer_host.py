"""Host-side checks of the layer object (no GPU): the smoothing factors it accepts and the
rounding of the bias to bf16."""
import numpy as np
import pytest
import torch

from bit_w4a4_quantized_group_b200.layer import W4A4LowRankLinear


def _packed(N=128, K=128, r=0):
    return {"w_codes": np.zeros(N * K // 2, np.uint8), "w_scales": np.zeros(N * K // 16, np.uint8),
            "w_gscale": 1.0, "L1_bf16": np.zeros((r, K), np.uint16), "L2_bf16": np.zeros((N, r), np.uint16)}


@pytest.mark.parametrize("bad", [0.0, -1.0, np.inf, np.nan, 1e-40])
def test_lambda_must_be_finite_normal_positive(bad):
    lam = np.ones(128, np.float32)
    lam[5] = bad
    with pytest.raises(ValueError):
        W4A4LowRankLinear("nvfp4", 128, 128, _packed(), lam, 1.0, device="cpu")


def test_lambda_shape_is_checked():
    with pytest.raises(ValueError):
        W4A4LowRankLinear("nvfp4", 128, 128, _packed(), np.ones(64, np.float32), 1.0, device="cpu")


def test_bias_rounds_to_nearest_even():
    """A bias that is not bf16-valued is rounded to nearest (ties to even), not truncated."""
    b = np.zeros(128, np.float32)
    # 1 + 2^-8 + 2^-10 lies above the midpoint between 1 and the next bf16 (1 + 2^-7)
    b[0] = 1.0 + 2.0 ** -8 + 2.0 ** -10
    b[1] = 1.0 + 2.0 ** -8                 # exact midpoint: ties to even -> 1.0
    b[2] = 1.0 + 3 * 2.0 ** -8             # midpoint between 1 + 2^-7 and 1 + 2^-6: ties to even -> 1 + 2^-6
    b[3] = -(1.0 + 2.0 ** -8 + 2.0 ** -10)
    lin = W4A4LowRankLinear("nvfp4", 128, 128, _packed(), None, 1.0, bias=b, device="cpu")
    got = lin.bias.to(torch.float32).numpy()
    assert got[0] == 1.0 + 2.0 ** -7
    assert got[1] == 1.0
    assert got[2] == 1.0 + 2.0 ** -6
    assert got[3] == -(1.0 + 2.0 ** -7)
    np.testing.assert_array_equal(got[4:], 0.0)
