"""The offline split on the GPU: residual iteration with cuSOLVER's fp64 SVD and the
deployment quantize-dequantize in PyTorch CUDA ops, against the CPU reference.

AutoRound "SVDQuant（实验性功能）", "Residual iteration".  The quantize-dequantize
must equal the weight pack's bit for bit on the device too (its E4M3 scale rounding
is torch's CUDA float8 conversion); the iteration follows the reference to SVD
rounding; and a layer built from the iterated split runs through the C ABI with
the same parity bars as every other layer.
"""
import numpy as np
import pytest
import torch

import oracle as O
from bit_w4a4_quantized_group_b200 import binding as B
from bit_w4a4_quantized_group_b200 import build as BUILD
from bit_w4a4_quantized_group_b200 import inputs as I
from bit_w4a4_quantized_group_b200 import prepare as P
from bit_w4a4_quantized_group_b200.layer import W4A4LowRankLinear

from gpu_helpers import assert_y_elementwise, check_device_error, dev_bf16, host_bf16, rel_fro, y_elementwise_slack
from layouts import codes_canonical, scales_canonical
from test_residual_iteration import FMTS, _deployed_qdq, _qdq_cases

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    BUILD.build()
    B.load()


@pytest.mark.parametrize("fmt", FMTS)
def test_cuda_qdq_is_the_pack_quantizer_bit_for_bit(fmt):
    for R in _qdq_cases(fmt):
        if fmt == "int4":
            R = np.where(np.abs(R) > 1e30, np.float32(1e4), R)
        want = _deployed_qdq(fmt, R.T.astype(np.float64)).T
        got = P.qdq_weight(fmt, torch.from_numpy(R).cuda()).cpu().numpy()
        assert np.array_equal(np.signbit(got), np.signbit(want))
        assert np.array_equal(got, want), np.abs(got - want).max()


@pytest.mark.parametrize("fmt", FMTS)
def test_cuda_iteration_follows_the_reference(fmt):
    layer = I.make_layer(I.TINY)
    lam = O.smoothing_factors(layer.X, layer.W)
    Wt = O.smooth_weight(layer.W, lam)
    Xh = O.smooth_activations(layer.X, lam)
    ref = O.residual_iteration(fmt, Wt, 16, 3, early_stop=True, X_hat=Xh)
    L1, L2, R, chosen, errs = P.residual_iteration(fmt, torch.from_numpy(Wt).cuda(), 16, 3, True,
                                                   torch.from_numpy(Xh.astype(np.float64)).cuda())
    assert chosen == ref["chosen"] and len(errs) == len(ref["errors"])
    assert np.allclose(errs, ref["errors"], rtol=2e-4)
    assert torch.equal(R, (torch.from_numpy(Wt).cuda() - L1 @ L2).to(torch.float32))


@pytest.mark.parametrize("fmt", FMTS)
def test_layer_from_iterated_split_runs_at_parity(fmt):
    cfg = I.LayerConfig(name="ri", b=512, m=1024, n=768, rank=32, seed=31, outlier_count=10,
                        outlier_mult=30.0, spike_rank=6, spike_sigma=2.0)
    layer = I.make_layer(cfg)
    prep = P.prepare(fmt, layer.X, layer.W, cfg.rank, device="cuda", residual_iters=4, early_stop=True)
    res = prep["residual"]
    assert res["errors"][res["chosen"]] <= res["errors"][0]
    pk = P.pack(fmt, prep)
    M, K, N, r = cfg.b, cfg.m, cfg.n, cfg.rank
    gx = prep["act_gscale"]
    lin = W4A4LowRankLinear(fmt, N, K, pk, prep["lam"], gx, layer.bias, device="cuda")
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.forward(dev_bf16(layer.X), Y)
    check_device_error()
    ws = lin.workspace(M)
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], gx)
    pro = O.prologue(fmt, layer.X, prep["lam"], gx, packed["L1_bf16"])
    np.testing.assert_array_equal(codes_canonical(fmt, ws["a_codes"].cpu().numpy(), M, K), pro["q"]["codes"])
    np.testing.assert_array_equal(scales_canonical(fmt, ws["a_scales"].cpu().numpy(), M, K), pro["q"]["scale_bits"])
    Zg = host_bf16(ws["Z"])
    Yg = host_bf16(Y)
    ref = O.gemm_forward(pro["q"], gx, packed["q"], packed["gscale"], Zg, packed["L2_bf16"], layer.bias)
    assert rel_fro(Yg, ref["Y"]) <= 1e-3
    assert_y_elementwise(Yg, ref["Y64"], y_elementwise_slack(pro["q"], gx, packed["q"], packed["gscale"], Zg,
                                                             packed["L2_bf16"], layer.bias))
    # the iterated weights reconstruct the layer output at least as well as the plain split
    plain = P.prepare(fmt, layer.X, layer.W, cfg.rank, device="cuda")
    Xh = O.smooth_activations(layer.X, prep["lam"]).astype(np.float64)
    Wt = prep["lam"].astype(np.float64)[:, None] * layer.W.astype(np.float64)

    def out_err(p):
        q = O.pack_weight(fmt, p["R_nk"], p["L1_rk"], p["L2_nr"], gx)
        W_hat = q["L1_bf16"].astype(np.float64).T @ q["L2_bf16"].astype(np.float64).T + O.dequantize(fmt, q["q"]).T
        return np.linalg.norm(Xh @ (W_hat - Wt))
    assert out_err(prep) <= out_err(plain) * (1 + 1e-6)
