"""GPU parity at the full DiT MLP-up size (4608 x 3072 x 12288, rank 32), in the launch
configuration the benchmark times, on sampled rows the CPU reference computes one by one.

The device runs the whole layer; the reference recomputes the prologue (smoothing,
quantization, down projection) and the GEMM for a sample of token rows spread over
every 256-row tile row, with all 12288 output columns (every column tile).  Codes and
scales must match bit for bit, Z within one bf16 ulp, Y within relative Frobenius 1e-3
of bf16(Y64) computed on the device's Z.
"""
import numpy as np
import pytest
import torch

import oracle as O
from bit_w4a4_quantized_group_b200 import binding as B
from bit_w4a4_quantized_group_b200 import build as BUILD
from bit_w4a4_quantized_group_b200 import inputs as I
from bit_w4a4_quantized_group_b200.layer import W4A4LowRankLinear

from gpu_helpers import check_device_error, dev_bf16, host_bf16, rel_fro
from layouts import bf16_ulp, scales_canonical, unpack_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mlp_up():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    BUILD.build()
    B.load()
    cfg = I.NAMED["mlp_up"]
    layer = I.make_layer(cfg)
    lam = O.smoothing_factors(layer.X, layer.W).astype(np.float32)
    xh_max = float(np.max(np.abs(O.smooth_activations(layer.X, lam))))
    # residual and branch factors of the layer's shapes (the GEMM does not depend on how
    # they were obtained); bf16-exact factors as the pack expects
    rng = np.random.default_rng(4242)
    R = (rng.standard_normal((cfg.n, cfg.m)) * cfg.sigma_w).astype(np.float32)
    L1 = O.bf16_rn(rng.standard_normal((cfg.rank, cfg.m)) * 0.05).astype(np.float32)
    L2 = O.bf16_rn(rng.standard_normal((cfg.n, cfg.rank)) * 0.05).astype(np.float32)
    rows = sorted(set([0, 1, 127, 128, 255, 256, cfg.b - 1] + [t * 256 + int(o) for t, o in
                      zip(range(cfg.b // 256), rng.integers(0, 256, cfg.b // 256))] +
                      [int(v) for v in rng.choice(cfg.b, 24, replace=False)]))
    return {"cfg": cfg, "layer": layer, "lam": lam, "xh_max": xh_max, "R": R, "L1": L1, "L2": L2,
            "rows": np.array(rows)}


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_full_size_layer_sampled_rows(mlp_up, fmt):
    d = mlp_up
    cfg, layer, rows = d["cfg"], d["layer"], d["rows"]
    M, K, N, r = cfg.b, cfg.m, cfg.n, cfg.rank
    gx = O.pow2_global_scale(d["xh_max"]) if fmt == "nvfp4" else 1.0
    pk = B.pack_weight_np(fmt, d["R"], d["L1"], d["L2"], gx)
    lin = W4A4LowRankLinear(fmt, N, K, pk, d["lam"], gx, layer.bias, device="cuda")
    X = dev_bf16(layer.X)
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.forward(X, Y)
    check_device_error()
    ws = lin.workspace(M)
    codes = unpack_codes(ws["a_codes"].cpu().numpy(), M, K)[rows]
    scales = scales_canonical(fmt, ws["a_scales"].cpu().numpy(), M, K)[rows]
    Zg = host_bf16(ws["Z"])[rows]
    Yall = host_bf16(Y)
    assert np.all(np.isfinite(Yall))
    Yg = Yall[rows]

    packed = O.pack_weight(fmt, d["R"], d["L1"], d["L2"], gx)
    pro = O.prologue(fmt, layer.X[rows], d["lam"], gx, packed["L1_bf16"])
    np.testing.assert_array_equal(codes, pro["q"]["codes"])
    np.testing.assert_array_equal(scales, pro["q"]["scale_bits"])
    S = np.abs(pro["xhat"].astype(np.float64)) @ np.abs(packed["L1_bf16"].astype(np.float64)).T
    assert np.all(np.abs(Zg.astype(np.float64) - pro["Z"]) <= bf16_ulp(pro["Z"]) + 2.0 ** -16 * S)
    ref = O.gemm_forward(pro["q"], gx, packed["q"], packed["gscale"], Zg, packed["L2_bf16"], layer.bias)
    assert rel_fro(Yg, ref["Y"]) <= 1e-3
    assert rel_fro(Yg, ref["Y64"]) <= 4e-3
