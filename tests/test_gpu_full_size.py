"""GPU parity at full layer sizes, in the launch configurations the benchmark times, on
sampled rows the CPU reference computes one by one.

The device runs the whole layer (prologue, then GEMM); the reference recomputes the
prologue (smoothing, quantization, down projection) and the GEMM for a sample of token
rows spread over every 256-row tile row, with all output columns (every column tile).
Codes and scales must match bit for bit, Z within one bf16 ulp (plus the fp32 summation
slack), Y within relative Frobenius 1e-3 of bf16(Y64) computed on the reference's own Z
(and, as a check that isolates the GEMM, on the device's Z).

Layers: the DiT MLP-up, fused QKV and MLP-down projections (4608 tokens) and the largest
point of the batch sweep (16384 tokens, 3072 -> 12288), plus rank and LoRA points of the
sweep at small batch compared on every row.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
from bit_w4a4_quantized_group_b200 import binding as B
from bit_w4a4_quantized_group_b200 import build as BUILD
from bit_w4a4_quantized_group_b200 import inputs as I
from bit_w4a4_quantized_group_b200.layer import W4A4LowRankLinear

from gpu_helpers import assert_y_elementwise, check_device_error, dev_bf16, host_bf16, rel_fro, y_elementwise_slack
from layouts import bf16_ulp, codes_canonical, scales_canonical

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    BUILD.build()
    B.load()


def _factors(cfg, layer, rng):
    """Residual and branch factors of the layer's shapes.  The kernels do not depend on
    how they were obtained; a LoRA point concatenates a rank-16 adapter onto the base
    branch with the reference's own concatenation (eq.(13))."""
    R = (rng.standard_normal((cfg.n, cfg.m)) * cfg.sigma_w).astype(np.float32)
    r0 = cfg.rank - cfg.lora_rank
    L1 = O.bf16_rn(rng.standard_normal((cfg.m, r0)) * 0.05)          # [K, r0] (Y = X W orientation)
    L2 = O.bf16_rn(rng.standard_normal((r0, cfg.n)) * 0.05)          # [r0, N]
    lam = O.smoothing_factors(layer.X, layer.W).astype(np.float32)
    if cfg.lora_rank:
        L1, L2 = O.lora_concat(L1, L2, lam, layer.lora_A, layer.lora_B)
        L1, L2 = O.bf16_rn(L1), O.bf16_rn(L2)
    return lam, R, np.ascontiguousarray(L1.T, np.float32), np.ascontiguousarray(L2.T, np.float32)


def _run_and_check(cfg, fmt, rows=None, seed=4242):
    layer = I.make_layer(cfg)
    rng = np.random.default_rng(seed)
    lam, R, L1, L2 = _factors(cfg, layer, rng)
    M, K, N, r = cfg.b, cfg.m, cfg.n, cfg.rank
    gx = O.pow2_global_scale(float(np.max(np.abs(O.smooth_activations(layer.X, lam))))) if fmt == "nvfp4" else 1.0
    pk = B.pack_weight_np(fmt, R, L1 if r else None, L2 if r else None, gx)
    lin = W4A4LowRankLinear(fmt, N, K, pk, lam, gx, layer.bias, device="cuda")
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.forward(dev_bf16(layer.X), Y)
    check_device_error()
    if rows is None:
        rows = np.arange(M)
    ws = lin.workspace(M)
    codes = codes_canonical(fmt, ws["a_codes"].cpu().numpy(), M, K)[rows]
    scales = scales_canonical(fmt, ws["a_scales"].cpu().numpy(), M, K)[rows]
    Yall = host_bf16(Y)
    assert np.all(np.isfinite(Yall))
    Yg = Yall[rows]

    packed = O.pack_weight(fmt, R, L1, L2, gx)
    pro = O.prologue(fmt, layer.X[rows], lam, gx, packed["L1_bf16"])
    np.testing.assert_array_equal(codes, pro["q"]["codes"])
    np.testing.assert_array_equal(scales, pro["q"]["scale_bits"])
    if r:
        Zg = host_bf16(ws["Z"])[rows]
        S = np.abs(pro["xhat"].astype(np.float64)) @ np.abs(packed["L1_bf16"].astype(np.float64)).T
        assert np.all(np.abs(Zg.astype(np.float64) - pro["Z"]) <= bf16_ulp(pro["Z"]) + 2.0 ** -16 * S)
    else:
        Zg = None
    ref = O.gemm_forward(pro["q"], gx, packed["q"], packed["gscale"], Zg, packed["L2_bf16"] if r else None,
                         layer.bias)
    own = O.gemm_forward(pro["q"], gx, packed["q"], packed["gscale"], pro["Z"] if r else None,
                         packed["L2_bf16"] if r else None, layer.bias)
    assert rel_fro(Yg, own["Y"]) <= 1e-3          # the reference's own Z
    assert rel_fro(Yg, ref["Y"]) <= 1e-3          # the device's Z (isolates the GEMM)
    assert rel_fro(Yg, ref["Y64"]) <= 4e-3
    assert_y_elementwise(Yg, ref["Y64"], y_elementwise_slack(pro["q"], gx, packed["q"], packed["gscale"], Zg,
                                                             packed["L2_bf16"] if r else None, layer.bias))


def _sample_rows(M, seed):
    rng = np.random.default_rng(seed)
    tiles = M // 256
    rows = set([0, 1, 127, 128, 255, 256, M - 1])
    rows.update(int(t * 256 + o) for t, o in zip(range(tiles), rng.integers(0, 256, tiles)))
    rows.update(int(v) for v in rng.choice(M, 24, replace=False))
    return np.array(sorted(rows))


@pytest.mark.parametrize("name,fmt", [("mlp_up", "nvfp4"), ("mlp_up", "int4"), ("mlp_up", "mxfp4"), ("qkv", "nvfp4"),
                                      ("mlp_down", "nvfp4"), ("mlp_down", "int4"), ("mlp_down", "mxfp4")])
def test_full_size_layer_sampled_rows(name, fmt):
    cfg = I.NAMED[name]
    _run_and_check(cfg, fmt, _sample_rows(cfg.b, 7))


@pytest.mark.parametrize("name", ["mlp_up", "mlp_down", "qkv"])
def test_full_size_w8a8_rank16_sampled_rows(name):
    """The 8-bit setting (per-token activations, per-channel weights, rank 16) at full size."""
    cfg = dataclasses.replace(I.NAMED[name], rank=16)
    _run_and_check(cfg, "w8a8", _sample_rows(cfg.b, 8))


def test_sweep_largest_batch_sampled_rows():
    cfg = [c for c in I.sweep_configs() if c.b == 16384 and c.n == 12288 and c.rank == 32][0]
    _run_and_check(cfg, "nvfp4", _sample_rows(cfg.b, 9))


@pytest.mark.parametrize("rank", [0, 16, 32, 48, 64, 128])
def test_sweep_small_batch_all_rows(rank):
    """b = 256, 3072 x 3072: every row; rank 48 is the rank-16 LoRA on the rank-32 branch."""
    cfg = [c for c in I.sweep_configs() if c.b == 256 and c.n == 3072 and c.rank == rank][0]
    _run_and_check(cfg, "nvfp4")
