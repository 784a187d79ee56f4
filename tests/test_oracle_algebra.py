"""Pins of the CPU reference's layer algebra (no GPU).

Identities and bounds from "SVDQuant 阅读笔记" (eq.(3), (4), (6), (7), (8),
(10), (11), (12), (13)) and the two-path reconstruction of "msModelSlim
SVDQuant" ("前向等价关系"), plus brute force on tiny shapes.
"""
import math

import numpy as np
import pytest

import oracle as O
from bit_w4a4_quantized_group_b200 import inputs as I


@pytest.fixture(scope="module")
def tiny():
    return I.make_layer(I.TINY)


def _small_cfg(**kw):
    base = dict(name="t", b=64, m=256, n=192, rank=16, seed=11, outlier_count=4,
                outlier_mult=30.0, spike_rank=3, spike_sigma=2.0)
    base.update(kw)
    return I.LayerConfig(**base)


# --------------------------------------------------------------- smoothing

def test_smoothing_factor_eq4_by_hand():
    X = np.array([[1.0, -4.0, 0.0], [2.0, 0.5, 0.0]])
    W = np.array([[0.5, -2.0], [1.0, 0.25], [3.0, 1.0]])
    lam = O.smoothing_factors(X, W, alpha=0.5)
    # max|X| = [2, 4, 0], max|W| = [2, 1, 3]: sqrt(2)/sqrt(2), sqrt(4)/sqrt(1), guard -> 1
    assert np.allclose(lam, [1.0, 2.0, 1.0])
    lam_a = O.smoothing_factors(X, W, alpha=0.25)
    assert np.isclose(lam_a[1], 4 ** 0.25 / 1 ** 0.75)
    assert np.isclose(lam_a[0], 2 ** 0.25 / 2 ** 0.75)


def test_smoothing_keeps_xw_eq3(tiny):
    lam = O.smoothing_factors(tiny.X, tiny.W)
    X = tiny.X.astype(np.float64)
    lam64 = lam.astype(np.float64)
    Xt = X / lam64[None, :]
    Wt = O.smooth_weight(tiny.W, lam)
    ref = X @ tiny.W
    assert np.linalg.norm(Xt @ Wt - ref) <= 1e-13 * np.linalg.norm(ref)
    # the smoothed activations have a much smaller range on the outlier channels
    ch = tiny.outlier_channels
    assert np.abs(Xt[:, ch]).max() < 0.5 * np.abs(X[:, ch]).max()


def test_lambda_one_is_identity(tiny):
    ones = np.ones(tiny.cfg.m, np.float32)
    xh = O.smooth_activations(tiny.X, ones)
    assert np.array_equal(xh, O.bf16_rn(tiny.X))
    assert np.array_equal(xh, tiny.X)        # X is already bf16
    assert np.array_equal(O.smooth_weight(tiny.W, ones), tiny.W)


# --------------------------------------------------------------- SVD split

def test_svd_split_reconstructs_and_eckart_young(tiny):
    lam = O.smoothing_factors(tiny.X, tiny.W)
    Wt = O.smooth_weight(tiny.W, lam)
    for r in (0, 4, 16, 32):
        sp = O.svd_split(Wt, r)
        # msModelSlim "前向等价关系": L1 L2 + R = W_tilde (fp64 residual)
        rec = sp["L1_bf16"] @ sp["L2_bf16"] + sp["R64"]
        assert np.linalg.norm(rec - Wt) <= 1e-14 * np.linalg.norm(Wt)
        # fp32 storage of R only adds its own rounding
        rec32 = sp["L1_bf16"] @ sp["L2_bf16"] + sp["R"].astype(np.float64)
        assert np.linalg.norm(rec32 - Wt) <= 2 ** -23 * np.linalg.norm(sp["R64"]) * 2
        # eq.(10): ||R||_F^2 = sum_{i>r} sigma_i^2 with exact fp64 factors
        tail = np.sum(sp["sigma"][r:] ** 2)
        assert abs(np.linalg.norm(sp["R_exact"]) ** 2 - tail) <= 1e-10 * max(tail, 1e-30)
        # the bf16 factors can only add energy on top of the optimum
        assert np.linalg.norm(sp["R64"]) ** 2 >= tail * (1 - 1e-12)


def test_spike_is_recovered_without_smoothing():
    cfg = I.TINY
    layer = I.make_layer(cfg)
    s = np.linalg.svd(layer.W, compute_uv=False)
    edge = cfg.sigma_w * (math.sqrt(cfg.m) + math.sqrt(cfg.n))
    assert np.all(np.abs(s[:4] - 2.5) < 0.25)
    assert s[4] < 1.2 * edge
    sp = O.svd_split(layer.W, 4)
    assert np.allclose(sp["sigma"][:4], s[:4])


def test_svd_orientation_matches_modelslim_shapes(tiny):
    prep = O.prepare_layer("int4", tiny.X, tiny.W, 16)
    K, N = tiny.cfg.m, tiny.cfg.n
    assert prep["R_nk"].shape == (N, K)
    assert prep["L1_rk"].shape == (16, K)     # l1 = V^T  [rank, in]
    assert prep["L2_nr"].shape == (N, 16)     # l2 = U S  [out, rank]
    Wt = prep["W_tilde"]
    rec = prep["L2_nr"] @ prep["L1_rk"] + prep["R_nk"].astype(np.float64)   # [N, K] = W_tilde^T
    assert np.linalg.norm(rec - Wt.T) <= 1e-6 * np.linalg.norm(Wt)


# --------------------------------------------------------------- branch algebra

def test_cancellation_eq8(tiny):
    fmt = "int4"
    lam = O.smoothing_factors(tiny.X, tiny.W)
    Xt = tiny.X.astype(np.float64) / lam.astype(np.float64)[None, :]
    Wt = O.smooth_weight(tiny.W, lam)
    sp = O.svd_split(Wt, 16)
    L1, L2, R = sp["L1"], sp["L2"], sp["R_exact"]
    QX = O.dequantize(fmt, O.quantize(fmt, O.bf16_rn(Xt)))
    QR = O.dequantize(fmt, O.quantize(fmt, R.T.astype(np.float32))).T
    Yhat = (Xt @ L1) @ L2 + QX @ QR                              # eq.(7)
    lhs = Xt @ Wt - Yhat
    rhs = Xt @ R - QX @ QR                                       # eq.(8)
    assert np.linalg.norm(lhs - rhs) <= 1e-12 * np.linalg.norm(Xt @ Wt)


def test_prop41_bound_eq6(tiny):
    for fmt in ("int4", "nvfp4", "mxfp4"):
        lam = O.smoothing_factors(tiny.X, tiny.W)
        xh = O.smooth_activations(tiny.X, lam)
        Wt = O.smooth_weight(tiny.W, lam).astype(np.float32)
        gx = O.pow2_global_scale(np.abs(xh).max()) if fmt == "nvfp4" else 1.0
        gw = O.pow2_global_scale(np.abs(Wt).max()) if fmt == "nvfp4" else 1.0
        QX = O.dequantize(fmt, O.quantize(fmt, xh, gx))
        QW = O.dequantize(fmt, O.quantize(fmt, Wt.T, gw)).T
        lhs, mid, rhs = O.prop41_bound(xh, Wt, QX, QW)
        assert lhs <= mid * (1 + 1e-12) and mid <= rhs * (1 + 1e-12)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "w8a8"])
def test_low_rank_branch_reduces_error(fmt, tiny):
    """The paper's central claim on a spike + outlier layer: W4A4 with the branch
    beats plain W4A4 on the same smoothed layer, and both beat no smoothing."""
    X = tiny.X.astype(np.float64)
    ref = X @ tiny.W
    prep = O.prepare_layer(fmt, tiny.X, tiny.W, 16)
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], prep["act_gscale"])
    out = O.layer_forward(fmt, tiny.X, prep["lam"], prep["act_gscale"], packed)
    err_svdq = np.linalg.norm(out["Y64"] - ref)
    prep0 = O.prepare_layer(fmt, tiny.X, tiny.W, 0)
    packed0 = O.pack_weight(fmt, prep0["R_nk"], prep0["L1_rk"], prep0["L2_nr"], prep0["act_gscale"])
    out0 = O.layer_forward(fmt, tiny.X, prep0["lam"], prep0["act_gscale"], packed0)
    err_plain = np.linalg.norm(out0["Y64"] - ref)
    assert err_svdq < 0.7 * err_plain
    assert err_svdq / np.linalg.norm(ref) < 0.2


def test_rank0_is_plain_w4a4(tiny):
    fmt = "nvfp4"
    prep = O.prepare_layer(fmt, tiny.X, tiny.W, 0)
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], prep["act_gscale"])
    out = O.layer_forward(fmt, tiny.X, prep["lam"], prep["act_gscale"], packed, tiny.bias)
    # with r = 0 the residual is W_tilde itself (rounded to fp32)
    assert np.array_equal(prep["R_nk"], prep["W_tilde"].T.astype(np.float32))
    QX = O.dequantize(fmt, out["q"])
    QW = O.dequantize(fmt, packed["q"])
    plain = QX @ QW.T + tiny.bias.astype(np.float64)[None, :]
    assert np.allclose(out["Y64"], plain, rtol=0, atol=1e-12 * np.abs(plain).max())


def test_lora_concatenation_eq13():
    cfg = _small_cfg(rank=24, lora_rank=8)
    layer = I.make_layer(cfg)
    lam = O.smoothing_factors(layer.X, layer.W)
    Xt = layer.X.astype(np.float64) / lam.astype(np.float64)[None, :]
    sp = O.svd_split(O.smooth_weight(layer.W, lam), 16)
    L1c, L2c = O.lora_concat(sp["L1"], sp["L2"], lam, layer.lora_A, layer.lora_B)
    assert L1c.shape == (cfg.m, 24) and L2c.shape == (24, cfg.n)
    base = Xt @ sp["L1"] @ sp["L2"]
    adapted = Xt @ L1c @ L2c
    want = base + layer.X.astype(np.float64) @ layer.lora_A @ layer.lora_B
    assert np.linalg.norm(adapted - want) <= 1e-12 * np.linalg.norm(want)
    # without the D in front of A the adapter is not reproduced
    L1w, L2w = O.lora_concat(sp["L1"], sp["L2"], None, layer.lora_A, layer.lora_B)
    assert np.linalg.norm(Xt @ L1w @ L2w - want) > 1e-3 * np.linalg.norm(want)


# --------------------------------------------------------------- counting formulas

def test_counting_formulas_eq11_eq12(golden):
    gd = golden("counting_formulas.txt")
    m, n, r = int(gd["m"]), int(gd["n"]), int(gd["r"])
    assert O.rho_mac(m, n, r) * 100 == gd["rho_mac_percent"]
    assert O.rho_bytes(m, n, r) * 100 == gd["rho_bytes_percent"]
    assert round(1 / O.rho_bytes(m, n, r), 2) == gd["compression_approx"]
    # eq.(11) from its definition: (bmr + brn) / bmn at any b
    b = 4608
    assert math.isclose((b * m * r + b * r * n) / (b * m * n), O.rho_mac(m, n, r))


# --------------------------------------------------------------- quantized GEMM

@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "w8a8"])
def test_quantized_gemm_matches_triple_loop(fmt):
    rng = np.random.default_rng(21)
    M, N, K = 6, 5, 128
    xa = O.bf16_rn(rng.standard_normal((M, K)))
    wb = O.bf16_rn(rng.standard_normal((N, K)) * 0.02)
    gx = O.pow2_global_scale(np.abs(xa).max()) if fmt == "nvfp4" else 1.0
    gw = O.pow2_global_scale(np.abs(wb).max()) if fmt == "nvfp4" else 1.0
    qa, qw = O.quantize(fmt, xa, gx), O.quantize(fmt, wb, gw)
    fast = O.w4a4_main(qa, qw)
    slow = O.brute_force_w4a4(fmt, qa, qw)
    # 4-bit products are exact in fp64; W8A8's fp32 scales times 8-bit codes are not, so
    # the bound there is relative to the sum of magnitudes (summation order differs)
    S = np.abs(O.dequantize(fmt, qa)) @ np.abs(O.dequantize(fmt, qw)).T / (gx * gw)
    atol = 1e-14 * S if fmt == "w8a8" else 0
    assert np.all(np.abs(fast - slow) <= 1e-15 * np.abs(slow) + atol)
    # Q(X) Q(W)^T from the dequantized operands equals g_x g_w times the same sum
    deq = O.dequantize(fmt, qa) @ O.dequantize(fmt, qw).T
    assert np.all(np.abs(deq - gx * gw * fast) <= 1e-15 * np.abs(deq) + gx * gw * atol)


def test_pack_weight_l2_prescale_is_exact(tiny):
    prep = O.prepare_layer("nvfp4", tiny.X, tiny.W, 16)
    packed = O.pack_weight("nvfp4", prep["R_nk"], prep["L1_rk"], prep["L2_nr"], prep["act_gscale"])
    f = prep["act_gscale"] * packed["gscale"]
    assert math.log2(f) == int(math.log2(f))
    assert np.array_equal(packed["L2_scaled"].astype(np.float64) * f, packed["L2_bf16"])


def test_planted_transposed_factor_is_caught(tiny):
    """Using L2 with rows and columns swapped (a transposed operand) must break the
    msModelSlim reconstruction pin."""
    prep = O.prepare_layer("int4", tiny.X, tiny.W, 16)
    Wt = prep["W_tilde"]
    bad = prep["L1_rk"].T @ prep["L2_nr"][: prep["L1_rk"].shape[0], :16]
    assert bad.shape != Wt.shape or np.linalg.norm(bad - Wt) > 1e-3
    good = (prep["L2_nr"] @ prep["L1_rk"]).T + prep["R_nk"].T.astype(np.float64)
    assert np.linalg.norm(good - Wt) <= 1e-6 * np.linalg.norm(Wt)


def test_planted_wrong_smoothing_side_is_caught(tiny):
    """The typo W diag(lambda) (scaling output columns) does not preserve XW."""
    lam = O.smoothing_factors(tiny.X, tiny.W).astype(np.float64)
    X = tiny.X.astype(np.float64)
    wrong = (X / lam[None, :]) @ (tiny.W * lam[: tiny.W.shape[1]][None, :])
    assert np.linalg.norm(wrong - X @ tiny.W) > 1e-2 * np.linalg.norm(X @ tiny.W)
