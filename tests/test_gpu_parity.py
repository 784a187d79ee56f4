"""GPU parity: the CUDA path (through the C ABI) against the CPU reference.

Bars (from the header contract and the reference's readings):
  * codes and scales: bit exact, including the zero padding rows;
  * Z: within one bf16 ulp of bf16(fp64 X_hat L1^T), plus the fp32
    accumulation slack 2^-16 * sum_k |x_hat_k L1_jk|;
  * Y: relative Frobenius error <= 1e-3 against bf16(Y64), Y64 being the fp64
    reference on the same quantized operands, with the reference's own Z wherever the
    device ran the whole layer (and, as a second check that isolates the GEMM, with the
    device's Z).
"""
import numpy as np
import pytest
import torch

import oracle as O
from bit_w4a4_quantized_group_b200 import binding as B
from bit_w4a4_quantized_group_b200 import build as BUILD
from bit_w4a4_quantized_group_b200 import inputs as I

from gpu_helpers import (assert_y_elementwise, codes_bytes, encode_scales, host_bf16, rel_fro, run_gemm,
                         run_prologue, y_elementwise_slack)
from layouts import bf16_ulp

pytestmark = pytest.mark.gpu

Y_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    BUILD.build()
    B.load()


def _layer(M, K, N, rank, seed, fmt, outliers=4):
    cfg = I.LayerConfig(name="t", b=M, m=K, n=N, rank=rank, seed=seed, outlier_count=outliers,
                        outlier_mult=30.0, spike_rank=4, spike_sigma=1.5)
    layer = I.make_layer(cfg)
    prep = O.prepare_layer(fmt, layer.X, layer.W, rank)
    return layer, prep


def _check_z(Zg, xh, L1_rk, Zref):
    if L1_rk is None or L1_rk.shape[0] == 0:
        return
    S = np.abs(xh.astype(np.float64)) @ np.abs(L1_rk.astype(np.float64)).T
    err = np.abs(Zg.astype(np.float64) - Zref.astype(np.float64))
    tol = bf16_ulp(Zref) + 2.0 ** -16 * S
    assert np.all(err <= tol), f"Z max excess {np.max(err - tol)}"
    # most elements round identically
    assert np.mean(Zg == Zref) > 0.99


def _check_prologue(fmt, X, lam, gx, L1_rk):
    got = run_prologue(fmt, X, lam, gx, L1_rk)
    ref = O.prologue(fmt, X, lam, gx, L1_rk)
    np.testing.assert_array_equal(got["codes"], ref["q"]["codes"])
    np.testing.assert_array_equal(got["scales"], ref["q"]["scale_bits"])
    assert np.all(got["scale_padding"] == 0)
    _check_z(got["Z"], ref["xhat"], L1_rk, ref["Z"])
    return got, ref


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
@pytest.mark.parametrize("M,K,rank", [(300, 640, 32), (128, 256, 16), (1, 128, 0), (257, 1024, 48),
                                      (96, 512, 128), (256, 3072, 32), (100, 2048, 16), (64, 1280, 128),
                                      (64, 2048, 0), (200, 3072, 0), (64, 3584, 16), (256, 12288, 32)])
def test_prologue_parity(fmt, M, K, rank):
    layer, prep = _layer(M, K, 256, rank, seed=7 + M + rank, fmt=fmt)
    _check_prologue(fmt, layer.X, prep["lam"], prep["act_gscale"], prep["L1_rk"] if rank else None)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
def test_prologue_without_smoothing_and_zero_rows(fmt):
    rng = np.random.default_rng(5)
    X = I.to_bf16(rng.standard_normal((200, 384)) * 3)
    X[7] = 0.0                      # an all-zero row: zero scales, zero codes
    X[9, 64:128] = 0.0              # a zero group
    gx = O.pow2_global_scale(np.abs(X).max()) if fmt == "nvfp4" else 1.0
    L1 = I.to_bf16(rng.standard_normal((16, 384)) * 0.05).astype(np.float64)
    _check_prologue(fmt, X, None, gx, L1)


def test_prologue_rounding_ties_nvfp4():
    """Values on E2M1 rounding midpoints (scale exactly 1) and small negatives (-0 code)."""
    M, K = 128, 128
    X = np.zeros((M, K), np.float32)
    X[:, 0] = 6.0
    vals = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -2.5, -5.0, -0.125, 0.125,
                     -0.0078125, 4.5], np.float32)
    X[:, 1:16] = vals
    X[:, 16] = -6.0
    X[:, 17:32] = -vals
    X = I.to_bf16(X)
    got, ref = _check_prologue("nvfp4", X, None, 1.0, None)
    assert got["codes"][0, 1] == 0 and got["codes"][0, 2] == 2 and got["codes"][0, 8] == 8


def test_prologue_rounding_mxfp4_scales_ties_and_saturation():
    """MXFP4: E8M0 byte from the group absmax exponent (including a zero group and a
    subnormal-range group), E2M1 midpoints after the exact power-of-two scaling, and the
    clamp of values in (6 X, 8 X) to 6."""
    M, K = 128, 256
    X = np.zeros((M, K), np.float32)
    X[:, 0] = 7.0                                      # amax 7: X = 1, 7 -> 6
    X[:, 1:9] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25]
    X[:, 32] = 6.0 * 2.0 ** -20                        # second group: X = 2^-20
    X[:, 33] = 2.5 * 2.0 ** -20
    X[:, 64:96] = 0.0                                  # zero group: byte 0
    X[:, 96] = 2.0 ** -127                             # tiny group: byte 0, code 0
    X[:, 128] = -3.0 * 2.0 ** 30
    X[:, 129] = 0.75 * 2.0 ** 30
    X = I.to_bf16(X)
    _check_prologue("mxfp4", X, None, 1.0, None)


def test_prologue_rounding_w8a8_rows():
    """W8A8 per-token rows: max 127 (s = 1) with midpoints that round to even, a row whose
    maximum sits in the last K stage, a zero row (s = 0, zero codes), a row small enough that
    the divide takes the power-of-two prescale (s < 2^-64), a subnormal-scale row and a row
    near the bf16 maximum; K spans several stages and M leaves padding rows."""
    M, K = 200, 1280
    X = np.zeros((M, K), np.float32)
    X[:, 0] = 127.0
    X[:, 1:9] = [0.5, 1.5, 2.5, -0.5, -126.5, 63.5, 0.49609375, -3.5]
    X[1, 0] = 1.0
    X[1, K - 1] = -300.0                                 # the row maximum in the last stage
    X[2:6] = 0.0                                         # zero row (2); rows 3-5 start empty
    X[3, :4] = [2.0 ** -70, -3.0 * 2.0 ** -72, 2.0 ** -80, 0.0]   # s < 2^-64
    X[4, :3] = [2.0 ** -125, -2.0 ** -127, 2.0 ** -133]            # subnormal scale
    X[5, :3] = [3.0e38, -1.0e38, 1.0]
    rng = np.random.default_rng(41)
    X[6:] = rng.standard_normal((M - 6, K)) * np.exp2(rng.integers(-8, 8, (M - 6, 1)))
    X = I.to_bf16(X)
    got, ref = _check_prologue("w8a8", X, None, 1.0, None)
    assert list(got["codes"][0, :9].view(np.int8)) == [127, 0, 2, 2, 0, -126, 64, 0, -4]
    assert got["scales"][2, 0] == 0 and np.all(got["codes"][2] == 0)


def test_prologue_rounding_ties_int4():
    M, K = 128, 128
    X = np.zeros((M, K), np.float32)
    X[:, 0] = 7.0
    X[:, 1:9] = [0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, -6.5]
    X = I.to_bf16(X)
    _check_prologue("int4", X, None, 1.0, None)


def _gemm_case(fmt, M, N, K, rank, seed, with_bias=True, y_offset=0):
    layer, prep = _layer(M, K, N, rank, seed=seed, fmt=fmt)
    gx = prep["act_gscale"]
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], gx)
    pro = O.prologue(fmt, layer.X, prep["lam"], gx, packed["L1_bf16"] if rank else None)
    bias = layer.bias if with_bias else None
    ref = O.gemm_forward(pro["q"], gx, packed["q"], packed["gscale"], pro["Z"], packed["L2_bf16"], bias)
    Y = run_gemm(fmt, M, N, K, rank,
                 codes_bytes(fmt, pro["q"]["codes"]), encode_scales(fmt, pro["q"]["scale_bits"], M, K), gx,
                 codes_bytes(fmt, packed["q"]["codes"]), encode_scales(fmt, packed["q"]["scale_bits"], N, K),
                 packed["gscale"], pro["Z"], packed["L2_scaled"], bias, y_offset=y_offset)
    Yg = host_bf16(Y)
    assert np.all(np.isfinite(Yg))
    e_ref = rel_fro(Yg, ref["Y"])
    e_64 = rel_fro(Yg, ref["Y64"])
    assert e_ref <= Y_TOL, (e_ref, e_64)
    assert e_64 <= 4e-3
    assert_y_elementwise(Yg, ref["Y64"], y_elementwise_slack(pro["q"], gx, packed["q"], packed["gscale"], pro["Z"],
                                                             packed["L2_bf16"], bias))
    return Yg, ref


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
@pytest.mark.parametrize("M,N,K,rank", [(300, 640, 640, 32), (256, 512, 512, 16), (128, 256, 256, 0),
                                        (200, 384, 384, 48), (129, 256, 1024, 128), (64, 768, 256, 64),
                                        (130, 256, 128, 16), (1, 128, 128, 0), (257, 128, 384, 32)])
def test_gemm_parity(fmt, M, N, K, rank):
    _gemm_case(fmt, M, N, K, rank, seed=11 + M + N + rank)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
@pytest.mark.parametrize("M,N,K,rank", [(2304, 3072, 512, 32), (2560, 2560, 256, 0), (2304, 3072, 256, 128),
                                        (1300, 3072, 768, 16)])
def test_gemm_parity_many_tiles_per_cta(fmt, M, N, K, rank):
    """More output tiles than resident CTAs (clusters), so each persistent CTA drains several
    accumulators; short K (one to three pipeline steps per tile) and a two-step branch."""
    _gemm_case(fmt, M, N, K, rank, seed=5 + M + K + rank)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("M,N,K,rank", [(200, 384, 3072, 32), (256, 512, 2048, 0), (1, 256, 1024, 128),
                                        (129, 768, 6144, 16)])
def test_gemm_parity_few_tiles(fmt, M, N, K, rank):
    """Few tiles with long K (one to three tiles on the whole GPU): ragged M, a half tile past
    N, rank 0 and a long branch."""
    _gemm_case(fmt, M, N, K, rank, seed=29 + M + K + rank)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
def test_gemm_parity_y_not_32_byte_aligned(fmt):
    """Y 16-byte but not 32-byte aligned: the FP4 epilogue falls back from 32-byte to
    16-byte stores (and a ragged M keeps the row guard in play)."""
    _gemm_case(fmt, 300, 640, 512, 32, seed=23, y_offset=8)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
def test_gemm_parity_no_bias(fmt):
    _gemm_case(fmt, 160, 512, 512, 32, seed=3, with_bias=False)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
def test_gemm_lowrank_branch_is_added(fmt):
    """Y(r) - Y(r=0 on the same 4-bit operands) equals Z L2 (the branch really lands in Y)."""
    M, N, K, rank = 128, 256, 256, 32
    layer, prep = _layer(M, K, N, rank, seed=19, fmt=fmt)
    gx = prep["act_gscale"]
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], gx)
    pro = O.prologue(fmt, layer.X, prep["lam"], gx, packed["L1_bf16"])
    args = (codes_bytes(fmt, pro["q"]["codes"]), encode_scales(fmt, pro["q"]["scale_bits"], M, K), gx,
            codes_bytes(fmt, packed["q"]["codes"]), encode_scales(fmt, packed["q"]["scale_bits"], N, K),
            packed["gscale"])
    Y1 = host_bf16(run_gemm(fmt, M, N, K, rank, *args, pro["Z"], packed["L2_scaled"], None)).astype(np.float64)
    Y0 = host_bf16(run_gemm(fmt, M, N, K, 0, *args, None, None, None)).astype(np.float64)
    branch = pro["Z"].astype(np.float64) @ packed["L2_bf16"].astype(np.float64).T
    assert rel_fro(Y1 - Y0, branch) < 2e-2


@pytest.mark.parametrize("fmt,rank", [("nvfp4", 32), ("nvfp4", 0), ("nvfp4", 128), ("int4", 32), ("int4", 0),
                                      ("int4", 128), ("mxfp4", 32), ("mxfp4", 0), ("mxfp4", 128),
                                      ("w8a8", 16), ("w8a8", 0), ("w8a8", 128)])
def test_layer_end_to_end_small(fmt, rank):
    """Prologue then GEMM on the device (Z never leaves the GPU) vs the reference layer."""
    M, K, N = 384, 768, 768
    layer, prep = _layer(M, K, N, rank, seed=23 + rank, fmt=fmt)
    gx = prep["act_gscale"]
    pk = B.pack_weight_np(fmt, prep["R_nk"].astype(np.float32), prep["L1_rk"].astype(np.float32) if rank else None,
                          prep["L2_nr"].astype(np.float32) if rank else None, gx)
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], gx)
    L1 = packed["L1_bf16"] if rank else None
    got = run_prologue(fmt, layer.X, prep["lam"], gx, L1)
    L2s_dev = None
    if rank:
        L2s_dev = torch.from_numpy(pk["L2_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    Y = run_gemm(fmt, M, N, K, rank, got["dev"]["codes"], got["dev"]["scales"], gx,
                 pk["w_codes"], pk["w_scales"], pk["w_gscale"], got["dev"]["Z"], L2s_dev, layer.bias)
    ref = O.layer_forward(fmt, layer.X, prep["lam"], gx, packed, layer.bias)
    Yg = host_bf16(Y)
    # the bar: the reference layer with its own Z (independent of the device's Z) ...
    assert rel_fro(Yg, ref["Y"]) <= Y_TOL
    # ... and, to isolate the GEMM, the reference GEMM fed the device's Z (which may differ
    # from the reference Z by one bf16 ulp in a few elements)
    ref_gz = O.gemm_forward(ref["q"], gx, packed["q"], packed["gscale"], got["Z"], packed["L2_bf16"], layer.bias)
    assert rel_fro(Yg, ref_gz["Y"]) <= Y_TOL
    # and the layer approximates the unquantized X W + b (MXFP4's power-of-two scales clamp
    # values in (6 X, 8 X), so its plain W4A4 error, at rank 0, is the largest)
    exact = layer.X.astype(np.float64) @ layer.W + layer.bias.astype(np.float64)
    assert rel_fro(Yg, exact) < (0.25 if fmt == "mxfp4" else 0.15)


def _finite_bf16_values(lo=1e-30, hi=1e30):
    bits = np.arange(65536, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    a = np.abs(v)
    keep = np.isfinite(v) & (((a >= lo) & (a <= hi)) | (a == 0))
    return v[keep]


@pytest.mark.parametrize("run", range(4))
def test_smoothing_divide_exhaustive_over_bf16(run):
    """X_hat = bf16(fp32(x) / lambda) for every finite bf16 x (|x| in [1e-30, 1e30] or 0)
    and 16 lambdas per run, read back through Z with a 0/1 selector as L1."""
    rng = np.random.default_rng(1000 + run)
    special = np.array([1.0, 3.0, 0.1, 7.0, 1 / 3, 0.99999994, 1.0000001, 2.0 ** -7, 1.9999999, 1e-5, 1e5,
                        6.0, 0.75, 1.5, 123.456, 0.0123], np.float32)
    lams = special if run == 0 else np.exp(rng.uniform(np.log(1e-5), np.log(1e5), 16)).astype(np.float32)
    xs = _finite_bf16_values()
    M, K, r = len(xs), 128, 16
    X = np.repeat(xs[:, None], K, axis=1).astype(np.float32)
    lam = np.ones(K, np.float32)
    cols = np.arange(16) * 8 + 3
    lam[cols] = lams
    L1 = np.zeros((r, K), np.float64)
    L1[np.arange(16), cols] = 1.0
    got = run_prologue("int4", X, lam, 1.0, L1)
    want = O.smooth_activations(X[:, cols], lam[cols])
    Zg = got["Z"]
    bad = ~((Zg == want) | (np.isnan(Zg) & np.isnan(want)))
    # -0 and +0 compare equal above; check the sign bit too where it can be observed
    # (a zero comes back through the fp32 accumulator of Z as +0 whatever its sign)
    bad |= (np.signbit(Zg) != np.signbit(want)) & (want != 0)
    assert not bad.any(), f"{bad.sum()} mismatches, first x={X[np.argwhere(bad)[0][0], 0]}"


def test_tiny_layer_int4_end_to_end():
    """The tiny INT4 layer (256 x 512 x 512, rank 16, 8 outlier channels x 50) through both calls."""
    cfg = I.TINY
    layer = I.make_layer(cfg)
    fmt = "int4"
    prep = O.prepare_layer(fmt, layer.X, layer.W, cfg.rank)
    pk = B.pack_weight_np(fmt, prep["R_nk"], prep["L1_rk"].astype(np.float32), prep["L2_nr"].astype(np.float32), 1.0)
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], 1.0)
    got = _check_prologue(fmt, layer.X, prep["lam"], 1.0, packed["L1_bf16"])[0]
    L2s = torch.from_numpy(pk["L2_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    Y = run_gemm(fmt, cfg.b, cfg.n, cfg.m, cfg.rank, got["dev"]["codes"], got["dev"]["scales"], 1.0,
                 pk["w_codes"], pk["w_scales"], pk["w_gscale"], got["dev"]["Z"], L2s, layer.bias)
    ref = O.layer_forward(fmt, layer.X, prep["lam"], 1.0, packed, layer.bias)
    ref_gz = O.gemm_forward(ref["q"], 1.0, packed["q"], 1.0, got["Z"], packed["L2_bf16"], layer.bias)
    Yg = host_bf16(Y)
    assert rel_fro(Yg, ref["Y"]) <= Y_TOL          # the reference's own Z
    assert rel_fro(Yg, ref_gz["Y"]) <= Y_TOL       # the device's Z (isolates the GEMM)
    exact = layer.X.astype(np.float64) @ layer.W + layer.bias.astype(np.float64)
    assert rel_fro(Yg, exact) < 0.15


def _bf16_values_up_to(bound):
    """Every finite bf16 value v with |v| <= bound (both signs, zeros and subnormals included)."""
    bits = np.arange(65536, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    return v[np.isfinite(v) & (np.abs(v) <= bound)]


@pytest.mark.parametrize("fmt,gmax", [("nvfp4", 6.0), ("nvfp4", 6.75), ("nvfp4", 2688.0), ("mxfp4", 7.5),
                                      ("mxfp4", 6.0 * 2.0 ** -20), ("int4", 7.0), ("int4", 7.75),
                                      ("w8a8", 127.0), ("w8a8", 100.5)])
def test_prologue_codes_exhaustive_over_bf16(fmt, gmax):
    """The quantizer's input is a bf16 X_hat, so every bf16 value under a group's (or row's)
    maximum is the whole input space for that scale: each group holds the maximum in its
    first slot and a run of the sweep in the others; codes and scales must match the
    reference bit for bit (unit scales, scales with more mantissa bits, saturation)."""
    g = {"nvfp4": 16, "mxfp4": 32, "int4": 64, "w8a8": 128}[fmt]
    K = 128
    vals = _bf16_values_up_to(gmax)
    per_group = g - 1
    ngroups = -(-len(vals) // per_group)
    pad = np.zeros(ngroups * per_group, np.float32)
    pad[: len(vals)] = vals
    grp = np.concatenate([np.full((ngroups, 1), gmax, np.float32), pad.reshape(ngroups, per_group)], axis=1)
    rows = -(-ngroups // (K // g))
    allg = np.zeros((rows * (K // g), g), np.float32)
    allg[:ngroups] = grp
    X = I.to_bf16(allg.reshape(rows, K))
    assert np.array_equal(X, allg.reshape(rows, K))           # every value is already bf16
    _check_prologue(fmt, X, None, 1.0, None)


def _groups_over_bf16(g, gmax, K=128):
    """Rows of K elements cut into groups of g; each group holds gmax first and a run of
    the sweep of every finite bf16 value v with |v| <= gmax in the rest."""
    vals = _bf16_values_up_to(gmax)
    per_group = g - 1
    ngroups = -(-len(vals) // per_group)
    pad = np.zeros(ngroups * per_group, np.float32)
    pad[: len(vals)] = vals
    grp = np.concatenate([np.full((ngroups, 1), gmax, np.float32), pad.reshape(ngroups, per_group)], axis=1)
    rows = -(-ngroups // (K // g))
    allg = np.zeros((rows * (K // g), g), np.float32)
    allg[:ngroups] = grp
    X = I.to_bf16(allg.reshape(rows, K))
    assert np.array_equal(X, allg.reshape(rows, K))
    return X


@pytest.mark.parametrize("gx_exp,gmax", [(-4, 4096.0), (-8, 30720.0), (0, 2816.0), (0, 2704.0),
                                         (3, 0.25), (6, 4.0), (3, 0.0234375), (0, 2.0 ** -11)])
def test_prologue_nvfp4_tensor_scale_saturation_and_subnormal_scales(gx_exp, gmax):
    """NVFP4 with an activation tensor scale g_x that does not fit the groups (Note §2.2
    and §8: E4M3 group scales; the tensor scale is a static power of two from calibration):
      * g_x too small for the data (a / 6 / g_x > 448): the E4M3 scale saturates at 448 and
        the codes of the large elements clamp at +-6;
      * g_x too large: the group scales land in E4M3's subnormal range (below 2^-6), or
        round to zero, which makes every code of the group 0.
    Every bf16 value under the group maximum, bit for bit against the reference."""
    gx = 2.0 ** gx_exp
    X = _groups_over_bf16(16, gmax)
    got, ref = _check_prologue("nvfp4", X, None, gx, None)
    s = got["scales"]
    t = np.float32(np.float32(gmax / 6.0) / np.float32(gx))
    if t > 448:
        assert np.all(s[:, 0] == 0x7E)                  # E4M3 448 (saturated)
        assert np.any(got["codes"] == 0x7) and np.any(got["codes"] == 0xF)
    elif t >= 2.0 ** -10 and t < 2.0 ** -6:
        assert np.all(s[:, 0] < 0x08) and np.all(s[:, 0] > 0)   # subnormal E4M3 scales
    elif t < 2.0 ** -10:
        assert np.all(s == 0) and np.all(got["codes"] == 0)


@pytest.mark.parametrize("shift", [-3, 11, 14])
def test_layer_nvfp4_tensor_scale_from_other_calibration(shift):
    """The whole NVFP4 layer when g_x comes from a calibration batch whose amax differs from
    the quantized batch by 2^shift: with shift < 0 the outlier groups saturate their E4M3
    scales (and codes clamp at +-6, about 3% of the groups at shift -3); with shift > 0 the
    groups get subnormal scales (and, at shift 14, some zero scales).  Codes and scales bit for bit; Y against the reference layer with its own Z."""
    M, K, N, rank = 384, 768, 768, 32
    layer, prep = _layer(M, K, N, rank, seed=31 + shift, fmt="nvfp4")
    xh = O.smooth_activations(layer.X, prep["lam"])
    gx = O.pow2_global_scale(float(np.abs(xh).max()) * 2.0 ** shift)
    t = (np.abs(xh).reshape(M, K // 16, 16).max(axis=2) / 6.0) / gx
    if shift < 0:
        assert np.any(t > 448) and np.any(t <= 448)
    else:
        assert np.any((t >= 2.0 ** -10) & (t < 2.0 ** -6))
    pk = B.pack_weight_np("nvfp4", prep["R_nk"].astype(np.float32), prep["L1_rk"].astype(np.float32),
                          prep["L2_nr"].astype(np.float32), gx)
    packed = O.pack_weight("nvfp4", prep["R_nk"], prep["L1_rk"], prep["L2_nr"], gx)
    got, pro = _check_prologue("nvfp4", layer.X, prep["lam"], gx, packed["L1_bf16"])
    if shift < 0:
        assert np.any(got["scales"] == 0x7E)
    L2s = torch.from_numpy(pk["L2_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    Y = run_gemm("nvfp4", M, N, K, rank, got["dev"]["codes"], got["dev"]["scales"], gx,
                 pk["w_codes"], pk["w_scales"], pk["w_gscale"], got["dev"]["Z"], L2s, layer.bias)
    Yg = host_bf16(Y)
    ref = O.layer_forward("nvfp4", layer.X, prep["lam"], gx, packed, layer.bias)
    assert rel_fro(Yg, ref["Y"]) <= Y_TOL
    assert_y_elementwise(Yg, ref["Y64"], y_elementwise_slack(ref["q"], gx, packed["q"], packed["gscale"], got["Z"],
                                                             packed["L2_bf16"], layer.bias))


@pytest.mark.parametrize("case", range(16))
def test_layer_random_shapes(case):
    """Seeded random shapes (ragged M, any multiple of 128 for N and K, every rank step) in
    every format, through both calls; the same bars as the fixed cases."""
    rng = np.random.default_rng(9000 + case)
    fmt = ["nvfp4", "int4", "mxfp4", "w8a8"][case % 4]
    M = int(rng.integers(1, 700))
    N = 128 * int(rng.integers(1, 9))
    K = 128 * int(rng.integers(1, 11))
    rank = 16 * int(rng.integers(0, 9))
    layer, prep = _layer(M, K, N, rank, seed=9100 + case, fmt=fmt, outliers=min(4, K // 64))
    gx = prep["act_gscale"]
    pk = B.pack_weight_np(fmt, prep["R_nk"].astype(np.float32), prep["L1_rk"].astype(np.float32) if rank else None,
                          prep["L2_nr"].astype(np.float32) if rank else None, gx)
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], gx)
    got, ref = _check_prologue(fmt, layer.X, prep["lam"], gx, packed["L1_bf16"] if rank else None)
    L2s_dev = torch.from_numpy(pk["L2_bf16"].view(np.int16)).cuda().view(torch.bfloat16) if rank else None
    Y = run_gemm(fmt, M, N, K, rank, got["dev"]["codes"], got["dev"]["scales"], gx,
                 pk["w_codes"], pk["w_scales"], pk["w_gscale"], got["dev"]["Z"], L2s_dev, layer.bias)
    Yg = host_bf16(Y)
    out = O.gemm_forward(ref["q"], gx, packed["q"], packed["gscale"], got["Z"] if rank else None,
                         packed["L2_bf16"] if rank else None, layer.bias)
    own = O.gemm_forward(ref["q"], gx, packed["q"], packed["gscale"], ref["Z"] if rank else None,
                         packed["L2_bf16"] if rank else None, layer.bias)
    assert rel_fro(Yg, own["Y"]) <= Y_TOL          # the reference's own Z
    assert rel_fro(Yg, out["Y"]) <= Y_TOL          # the device's Z (isolates the GEMM)
    assert_y_elementwise(Yg, out["Y64"], y_elementwise_slack(ref["q"], gx, packed["q"], packed["gscale"],
                                                             got["Z"] if rank else None,
                                                             packed["L2_bf16"] if rank else None, layer.bias))


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
@pytest.mark.parametrize("M,K,N,rank", [(256, 3072, 3072, 32), (1024, 3072, 1024, 64), (40, 2048, 512, 16),
                                        (256, 12288, 512, 32)])
def test_layer_small_batch_k_split(fmt, M, K, N, rank):
    """Small batches, where the prologue splits each row block's K stages over a cluster of
    CTAs and adds their Z partials through distributed shared memory (W8A8: after taking each
    row's maximum over the cluster); the whole layer against the reference."""
    layer, prep = _layer(M, K, N, rank, seed=77 + M + rank, fmt=fmt)
    gx = prep["act_gscale"]
    pk = B.pack_weight_np(fmt, prep["R_nk"].astype(np.float32), prep["L1_rk"].astype(np.float32),
                          prep["L2_nr"].astype(np.float32), gx)
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], gx)
    got, ref = _check_prologue(fmt, layer.X, prep["lam"], gx, packed["L1_bf16"])
    L2s_dev = torch.from_numpy(pk["L2_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    Y = run_gemm(fmt, M, N, K, rank, got["dev"]["codes"], got["dev"]["scales"], gx,
                 pk["w_codes"], pk["w_scales"], pk["w_gscale"], got["dev"]["Z"], L2s_dev, layer.bias)
    out = O.gemm_forward(ref["q"], gx, packed["q"], packed["gscale"], got["Z"], packed["L2_bf16"], layer.bias)
    own = O.gemm_forward(ref["q"], gx, packed["q"], packed["gscale"], ref["Z"], packed["L2_bf16"], layer.bias)
    assert rel_fro(host_bf16(Y), own["Y"]) <= Y_TOL    # the reference's own Z
    assert rel_fro(host_bf16(Y), out["Y"]) <= Y_TOL    # the device's Z (isolates the GEMM)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
@pytest.mark.parametrize("M,K,N,rank", [(300, 1280, 640, 32), (2304, 768, 3072, 16), (40, 2048, 512, 64)])
def test_repeated_calls_are_bit_identical(fmt, M, K, N, rank):
    """Every call is deterministic: the same inputs give the same codes, scales, Z and Y bits
    on repeated calls (fixed summation orders in every reduction, including the small-batch
    K split of the prologue and the persistent GEMM schedules)."""
    layer, prep = _layer(M, K, N, rank, seed=4000 + M + rank, fmt=fmt)
    gx = prep["act_gscale"]
    pk = B.pack_weight_np(fmt, prep["R_nk"].astype(np.float32), prep["L1_rk"].astype(np.float32),
                          prep["L2_nr"].astype(np.float32), gx)
    packed = O.pack_weight(fmt, prep["R_nk"], prep["L1_rk"], prep["L2_nr"], gx)
    L2s = torch.from_numpy(pk["L2_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    runs = []
    for i in range(3):
        got = run_prologue(fmt, layer.X, prep["lam"], gx, packed["L1_bf16"], fill=0x11 * (i + 1))
        Y = run_gemm(fmt, M, N, K, rank, got["dev"]["codes"], got["dev"]["scales"], gx,
                     pk["w_codes"], pk["w_scales"], pk["w_gscale"], got["dev"]["Z"], L2s, layer.bias)
        runs.append((got["codes"], got["scales"], got["Z"].view(np.uint32), Y.view(torch.int16).cpu().numpy()))
    for a, b in zip(runs[0], runs[1]):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(runs[0], runs[2]):
        np.testing.assert_array_equal(a, b)
