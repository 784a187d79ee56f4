"""Pins of the CPU reference's number formats and quantizers (no GPU).

Each test checks the reference against something other than itself: a
library cast (ml_dtypes, torch), a worked example printed on the pages, a
closed-form bound, or brute force over every code.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O


def _fp32_sweep(lo_exp, hi_exp, per_binade=4096, seed=0):
    """Dense fp32 sample: every binade in [2**lo_exp, 2**hi_exp) at ``per_binade`` points
    plus random bit patterns, both signs."""
    rng = np.random.default_rng(seed)
    vals = []
    for e in range(lo_exp, hi_exp):
        frac = np.arange(per_binade) / per_binade
        vals.append((1.0 + frac) * 2.0 ** e)
    v = np.concatenate(vals).astype(np.float32)
    bits = rng.integers(0, 2 ** 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    r = bits.view(np.float32)
    r = r[np.isfinite(r)]
    r = r[(np.abs(r) >= 2.0 ** lo_exp) & (np.abs(r) < 2.0 ** hi_exp)]
    v = np.concatenate([v, r, -v])
    return v.astype(np.float32)


# --------------------------------------------------------------------- bf16 / fp16

def test_bf16_rn_matches_ml_dtypes_on_fp32():
    x = _fp32_sweep(-40, 40)
    # exact ties: bf16 value plus half an ulp, both parities of the kept bit
    base = np.arange(0x0080, 0x7F00, 7, dtype=np.uint32) << 16   # normal exponents only
    ties = (base | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties, np.float32([0.0, -0.0, 1.0, -1.0])])
    ours = O.bf16_rn(x)
    lib = x.astype(ml_dtypes.bfloat16).astype(np.float32)
    assert np.array_equal(ours.view(np.uint32), lib.view(np.uint32))


def test_bf16_rn_fp64_is_nearest_even():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(50_000) * np.exp2(rng.integers(-20, 20, 50_000))
    r = O.bf16_rn(x).astype(np.float64)
    # neighbours on the bf16 grid: ulp = 2**(e-7) for |x| in [2**e, 2**(e+1))
    e = np.floor(np.log2(np.abs(x)))
    ulp = np.exp2(e - 7)
    lo = np.floor(x / ulp) * ulp
    hi = lo + ulp
    d_lo, d_hi = x - lo, hi - x
    m_lo = np.rint(lo / ulp).astype(np.int64)
    want = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(m_lo % 2 == 0, lo, hi)))
    assert np.array_equal(r, want)


def test_fp16_rn_matches_torch():
    x = _fp32_sweep(-24, 16)
    ours = O.fp16_rn(x)
    lib = torch.from_numpy(x).to(torch.float16).to(torch.float32).numpy()
    assert np.array_equal(ours, lib)


# --------------------------------------------------------------------- E4M3 / E2M1

def test_e4m3_grid_is_the_format():
    v = O.E4M3_VALUES
    assert len(v) == 127 and v[0] == 0.0 and v[-1] == 448.0
    assert v[1] == 2.0 ** -9 and v[8] == 2.0 ** -6           # min subnormal, min normal
    lib = np.arange(127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(v, lib)


def test_e4m3_rounding_matches_ml_dtypes():
    x = _fp32_sweep(-12, 9)
    x = x[np.abs(x) <= 448.0]
    # every midpoint of the grid, and one fp32 ulp either side of it
    mids = ((O.E4M3_VALUES[:-1] + O.E4M3_VALUES[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9)]).astype(np.float32)
    codes, vals = O.e4m3_rn_satfinite(x)
    lib = x.astype(ml_dtypes.float8_e4m3fn)
    assert np.array_equal(codes, lib.view(np.uint8))
    assert np.array_equal(vals, lib.astype(np.float32))


def test_e4m3_saturates():
    codes, vals = O.e4m3_rn_satfinite(np.array([448.0, 460.0, 1e6, np.float32(3e38)]))
    assert np.all(vals == 448.0) and np.all(codes == 0x7E)


def test_e2m1_rounding_matches_ml_dtypes_and_ties():
    x = _fp32_sweep(-6, 3)
    x = x[np.abs(x) <= 6.0]
    mids = ((O.E2M1_VALUES[:-1] + O.E2M1_VALUES[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 9)])
    codes, vals = O.e2m1_rn_satfinite(x)
    lib = x.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)
    assert np.array_equal(vals, lib)
    # ties go to the even code (reading 3)
    t_in = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    _, t_out = O.e2m1_rn_satfinite(t_in)
    assert list(t_out) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    # saturation at 6 and the kept sign of a small negative value
    c, v = O.e2m1_rn_satfinite(np.array([7.0, -100.0, -0.1, 0.1, 0.0]))
    assert list(v) == [6.0, -6.0, 0.0, 0.0, 0.0]
    assert list(c) == [7, 15, 8, 0, 0]
    assert np.signbit(v[2])


# --------------------------------------------------------------------- INT4 g64

def _int4_group(values):
    g = np.zeros(64, np.float32)
    g[: len(values)] = values
    return g[None, :]


def test_int4_worked_example(golden):
    gd = golden("int4_rounding_example.txt")
    grp = np.array(gd["group_with_outlier"], np.float32)
    q = O.quantize_int4_g64(_int4_group(grp))
    assert q["scale"][0, 0] == gd["step_with_outlier"]
    assert list(q["q"][0, 1:len(grp)]) == gd["small_codes_with_outlier"]
    # remove the large component: the remaining range is 1, the step is 1/7
    small = grp.copy()
    small[0] = np.float32(gd["remaining_range"])
    q2 = O.quantize_int4_g64(_int4_group(small))
    s = float(q2["scale"][0, 0])
    assert abs(s - gd["step_without_outlier"]) <= 2.0 ** -14   # one fp16 half-ulp at 1/7
    # with step 1/7 every one of the small elements gets a nonzero code
    assert np.count_nonzero(q2["q"][0, 1:len(grp)]) == len(grp) - 1


def test_int4_codes_are_argmin_over_all_codes():
    rng = np.random.default_rng(3)
    x = O.bf16_rn(rng.standard_normal((64, 256)) * np.exp2(rng.integers(-6, 6, (64, 1))))
    q = O.quantize_int4_g64(x)
    s = np.repeat(q["scale"], 64, axis=1).astype(np.float32)
    t = (x / s).astype(np.float64)
    cand = np.arange(-7, 8, dtype=np.float64)
    d = np.abs(t[..., None] - cand)
    best = d.min(axis=-1, keepdims=True)
    ties = d == best
    # among the nearest codes pick the even one (round half to even)
    even = ties & (cand % 2 == 0)
    pick = np.where(even.any(-1), cand[np.argmax(even, -1)], cand[np.argmax(ties, -1)])
    assert np.array_equal(q["q"], pick)
    assert q["q"].min() >= -7 and q["q"].max() <= 7
    assert np.array_equal(O.int4_value(q["codes"]), q["q"])


def test_int4_per_element_and_group_bound_eq9():
    rng = np.random.default_rng(4)
    x = O.bf16_rn(rng.standard_normal((32, 512)) * 0.02)
    q = O.quantize_int4_g64(x)
    s = np.repeat(q["scale"].astype(np.float64), 64, axis=1)
    err = np.abs(x - s * q["q"])
    unclamped = np.abs(x / s) <= 7.0
    assert np.all(err[unclamped] <= s[unclamped] / 2 * (1 + 1e-7))
    # eq.(9) per group with the group's own max: ||Z - Q(Z)||_F <= sqrt(N)/(2 qmax) max|Z|,
    # loosened by the fp16 rounding of the scale (relative 2**-11).
    e = (x - s * q["q"]).reshape(32, 8, 64)
    lhs = np.sqrt((e ** 2).sum(-1))
    rhs = math.sqrt(64) / (2 * 7) * np.abs(x.reshape(32, 8, 64)).max(-1) * (1 + 2.0 ** -10)
    assert np.all(lhs <= rhs)


def test_int4_zero_group_and_scale_precision():
    x = np.zeros((2, 128), np.float32)
    x[1, 64:] = 3.0
    q = O.quantize_int4_g64(x)
    assert np.all(q["q"][0] == 0) and q["scale"][0, 0] == 0
    assert q["scale"][1, 1] == O.fp16_rn(np.float32(3.0) / np.float32(7.0))
    assert np.all(q["q"][1, 64:] == 7)


# --------------------------------------------------------------------- NVFP4 g16

def test_nvfp4_scales_and_codes_are_nearest():
    rng = np.random.default_rng(5)
    x = O.bf16_rn(rng.standard_normal((48, 256)) * np.exp2(rng.integers(-8, 4, (48, 1))))
    g = O.pow2_global_scale(np.abs(x).max())
    q = O.quantize_nvfp4_g16(x, g)
    a = np.abs(x.reshape(48, 16, 16)).max(-1)
    t = ((a / np.float32(6.0)).astype(np.float32) / np.float32(g)).astype(np.float32)
    # scale = nearest E4M3 to t (brute force over the whole grid, ties to even code)
    d = np.abs(t[..., None].astype(np.float64) - O.E4M3_VALUES)
    best = d.min(-1, keepdims=True)
    ties = d == best
    even = ties & (np.arange(127) % 2 == 0)
    want = np.where(even.any(-1), np.argmax(even, -1), np.argmax(ties, -1))
    assert np.array_equal(q["scale_bits"].astype(np.int64), want)
    # codes = nearest E2M1 value of x / (s g), ties to even
    den = np.repeat((q["scale"] * np.float32(g)).astype(np.float32), 16, axis=1)
    v = (x / den).astype(np.float64)
    grid = np.concatenate([-O.E2M1_VALUES[::-1], O.E2M1_VALUES])
    dv = np.abs(np.minimum(np.abs(v), 6.0)[..., None] - O.E2M1_VALUES)
    assert np.all(np.abs(np.abs(q["q"]) - np.minimum(np.abs(v), 6.0)) <= dv.min(-1) + 1e-12)
    assert set(np.unique(q["q"])).issubset(set(grid))
    assert np.array_equal(np.sign(q["q"][q["q"] != 0]), np.sign(v[q["q"] != 0]))


def test_nvfp4_dequant_error_bound():
    rng = np.random.default_rng(6)
    x = O.bf16_rn(rng.standard_normal((16, 1024)) * 0.05)
    g = O.pow2_global_scale(np.abs(x).max())
    q = O.quantize_nvfp4_g16(x, g)
    deq = O.dequantize("nvfp4", q)
    s = np.repeat(q["scale"].astype(np.float64) * g, 16, axis=1)
    # the E2M1 grid gap is at most 2 (between 4 and 6), so half a gap times s,
    # plus the clamp when the rounded scale is below a/6
    a = np.repeat(np.abs(x.reshape(16, 64, 16)).max(-1), 16, axis=1)
    err = np.abs(x - deq)
    assert np.all(err <= s * 1.0 + np.maximum(a - 6 * s, 0) + 1e-12)


def test_pow2_global_scale():
    for amax in (1e-3, 0.02, 0.5, 3.0, 37.0, 1000.0):
        g = O.pow2_global_scale(amax)
        assert math.log2(g) == int(math.log2(g))
        assert 0.5 < amax / (6 * 448 * g) <= 1.0
    assert O.pow2_global_scale(0.0) == 1.0


# --------------------------------------------------------------------- planted mistakes

def test_planted_sign_drop_in_e2m1_is_caught(monkeypatch):
    """A quantizer that loses the sign must fail the library cross-check."""
    good = O.e2m1_rn_satfinite

    def bad(x):
        c, v = good(np.abs(x))
        return c, v
    monkeypatch.setattr(O, "e2m1_rn_satfinite", bad)
    x = np.array([-1.0, -3.0, 2.0], np.float32)
    _, v = O.e2m1_rn_satfinite(x)
    assert not np.array_equal(v, x.astype(ml_dtypes.float4_e2m1fn).astype(np.float32))


def test_planted_round_half_up_is_caught():
    """Rounding half away from zero (instead of to even) breaks the argmin pin on ties."""
    t = np.array([0.5, 1.5, 2.5, -2.5], np.float64)
    assert not np.array_equal(np.floor(t + 0.5), np.rint(t))


def test_pow2_global_scale_boundaries():
    # amax exactly 6 * 448 * 2**e must give g = 2**e (amax / (6 g) == 448 is allowed)
    for e in (-12, -3, 0, 5):
        amax = 6 * 448 * 2.0 ** e
        assert O.pow2_global_scale(amax) == 2.0 ** e
        assert O.pow2_global_scale(np.nextafter(amax, 1e30)) == 2.0 ** (e + 1)
        assert O.pow2_global_scale(np.nextafter(amax, 0)) == 2.0 ** e


# --------------------------------------------------------------------- MXFP4 g32 (reading 9)

def test_mxfp4_scale_is_the_mx_shared_exponent_and_codes_are_nearest():
    """X = 2^(floor(log2 amax) - 2) (OCP MX, E2M1 emax = 2), q = nearest E2M1 of x / X."""
    rng = np.random.default_rng(21)
    x = O.bf16_rn(rng.standard_normal((40, 256)) * np.exp2(rng.integers(-20, 12, (40, 1))))
    q = O.quantize_mxfp4_g32(x)
    a = np.abs(x.reshape(40, 8, 32)).max(-1).astype(np.float64)
    # floor(log2 a) by brute force over integer exponents: the largest e with 2^e <= a
    e = np.array([[max(k for k in range(-160, 160) if 2.0 ** k <= v) for v in row] for row in a])
    assert np.array_equal(q["scale_bits"].astype(np.int64), np.clip(e - 2, -127, 127) + 127)
    X = np.repeat(2.0 ** (q["scale_bits"].astype(np.int64) - 127), 32, axis=1)
    v = x.astype(np.float64) / X
    grid = np.concatenate([-O.E2M1_VALUES[::-1], O.E2M1_VALUES])
    dv = np.abs(np.minimum(np.abs(v), 6.0)[..., None] - O.E2M1_VALUES)
    assert np.all(np.abs(np.abs(q["q"]) - np.minimum(np.abs(v), 6.0)) <= dv.min(-1) + 1e-12)
    assert set(np.unique(q["q"])).issubset(set(grid))
    # E8M0 byte of the scale, cross-checked with ml_dtypes' float8_e8m0fnu
    if hasattr(ml_dtypes, "float8_e8m0fnu"):
        enc = np.asarray(q["scale"][:, :4], np.float32).astype(ml_dtypes.float8_e8m0fnu).view(np.uint8)
        assert np.array_equal(enc, q["scale_bits"][:, :4])


def test_mxfp4_worked_values_and_saturation():
    g = np.zeros((1, 32), np.float32)
    # amax 6 * 2^-3: X = 2^-3 and the max element is exactly 6 (code 0x7)
    g[0, 0] = 0.75
    g[0, 1] = -0.375                # -3 * 2^-3 -> code 0xD
    g[0, 2] = 0.03125               # 0.25 * 2^-3: a tie between 0 and 0.5 -> 0 (even)
    q = O.quantize_mxfp4_g32(g)
    assert q["scale_bits"][0, 0] == 127 - 3
    assert (q["codes"][0, 0], q["codes"][0, 1], q["codes"][0, 2]) == (0x7, 0xD, 0x0)
    # amax 7 * 2^-3: floor(log2) = -1 -> X = 2^-3 and 7 saturates to 6 (the MX conversion clamps)
    g[0, 0] = 0.875
    q = O.quantize_mxfp4_g32(g)
    assert q["scale_bits"][0, 0] == 127 - 3 and q["q"][0, 0] == 6.0
    # all-zero group: byte 0 (2^-127), zero codes
    q = O.quantize_mxfp4_g32(np.zeros((2, 64), np.float32))
    assert np.all(q["scale_bits"] == 0) and np.all(q["codes"] == 0)


def test_mxfp4_is_equivariant_under_powers_of_two():
    rng = np.random.default_rng(22)
    x = O.bf16_rn(rng.standard_normal((8, 128)))
    q0 = O.quantize_mxfp4_g32(x)
    for k in (-9, -1, 3, 17):
        qk = O.quantize_mxfp4_g32((x * np.float32(2.0 ** k)).astype(np.float32))
        assert np.array_equal(qk["codes"], q0["codes"])
        assert np.array_equal(qk["scale_bits"].astype(int), q0["scale_bits"].astype(int) + k)


def test_mxfp4_dequant_error_bound():
    rng = np.random.default_rng(23)
    x = O.bf16_rn(rng.standard_normal((16, 1024)) * 0.05)
    q = O.quantize_mxfp4_g32(x)
    deq = O.dequantize("mxfp4", q)
    X = np.repeat(q["scale"].astype(np.float64), 32, axis=1)
    a = np.repeat(np.abs(x.reshape(16, 32, 32)).max(-1), 32, axis=1)
    # half the largest E2M1 gap (1) times X, plus the clamp of values in (6 X, 8 X)
    assert np.all(np.abs(x - deq) <= X * 1.0 + np.maximum(a - 6 * X, 0) + 1e-12)


# ------------------------------------------------------- W8A8 per row (reading 10)

def test_int8_rowwise_worked_example_eq1_with_8_bits():
    """eq.(1) with the symmetric 8-bit range: max 127 gives step 1; max 1 gives step 1/127."""
    x = np.zeros((2, 128), np.float32)
    x[0, 0] = 127.0
    x[0, 1:6] = [0.4, -0.6, 2.5, 3.5, -126.5]        # 0.4 -> 0, ties to even: 2, 4, -126
    x[1, 0] = -1.0
    x[1, 1] = 0.5
    q = O.quantize_int8_rowwise(x)
    assert q["scale"][0, 0] == 1.0
    assert list(q["q"][0, :6]) == [127, 0, -1, 2, 4, -126]
    assert q["scale"][1, 0] == np.float32(1.0) / np.float32(127.0)
    assert q["q"][1, 0] == -127
    assert q["codes"][1, 0] == 0x81 and q["codes"][0, 0] == 0x7F and q["codes"][0, 2] == 0xFF
    # 0.5 / fp32(1/127) = 63.5 up to the fp32 rounding of the scale and of the quotient
    assert q["q"][1, 1] in (63.0, 64.0)
    assert q["q"][1, 1] == np.rint(np.float32(0.5) / q["scale"][1, 0])


def test_int8_rowwise_codes_are_nearest_and_bounded():
    """Against exact rational arithmetic: q is the nearest integer to x/s except within
    the fp32 quotient's rounding of a midpoint; |x - s q| <= s/2 up to that rounding."""
    from fractions import Fraction
    rng = np.random.default_rng(31)
    x = O.bf16_rn(rng.standard_normal((24, 256)) * np.exp2(rng.integers(-30, 30, (24, 1))))
    x[3] = 0.0
    q = O.quantize_int8_rowwise(x)
    assert np.all(q["q"][3] == 0) and q["scale"][3, 0] == 0
    for i in range(24):
        if i == 3:
            continue
        a = Fraction(float(np.abs(x[i]).max()))
        s = Fraction(float(q["scale"][i, 0]))
        assert abs(s - a / 127) <= s * Fraction(1, 2 ** 24)          # s = fp32 of amax / 127
        for k in range(0, 256, 7):
            t = Fraction(float(x[i, k])) / s
            qi = int(q["q"][i, k])
            assert -127 <= qi <= 127
            assert abs(t - qi) <= Fraction(1, 2) + abs(t) * Fraction(1, 2 ** 23)
        # the max element maps to +-127
        j = int(np.argmax(np.abs(x[i])))
        assert abs(int(q["q"][i, j])) == 127


def test_int8_rowwise_matches_torch_fp32_semantics():
    """rint(fp32(x / s)) checked against torch's IEEE fp32 divide and round-half-even."""
    import torch
    rng = np.random.default_rng(32)
    x = O.bf16_rn(rng.standard_normal((16, 512)) * np.exp2(rng.integers(-10, 10, (16, 1))))
    x[5, :4] = [127.0, 63.5, -0.5, 1.5]           # exact midpoints with s = 1
    x[5, 4:] = 0.0
    q = O.quantize_int8_rowwise(x)
    xt = torch.from_numpy(x)
    st = (xt.abs().amax(1, keepdim=True) / 127.0)
    assert np.array_equal(st.numpy(), q["scale"])
    qt = torch.clamp(torch.round(xt / st), -127, 127)
    assert np.array_equal(qt.numpy().astype(np.float64), q["q"])
    assert list(q["q"][5, :4]) == [127, 64, -0.0, 2]


def test_int8_rowwise_sign_symmetry_and_power_of_two_equivariance():
    rng = np.random.default_rng(33)
    x = O.bf16_rn(rng.standard_normal((8, 384)))
    q0 = O.quantize_int8_rowwise(x)
    qn = O.quantize_int8_rowwise(-x)
    assert np.array_equal(qn["q"], -q0["q"]) and np.array_equal(qn["scale"], q0["scale"])
    for k in (-40, -3, 5, 60):
        qk = O.quantize_int8_rowwise((x * np.float32(2.0 ** k)).astype(np.float32))
        assert np.array_equal(qk["q"], q0["q"])
        assert np.array_equal(qk["scale"], (q0["scale"] * np.float32(2.0 ** k)).astype(np.float32))


def test_int8_rowwise_dequant_is_per_row_scale_times_code():
    rng = np.random.default_rng(34)
    x = O.bf16_rn(rng.standard_normal((4, 256)))
    q = O.quantize_int8_rowwise(x)
    deq = O.dequantize("w8a8", q)
    for i in range(4):
        for k in (0, 17, 255):
            assert deq[i, k] == float(q["scale"][i, 0]) * int(np.int8(q["codes"][i, k]))
    assert np.all(np.abs(x - deq) <= q["scale"].astype(np.float64) * (0.5 + 2.0 ** -16))


def test_planted_w8a8_mistakes_are_caught(monkeypatch):
    """A 128 code range (instead of 127) or scales taken per column (a transposed operand)
    must break the eq.(1) worked example the W8A8 pins rest on."""
    x = np.zeros((2, 128), np.float32)
    x[0, 0] = 127.0
    x[0, 1:4] = [2.5, 3.5, -126.5]
    x[1, 0] = -1.0
    good = O.quantize_int8_rowwise(x)
    assert good["scale"][0, 0] == 1.0 and list(good["q"][0, :4]) == [127, 2, 4, -126]
    import oracle.svdq_oracle as OM
    monkeypatch.setattr(OM, "INT8_QMAX", 128)
    wide = O.quantize_int8_rowwise(x)
    assert wide["scale"][0, 0] != 1.0
    monkeypatch.undo()
    per_col = O.quantize_int8_rowwise(np.ascontiguousarray(x.T))
    assert per_col["scale"].shape[0] != good["scale"].shape[0] or per_col["scale"][0, 0] != 1.0
