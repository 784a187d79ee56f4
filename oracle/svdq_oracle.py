"""Plain CPU reference for the SVDQuant W4A4 + low-rank linear layer.

TEST INFRASTRUCTURE ONLY.  This module is the independent checker of the CUDA
path: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline legs may import it.  It shares no code, table or helper with the
CUDA library or its binding.

Everything is NumPy; floating point is fp64 unless a step is defined in a
narrower format (bf16 / fp16 / fp32 / E4M3 / E2M1), in which case the exact
rounding of that format is written out below.

Sources (cited by page title and section / equation):

* "SVDQuant 阅读笔记：用少量高精度计算保护 4-bit 扩散模型" (cited as
  *SVDQuant 阅读笔记*): eq.(1) symmetric INT4 round-to-nearest, §2.2 group
  sizes (INT4 g64 with 16-bit scale, NVFP4 g16 with FP8 scale), eq.(3)
  smoothing, eq.(4) smoothing factor, eq.(5)/(6) error decomposition and
  Prop. 4.1 bound, eq.(7) two-branch forward, eq.(8) cancellation, eq.(9)
  per-group RTN bound, eq.(10) truncated SVD split, eq.(11)/(12) MAC and byte
  ratios, eq.(13) LoRA concatenation, §8 (appendix D settings).
* "SVDQuant（实验性功能）" (AutoRound docs, cited as *AutoRound SVDQuant*),
  "Residual iteration": the low-rank factors are materialised in the
  low-rank dtype before the residual ``R = W - U V`` is formed.
* "SVDQuant：基于低秩残差重构的扩散模型后训练量化算法说明" (msModelSlim,
  cited as *msModelSlim SVDQuant*), "SVD 分解过程": factor shapes
  ``l1 = V^T`` [rank, in] and ``l2 = U S`` [out, rank]; "前向等价关系".

Readings where the pages are silent:

1. ``round`` in eq.(1) is round-half-to-even (``np.rint``).
2. INT4 scale: ``s = fp16_rn(fp32(a / 7))`` (saturating at 65504), and the
   codes use the stored scale: ``q = clamp(rint(fp32(x / float(s))), -7, 7)``;
   ``s == 0`` gives ``q = 0``.  Codes are -7..7.
3. NVFP4: ``s = e4m3_rn_satfinite(fp32(fp32(a / 6) / g))`` and
   ``q = e2m1_rn_satfinite(fp32(x / (float(s) * g)))`` with ties to the even
   code; the sign of ``x / (s g)`` is kept, so a small negative value gives
   code 0x8 (-0).  ``s == 0`` gives code 0.
4. ``g`` is a per-tensor power of two: ``2 ** ceil(log2(amax / (6 * 448)))``
   (1 when ``amax == 0``).  INT4 uses ``g = 1``.
5. Groups run along the reduction dimension (input features) for both
   operands.
6. Smoothing guard: lambda_i = 1 when either statistic is 0, else
   ``max(lambda_i, 1e-5)``.
7. ``X_hat = bf16_rn(fp32(X) / lambda)`` (IEEE fp32 divide, then one rounding
   to bf16); it feeds both the quantizer and the down projection.  L1, L2 and
   Z are bf16.
8. Sigma goes into L1 (eq.(10) of *SVDQuant 阅读笔记*).
9. MXFP4 (*AutoRound SVDQuant*: its Nunchaku export needs E2M1 weights and activations in
   32-element groups, quantized symmetrically): the MX shared scale of the OCP Microscaling
   format,
   ``X = 2 ** clip(floor(log2(amax)) - 2, -127, 127)`` (2 = exponent of the largest
   E2M1 value 6), stored as its E8M0 byte ``log2(X) + 127``; ``q = e2m1_rn_satfinite(x / X)``
   (the divide is exact).  ``amax == 0`` gives byte 0.  No tensor scale (g = 1).
10. W8A8 (*SVDQuant 阅读笔记* §8, the appendix-D 8-bit setting: rank 16, activations
    quantized per token and dynamically, weights per output channel): eq.(1) with the
    8-bit symmetric range, one group per row spanning all of K:
    ``s = fp32(amax / 127)``, ``q = clamp(rint(fp32(x / s)), -127, 127)``; ``s == 0``
    gives ``q = 0``.  The scale is kept in fp32 (the pages give no precision for it).
    No tensor scale (g = 1).
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

__all__ = [
    "bf16_rn", "fp16_rn", "e4m3_rn_satfinite", "e2m1_rn_satfinite",
    "E4M3_VALUES", "E2M1_VALUES", "e4m3_value", "e2m1_value", "int4_value",
    "smoothing_factors", "smooth_activations", "smooth_weight", "svd_split",
    "lora_concat", "pow2_global_scale", "quantize_int4_g64", "quantize_nvfp4_g16",
    "dequantize", "quantize", "prologue", "pack_weight", "w4a4_main", "gemm_forward",
    "layer_forward", "prepare_layer", "rho_mac", "rho_bytes", "prop41_bound",
    "brute_force_w4a4", "INT4_QMAX", "NVFP4_QMAX", "E4M3_MAX", "quantize_mxfp4_g32", "MXFP4_EMAX",
    "residual_iteration", "quantize_int8_rowwise", "INT8_QMAX",
]

INT4_QMAX = 7          # eq.(1): symmetric codes -7..7
NVFP4_QMAX = 6.0       # largest E2M1 magnitude
E4M3_MAX = 448.0       # largest finite E4M3 magnitude
MXFP4_EMAX = 2         # exponent of the largest E2M1 magnitude: 6 = 1.5 * 2^2
INT8_QMAX = 127        # eq.(1) with 8 bits: symmetric codes -127..127


# ---------------------------------------------------------------------------
# Number formats.  Each rounding is written from the format's definition.
# ---------------------------------------------------------------------------

def _round_significand(x: np.ndarray, bits: int) -> np.ndarray:
    """Round fp64 values to ``bits`` significant bits, ties to even (no range limits)."""
    x = np.asarray(x, dtype=np.float64)
    f, e = np.frexp(x)                       # x = f * 2**e, 0.5 <= |f| < 1
    return np.ldexp(np.rint(np.ldexp(f, bits)), e - bits)


def bf16_rn(x) -> np.ndarray:
    """Round to bfloat16 (8 significant bits, fp32 exponent range), nearest-even.

    Returns float32 arrays holding the bf16 values.  Magnitudes here never reach
    the bf16 subnormal range (< 2**-126), so only the significand is rounded.
    """
    return _round_significand(x, 8).astype(np.float32)


def fp16_rn(x) -> np.ndarray:
    """Round to IEEE binary16, nearest-even (NumPy's conversion), as float32."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


def _grid_round_even(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the nearest grid value to ``mag`` (>= 0); ties go to the even index.

    ``grid`` is sorted ascending and its index is the format's code, so an
    even index is an even (last mantissa bit 0) code.  Magnitudes above the
    last grid value saturate to it (``satfinite``).
    """
    mag = np.asarray(mag, dtype=np.float64)
    top = len(grid) - 1
    hi = np.searchsorted(grid, mag, side="left")          # grid[hi-1] < mag <= grid[hi]
    hi = np.clip(hi, 0, top)
    lo = np.clip(hi - 1, 0, top)
    d_lo = mag - grid[lo]
    d_hi = grid[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(mag >= grid[top], top, idx)
    idx = np.where(mag <= 0.0, 0, idx)
    return idx.astype(np.int64)


def _e4m3_grid() -> np.ndarray:
    vals = []
    for code in range(0x7F):                 # 0x7F is NaN in E4M3 (fn variant)
        e, m = code >> 3, code & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals)


E4M3_VALUES = _e4m3_grid()                     # 127 non-negative finite values, code order
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e4m3_rn_satfinite(x):
    """Round to E4M3 (bias 7, 3 mantissa bits, max 448), nearest-even, saturating.

    Returns (codes uint8, values float32).  Sign bit kept for negative inputs.
    """
    x = np.asarray(x, dtype=np.float64)
    idx = _grid_round_even(np.abs(x), E4M3_VALUES)
    neg = np.signbit(x)
    codes = (idx | np.where(neg, 0x80, 0)).astype(np.uint8)
    vals = np.where(neg, -E4M3_VALUES[idx], E4M3_VALUES[idx]).astype(np.float32)
    return codes, vals


def e2m1_rn_satfinite(x):
    """Round to E2M1 ({0, .5, 1, 1.5, 2, 3, 4, 6}), nearest-even, saturating at 6.

    Returns (codes uint8 in 0..15, values float32).  The sign is kept: a
    negative input that rounds to 0 gives code 0x8.
    """
    x = np.asarray(x, dtype=np.float64)
    idx = _grid_round_even(np.abs(x), E2M1_VALUES)
    neg = np.signbit(x)
    codes = (idx | np.where(neg, 8, 0)).astype(np.uint8)
    vals = np.where(neg, -E2M1_VALUES[idx], E2M1_VALUES[idx]).astype(np.float32)
    return codes, vals


def e4m3_value(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    v = E4M3_VALUES[codes & 0x7F]
    return np.where(codes & 0x80, -v, v)


def e2m1_value(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    v = E2M1_VALUES[codes & 7]
    return np.where(codes & 8, -v, v)


def int4_value(codes) -> np.ndarray:
    """4-bit two's complement code -> integer value."""
    codes = np.asarray(codes, dtype=np.int64) & 0xF
    return np.where(codes >= 8, codes - 16, codes).astype(np.float64)


# ---------------------------------------------------------------------------
# Smoothing (SVDQuant 阅读笔记 §3.1 eq.(3), eq.(4); msModelSlim SVDQuant 阶段一)
# ---------------------------------------------------------------------------

def smoothing_factors(X: np.ndarray, W: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """lambda_i = max|X[:, i]|**alpha / max|W[i, :]|**(1 - alpha)   (eq.(4)).

    ``X`` is [b, m] and ``W`` is [m, n] (Y = X W).  Computed in fp64 and stored
    as fp32.  Guard (reading 6): a zero statistic gives lambda_i = 1; otherwise
    lambda_i is at least 1e-5.
    """
    ax = np.max(np.abs(np.asarray(X, np.float64)), axis=0)
    aw = np.max(np.abs(np.asarray(W, np.float64)), axis=1)
    lam = np.ones_like(ax)
    ok = (ax > 0) & (aw > 0)
    lam[ok] = ax[ok] ** alpha / aw[ok] ** (1.0 - alpha)
    lam[ok] = np.maximum(lam[ok], 1e-5)
    return lam.astype(np.float32)


def smooth_activations(X: np.ndarray, lam: Optional[np.ndarray]) -> np.ndarray:
    """X_hat = bf16_rn(fp32(X) / lambda): the X D^-1 of eq.(3), rounded once to bf16."""
    X32 = np.asarray(X, dtype=np.float32)
    if lam is None:
        return bf16_rn(X32)
    q = (X32 / np.asarray(lam, dtype=np.float32)[None, :]).astype(np.float32)
    return bf16_rn(q)


def smooth_weight(W: np.ndarray, lam: Optional[np.ndarray]) -> np.ndarray:
    """W_tilde = D W (eq.(3)), fp64; row i of W (input channel i) times lambda_i."""
    W = np.asarray(W, dtype=np.float64)
    if lam is None:
        return W.copy()
    return np.asarray(lam, dtype=np.float64)[:, None] * W


# ---------------------------------------------------------------------------
# Low-rank split (SVDQuant 阅读笔记 §5 eq.(10); AutoRound SVDQuant "Residual iteration")
# ---------------------------------------------------------------------------

def svd_split(W_tilde: np.ndarray, rank: int):
    """Truncated SVD split of W_tilde [m, n] (eq.(10)).

    L1 = U[:, :r] Sigma_r (m x r), L2 = V[:, :r]^T (r x n).  The factors are
    rounded to bf16 first and R = W_tilde - L1_bf16 L2_bf16 is formed in fp64,
    then stored as fp32.  Returns a dict with the fp64 factors, the bf16
    factors, R (fp64 and fp32) and all singular values.
    """
    W_tilde = np.asarray(W_tilde, dtype=np.float64)
    U, S, Vt = np.linalg.svd(W_tilde, full_matrices=False)
    L1 = U[:, :rank] * S[:rank]
    L2 = Vt[:rank, :]
    L1b = bf16_rn(L1).astype(np.float64)
    L2b = bf16_rn(L2).astype(np.float64)
    R64 = W_tilde - L1b @ L2b
    return {
        "L1": L1, "L2": L2, "L1_bf16": L1b, "L2_bf16": L2b,
        "R64": R64, "R": R64.astype(np.float32), "sigma": S,
        "R_exact": W_tilde - L1 @ L2,
    }


def residual_iteration(fmt: str, W_tilde: np.ndarray, rank: int, iters: int,
                       early_stop: bool = False, X_hat: Optional[np.ndarray] = None):
    """AutoRound "SVDQuant（实验性功能）", "Residual iteration": alternate a low-rank fit
    with the deployment RTN quantize-dequantize of the residual (reading 17).

    Iteration 0 is the plain split of eq.(10): L1 L2 = SVD_r(W_tilde), R = W_tilde - L1 L2
    with bf16 factors.  Each further outer iteration fits the branch to W_tilde - Q(R_prev),
    forms the new residual R = W_tilde - L1 L2 and quantize-dequantizes it as it is deployed
    (per output channel along the input dimension, with the tensor scale of reading 4 for
    NVFP4).  The target error is the weight reconstruction error ||L1 L2 + Q(R) - W_tilde||_F,
    or, with calibration activations X_hat (smoothing on), the calibration output error
    ||X_hat (L1 L2 + Q(R) - W_tilde)||_F.  With early_stop the best candidate so far is kept
    and the loop ends at the first candidate whose error is worse; without it all iterations
    run and the last candidate is returned.
    """
    W_tilde = np.asarray(W_tilde, dtype=np.float64)
    Xh = None if X_hat is None else np.asarray(X_hat, dtype=np.float64)

    def qdq(R32):
        gw = pow2_global_scale(np.max(np.abs(R32)) if R32.size else 0.0) if fmt == "nvfp4" else 1.0
        return dequantize(fmt, quantize(fmt, np.ascontiguousarray(R32.T), gw)).T

    def target(L1b, L2b, QR):
        E = L1b @ L2b + QR - W_tilde
        return float(np.linalg.norm(E if Xh is None else Xh @ E))

    sp = svd_split(W_tilde, rank)
    cand = (sp["L1_bf16"], sp["L2_bf16"], sp["R"])
    QR = qdq(cand[2])
    errs = [target(cand[0], cand[1], QR)]
    best, best_err, best_it = cand, errs[0], 0
    for it in range(1, max(int(iters), 1)):
        fit = svd_split(W_tilde - QR, rank)
        L1b, L2b = fit["L1_bf16"], fit["L2_bf16"]
        cand = (L1b, L2b, (W_tilde - L1b @ L2b).astype(np.float32))
        QR = qdq(cand[2])
        errs.append(target(L1b, L2b, QR))
        if early_stop:
            if errs[-1] < best_err:
                best, best_err, best_it = cand, errs[-1], it
            else:
                break
        else:
            best, best_err, best_it = cand, errs[-1], it
    return {"L1_bf16": best[0], "L2_bf16": best[1], "R": best[2], "chosen": best_it, "errors": errs}


def lora_concat(L1: np.ndarray, L2: np.ndarray, lam: Optional[np.ndarray],
                A: np.ndarray, B: np.ndarray):
    """eq.(13): branch [L1, D A] x [L2; B]; the residual R is not re-quantized."""
    DA = A if lam is None else np.asarray(lam, np.float64)[:, None] * np.asarray(A, np.float64)
    return (np.concatenate([np.asarray(L1, np.float64), DA], axis=1),
            np.concatenate([np.asarray(L2, np.float64), np.asarray(B, np.float64)], axis=0))


# ---------------------------------------------------------------------------
# Group quantizers (SVDQuant 阅读笔记 §2.2 eq.(1), group sizes of §2.2 and §8)
# ---------------------------------------------------------------------------

def pow2_global_scale(amax: float) -> float:
    """Reading 4: smallest power of two g with amax / (6 g) <= 448."""
    amax = float(amax)
    if not amax > 0.0:
        return 1.0
    lim = NVFP4_QMAX * E4M3_MAX
    e = math.frexp(amax / lim)[1]
    # exact comparisons decide the boundary cases (amax / lim a power of two)
    while lim * 2.0 ** (e - 1) >= amax:
        e -= 1
    while lim * 2.0 ** e < amax:
        e += 1
    return float(2.0 ** e)


def quantize_int4_g64(x: np.ndarray):
    """eq.(1) per 64-element group along the last axis: s = max|Z| / 7, q = round(Z / s).

    ``x`` is [rows, K] float32 (bf16 values).  Returns dict with nibble codes
    [rows, K] (4-bit two's complement), scale values [rows, K/64] (fp16 values
    as float32), scale bits (uint16) and the integer values.
    """
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    xg = x.reshape(rows, K // 64, 64)
    a = np.max(np.abs(xg), axis=2)
    t = (a / np.float32(INT4_QMAX)).astype(np.float32)
    s16 = np.minimum(t.astype(np.float16), np.float16(65504.0))
    s = s16.astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0))
    v = (xg / safe[..., None]).astype(np.float32)
    q = np.clip(np.rint(v), -INT4_QMAX, INT4_QMAX)
    q = np.where((s > 0)[..., None], q, 0.0).reshape(rows, K)
    codes = (q.astype(np.int64) & 0xF).astype(np.uint8)
    return {"codes": codes, "q": q.astype(np.float64), "scale": s,
            "scale_bits": s16.view(np.uint16), "gscale": 1.0}


def quantize_nvfp4_g16(x: np.ndarray, gscale: float):
    """NVFP4 per 16-element group with E4M3 scales and a power-of-two tensor scale.

    s = e4m3_rn_satfinite(fp32(fp32(a / 6) / g));  q = e2m1_rn_satfinite(fp32(x / (s g))).
    """
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    g = np.float32(gscale)
    xg = x.reshape(rows, K // 16, 16)
    a = np.max(np.abs(xg), axis=2)
    t = ((a / np.float32(NVFP4_QMAX)).astype(np.float32) / g).astype(np.float32)
    s_bits, s = e4m3_rn_satfinite(t)
    denom = (s * g).astype(np.float32)
    safe = np.where(denom > 0, denom, np.float32(1.0))
    v = (xg / safe[..., None]).astype(np.float32)
    codes, vals = e2m1_rn_satfinite(v)
    codes = np.where((denom > 0)[..., None], codes, 0).astype(np.uint8)
    vals = np.where((denom > 0)[..., None], vals, 0.0)
    return {"codes": codes.reshape(rows, K), "q": vals.reshape(rows, K).astype(np.float64),
            "scale": s.astype(np.float32), "scale_bits": s_bits, "gscale": float(gscale)}


def quantize_mxfp4_g32(x: np.ndarray):
    """MXFP4 per 32-element group with a shared power-of-two (E8M0) scale (reading 9).

    X = 2^clip(floor(log2 a) - 2, -127, 127), a = max |x| of the group; q = e2m1(x / X).
    """
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    xg = x.reshape(rows, K // 32, 32)
    a = np.max(np.abs(xg), axis=2).astype(np.float64)
    mant, ex = np.frexp(a)                     # a = mant * 2^ex, mant in [0.5, 1): floor(log2 a) = ex - 1
    e = np.where(a > 0, ex - 1 - MXFP4_EMAX, -127)
    e = np.clip(e, -127, 127).astype(np.int64)
    X = np.ldexp(1.0, e)                       # exact powers of two
    v = (xg.astype(np.float64) / X[..., None]).astype(np.float32)   # exact: division by 2^e
    codes, vals = e2m1_rn_satfinite(v)
    return {"codes": codes.reshape(rows, K).astype(np.uint8), "q": vals.reshape(rows, K).astype(np.float64),
            "scale": X, "scale_bits": (e + 127).astype(np.uint8), "gscale": 1.0}


def quantize_int8_rowwise(x: np.ndarray):
    """eq.(1) with 8-bit codes and one group per row (reading 10): per-token activations,
    per-output-channel weights.

    s = fp32(max|x_row| / 127) kept in fp32;  q = clamp(rint(fp32(x / s)), -127, 127).
    Returns codes as uint8 two's-complement bytes [rows, K], the integer values, the
    fp32 scale per row (as a [rows, 1] array) and its bits.
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.max(np.abs(x), axis=1, keepdims=True) if x.shape[1] else np.zeros((x.shape[0], 1), np.float32)
    s = (a / np.float32(INT8_QMAX)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0))
    v = (x / safe).astype(np.float32)
    q = np.clip(np.rint(v), -INT8_QMAX, INT8_QMAX)
    q = np.where(s > 0, q, 0.0)
    codes = (q.astype(np.int64) & 0xFF).astype(np.uint8)
    return {"codes": codes, "q": q.astype(np.float64), "scale": s,
            "scale_bits": s.view(np.uint32), "gscale": 1.0}


def quantize(fmt: str, x: np.ndarray, gscale: float = 1.0):
    if fmt == "w8a8":
        return quantize_int8_rowwise(x)
    if fmt == "int4":
        return quantize_int4_g64(x)
    if fmt == "nvfp4":
        return quantize_nvfp4_g16(x, gscale)
    if fmt == "mxfp4":
        return quantize_mxfp4_g32(x)
    raise ValueError(fmt)


def group_size(fmt: str, K: Optional[int] = None) -> int:
    """Elements per scale along K; W8A8 has one scale per row (the whole of K)."""
    if fmt == "w8a8":
        return K
    return {"int4": 64, "nvfp4": 16, "mxfp4": 32}[fmt]


def dequantize(fmt: str, qd) -> np.ndarray:
    """Q(Z) = g * s * q (fp64, exact)."""
    q = qd["q"]
    rows, K = q.shape
    gsz = group_size(fmt, K)
    s = np.repeat(qd["scale"].astype(np.float64), gsz, axis=1)
    return qd["gscale"] * s * q


# ---------------------------------------------------------------------------
# The hot path as two steps (SVDQuant 阅读笔记 §6.1 "算法 2" data flow, eq.(7))
# ---------------------------------------------------------------------------

def prologue(fmt: str, X: np.ndarray, lam: Optional[np.ndarray], act_gscale: float,
             L1_rk: Optional[np.ndarray]):
    """Steps 1-3 of the fused data flow: smooth, quantize, down-project.

    ``L1_rk`` is the bf16 down factor stored [r, K] (msModelSlim l1 shape).
    Z = bf16_rn(X_hat L1) with the product formed in fp64.
    """
    xh = smooth_activations(X, lam)
    qd = quantize(fmt, xh, act_gscale)
    if L1_rk is None or np.asarray(L1_rk).shape[0] == 0:
        Z = np.zeros((xh.shape[0], 0), np.float32)
    else:
        Z = bf16_rn(xh.astype(np.float64) @ np.asarray(L1_rk, np.float64).T)
    return {"xhat": xh, "q": qd, "Z": Z}


def pack_weight(fmt: str, R_nk: np.ndarray, L1_rk: np.ndarray, L2_nr: np.ndarray,
                act_gscale: float = 1.0):
    """Offline pack of an already-decomposed layer.

    R_nk [N, K] fp32 is quantized per output channel along K; the global scale
    is the power of two of reading 4 for NVFP4 (1 for INT4).  L1 and L2 are
    rounded to bf16; L2 is also returned divided by (g_x g_w), the form in
    which the fused kernel adds Z L2 into the block-scaled accumulator before
    the common (g_x g_w) factor is applied.
    """
    R_nk = np.asarray(R_nk, dtype=np.float32)
    if fmt == "nvfp4":
        gw = pow2_global_scale(np.max(np.abs(R_nk)) if R_nk.size else 0.0)
    else:
        gw = 1.0      # INT4, MXFP4 and W8A8 have no tensor scale
    qd = quantize(fmt, R_nk, gw)
    L1b = bf16_rn(L1_rk)
    L2b = bf16_rn(L2_nr)
    L2s = bf16_rn(L2b.astype(np.float64) / (act_gscale * gw))
    return {"q": qd, "gscale": gw, "L1_bf16": L1b, "L2_bf16": L2b, "L2_scaled": L2s}


def w4a4_main(qa, qw) -> np.ndarray:
    """sum_G s_x s_w sum_{k in G} q_x q_w (without the tensor scales), fp64 [M, N]."""
    fmt_g = qa["q"].shape[1] // qa["scale"].shape[1]
    xa = qa["q"] * np.repeat(qa["scale"].astype(np.float64), fmt_g, axis=1)
    wb = qw["q"] * np.repeat(qw["scale"].astype(np.float64), fmt_g, axis=1)
    return xa @ wb.T


def gemm_forward(qa, act_gscale: float, qw, w_gscale: float, Z: np.ndarray,
                 L2_nr: np.ndarray, bias: Optional[np.ndarray]):
    """Y = g_x g_w Q(X_hat) Q(R) + Z L2 + bias (eq.(7)), fp64, and its bf16 rounding."""
    Y = act_gscale * w_gscale * w4a4_main(qa, qw)
    if Z is not None and Z.shape[1] > 0:
        Y = Y + np.asarray(Z, np.float64) @ np.asarray(L2_nr, np.float64).T
    if bias is not None:
        Y = Y + np.asarray(bias, np.float64)[None, :]
    return {"Y64": Y, "Y": bf16_rn(Y)}


def layer_forward(fmt: str, X, lam, act_gscale, packed, bias=None):
    """Whole layer: prologue then GEMM, on already packed weights."""
    pro = prologue(fmt, X, lam, act_gscale, packed["L1_bf16"])
    out = gemm_forward(pro["q"], act_gscale, packed["q"], packed["gscale"], pro["Z"],
                       packed["L2_bf16"], bias)
    out.update(pro)
    return out


def prepare_layer(fmt: str, X_calib: np.ndarray, W: np.ndarray, rank: int,
                  alpha: float = 0.5, smooth: bool = True, lora=None,
                  residual_iters: int = 1, early_stop: bool = False):
    """Offline build of one layer: lambda (eq.(4)), W_tilde (eq.(3)), SVD split (eq.(10)).

    With residual_iters > 1 the split is refined by ``residual_iteration``, whose
    target is the calibration output error when smoothing is on and the weight
    reconstruction error when it is off.  Returns the ABI-orientation arrays:
    R_nk [N, K] fp32, L1_rk [r, K] and L2_nr [N, r] (fp64 values of the bf16
    factors), lambda [K] fp32 and the activation tensor scale g_x (reading 4,
    from the calibration X_hat).
    """
    lam = smoothing_factors(X_calib, W, alpha) if smooth else None
    Wt = smooth_weight(W, lam)
    if residual_iters > 1:
        ri = residual_iteration(fmt, Wt, rank, residual_iters, early_stop,
                                smooth_activations(X_calib, lam) if smooth else None)
        sp = {"L1_bf16": ri["L1_bf16"], "L2_bf16": ri["L2_bf16"], "R": ri["R"], "residual": ri}
    else:
        sp = svd_split(Wt, rank)
    L1, L2 = sp["L1_bf16"], sp["L2_bf16"]
    if lora is not None:
        L1, L2 = lora_concat(L1, L2, lam, lora[0], lora[1])
        L1, L2 = bf16_rn(L1).astype(np.float64), bf16_rn(L2).astype(np.float64)
    xh = smooth_activations(X_calib, lam)
    gx = pow2_global_scale(np.max(np.abs(xh))) if fmt == "nvfp4" else 1.0
    return {"lam": lam, "W_tilde": Wt, "split": sp, "R_nk": np.ascontiguousarray(sp["R"].T),
            "L1_rk": np.ascontiguousarray(L1.T), "L2_nr": np.ascontiguousarray(L2.T),
            "act_gscale": gx}


# ---------------------------------------------------------------------------
# Counting formulas and bounds (SVDQuant 阅读笔记 eq.(6), eq.(11), eq.(12))
# ---------------------------------------------------------------------------

def rho_mac(m: int, n: int, r: int) -> float:
    """eq.(11): extra multiply-adds of the branch, (bmr + brn) / bmn = r/m + r/n."""
    return r / m + r / n


def rho_bytes(m: int, n: int, r: int) -> float:
    """eq.(12): (mn/2 + 2r(m+n)) / (2mn) = 1/4 + r/m + r/n."""
    return (m * n / 2 + 2 * r * (m + n)) / (2 * m * n)


def prop41_bound(X, W, QX, QW):
    """eq.(6): returns (lhs, middle, rhs) of the Prop. 4.1 chain (Frobenius norms)."""
    X, W, QX, QW = (np.asarray(a, np.float64) for a in (X, W, QX, QW))
    dX, dW = X - QX, W - QW
    fro = np.linalg.norm
    lhs = fro(X @ W - QX @ QW)
    mid = fro(X) * fro(dW) + fro(dX) * fro(QW)
    rhs = fro(X) * fro(dW) + fro(dX) * (fro(W) + fro(dW))
    return lhs, mid, rhs


def brute_force_w4a4(fmt: str, qa, qw) -> np.ndarray:
    """Triple loop over (i, j, k) with per-element dequantization (tiny shapes only)."""
    M, K = qa["q"].shape
    gsz = group_size(fmt, K)
    N = qw["q"].shape[0]
    out = np.zeros((M, N))
    for i in range(M):
        for j in range(N):
            acc = 0.0
            for k in range(K):
                g = k // gsz
                acc += (qa["scale"][i, g] * qa["q"][i, k]) * (qw["scale"][j, g] * qw["q"][j, k])
            out[i, j] = acc
    return out
