"""Offline preparation of one layer with PyTorch (not on the timed path).

Follows "SVDQuant 阅读笔记" §3.1 eq.(4) (smoothing factor, alpha = 0.5),
eq.(3) (W_tilde = D W) and §5 eq.(10) (truncated SVD split, Sigma in L1),
with the factors materialised in bf16 before the residual is formed as in
"SVDQuant（实验性功能）" ("Residual iteration").  The LoRA concatenation is
eq.(13).  Used to build benchmark layers; the decomposition runs on the GPU
when one is present (torch.linalg.svd in fp64).

``residual_iters > 1`` refines the split as AutoRound's "Residual iteration"
describes: each outer iteration refits the low-rank branch to W_tilde - Q(R_prev)
and quantize-dequantizes the new residual exactly as the weight pack does (same
group sizes, scale rounding and code rounding), keeping the best candidate when
early stop is on.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch

from . import binding as B


def _bf16_round(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16).to(t.dtype)


def pow2_tensor_scale(amax: float) -> float:
    """Smallest power of two g with amax <= 6 * 448 * g (1 when amax == 0)."""
    if not amax > 0.0:
        return 1.0
    lim = 6.0 * 448.0
    e = math.frexp(amax / lim)[1]
    while lim * 2.0 ** (e - 1) >= amax:
        e -= 1
    while lim * 2.0 ** e < amax:
        e += 1
    return 2.0 ** e


# E2M1 decision thresholds on |v|: code index i+1 is taken when |v| passes the
# midpoint between grid values i and i+1; a tie goes to the even index.
_E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
_E2M1_MIDS = ((0.25, False), (0.75, True), (1.25, False), (1.75, True),
              (2.5, False), (3.5, True), (5.0, False))      # (midpoint, tie rounds up)


def _e2m1_rn(v: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 value of fp32 v (ties to even, saturating at 6), as fp64."""
    m = v.abs()
    idx = torch.zeros_like(m, dtype=torch.int64)
    for t, up in _E2M1_MIDS:
        idx += (m >= t) if up else (m > t)
    mag = torch.tensor(_E2M1_GRID, dtype=torch.float64, device=v.device)[idx]
    return torch.where(torch.signbit(v), -mag, mag)


def qdq_weight(fmt: str, R_nk: torch.Tensor) -> torch.Tensor:
    """Quantize-dequantize R [N, K] fp32 per output row along K as the weight pack does.

    INT4 g64: s = fp16(fp32(a / 7)) (clamped to 65504), q = rint(fp32(R / s)) in [-7, 7].
    NVFP4 g16: s = e4m3(fp32(fp32(a / 6) / g_w)) with g_w the power-of-two tensor scale,
    q = e2m1(fp32(R / fp32(s g_w))).  MXFP4 g32: X = 2^clip(floor(log2 a) - 2, -127, 127),
    q = e2m1(R / X).  W8A8: one scale per row, s = fp32(a / 127), q = clamp(rint(fp32(R / s)),
    -127, 127).  Returns g s q in fp64.
    """
    R = R_nk.to(torch.float32)
    N, K = R.shape

    def div(x: torch.Tensor, c: float) -> torch.Tensor:
        # a tensor divisor keeps the IEEE divide (a Python-scalar divisor may become a
        # multiply by its reciprocal on the device, which is not the same rounding)
        return x / torch.full_like(x, c)
    if fmt == "int4":
        Rg = R.reshape(N, K // 64, 64)
        t = div(Rg.abs().amax(2), 7.0)
        s = torch.clamp(t.to(torch.float16).to(torch.float32), max=65504.0)
        safe = torch.where(s > 0, s, torch.ones_like(s))
        q = torch.clamp(torch.round(Rg / safe[..., None]), -7.0, 7.0)
        q = torch.where((s > 0)[..., None], q, torch.zeros_like(q))
        return (q.to(torch.float64) * s.to(torch.float64)[..., None]).reshape(N, K)
    if fmt == "nvfp4":
        gw = pow2_tensor_scale(float(R.abs().max())) if R.numel() else 1.0
        Rg = R.reshape(N, K // 16, 16)
        t = div(div(Rg.abs().amax(2), 6.0), gw)
        s = torch.clamp(t, max=448.0).to(torch.float8_e4m3fn).to(torch.float32)
        den = s * gw
        safe = torch.where(den > 0, den, torch.ones_like(den))
        q = _e2m1_rn(Rg / safe[..., None])
        q = torch.where((den > 0)[..., None], q, torch.zeros_like(q))
        return (q * den.to(torch.float64)[..., None]).reshape(N, K)
    if fmt == "w8a8":
        s = div(R.abs().amax(1, keepdim=True), 127.0)
        safe = torch.where(s > 0, s, torch.ones_like(s))
        q = torch.clamp(torch.round(R / safe), -127.0, 127.0)
        q = torch.where(s > 0, q, torch.zeros_like(q))
        return q.to(torch.float64) * s.to(torch.float64)
    if fmt == "mxfp4":
        Rg = R.reshape(N, K // 32, 32)
        a = Rg.abs().amax(2).to(torch.float64)
        ex = torch.frexp(a).exponent.to(torch.int64)
        e = torch.where(a > 0, ex - 3, torch.full_like(ex, -127)).clamp(-127, 127)
        X = ((e + 1023) << 52).view(torch.float64)                       # 2^e, built exactly
        q = _e2m1_rn((Rg.to(torch.float64) / X[..., None]).to(torch.float32))
        return (q * X[..., None]).reshape(N, K)
    raise ValueError(fmt)


def _split(Wt: torch.Tensor, rank: int):
    U, S, Vh = torch.linalg.svd(Wt, full_matrices=False)
    return _bf16_round(U[:, :rank] * S[:rank]), _bf16_round(Vh[:rank, :])


def residual_iteration(fmt: str, Wt: torch.Tensor, rank: int, iters: int,
                       early_stop: bool = False, X_hat: Optional[torch.Tensor] = None):
    """Refine the split of W_tilde [K, N] (fp64) by residual iteration.

    Iteration 0 is the plain split; iteration i > 0 fits the branch to
    W_tilde - Q(R_{i-1}).  The error is ||L1 L2 + Q(R) - W_tilde||_F, measured
    through X_hat when it is given.  Returns (L1 [K, r], L2 [r, N], R [K, N] fp32,
    chosen iteration, list of errors).
    """
    def run(L1, L2):
        R = (Wt - L1 @ L2).to(torch.float32)
        QR = qdq_weight(fmt, R.T).T
        E = L1 @ L2 + QR - Wt
        err = float(torch.linalg.norm(E if X_hat is None else X_hat @ E))
        return R, QR, err

    L1, L2 = _split(Wt, rank)
    R, QR, err = run(L1, L2)
    errs = [err]
    best = (L1, L2, R, 0, err)
    for it in range(1, max(int(iters), 1)):
        L1, L2 = _split(Wt - QR, rank)
        R, QR, err = run(L1, L2)
        errs.append(err)
        if early_stop and not err < best[4]:
            break
        if not early_stop or err < best[4]:
            best = (L1, L2, R, it, err)
    return best[0], best[1], best[2], best[3], errs


def prepare(fmt: str, X: np.ndarray, W: np.ndarray, rank: int, alpha: float = 0.5,
            lora: Optional[tuple] = None, device: Optional[str] = None,
            residual_iters: int = 1, early_stop: bool = False):
    """Return lambda [K] fp32, R [N, K] fp32, L1 [r, K] fp32, L2 [N, r] fp32 and g_x.

    Smoothing is always on here, so residual iterations measure the calibration
    output error through X_hat = bf16(X / lambda).
    """
    dev = device or ("cuda" if torch.cuda.is_available() else "cpu")
    Xt = torch.from_numpy(np.ascontiguousarray(X, np.float32)).to(dev, torch.float64)
    Wt = torch.from_numpy(np.ascontiguousarray(W, np.float64)).to(dev)
    ax = Xt.abs().amax(0)
    aw = Wt.abs().amax(1)
    lam = torch.ones_like(ax)
    ok = (ax > 0) & (aw > 0)
    lam[ok] = torch.clamp(ax[ok] ** alpha / aw[ok] ** (1.0 - alpha), min=1e-5)
    lam32 = lam.to(torch.float32)
    Ws = lam32.to(torch.float64)[:, None] * Wt                       # D W
    xh = (Xt.to(torch.float32) / lam32[None, :]).to(torch.bfloat16).float()
    info = {}
    if residual_iters > 1:
        L1, L2, R, chosen, errs = residual_iteration(fmt, Ws, rank, residual_iters, early_stop,
                                                     xh.to(torch.float64))
        info = {"chosen": chosen, "errors": errs}
    else:
        L1, L2 = _split(Ws, rank)                                      # [K, r], [r, N]
        R = (Ws - L1 @ L2).to(torch.float32)                           # [K, N]
    if lora is not None:
        A = torch.from_numpy(np.asarray(lora[0], np.float64)).to(dev)
        Bm = torch.from_numpy(np.asarray(lora[1], np.float64)).to(dev)
        L1 = _bf16_round(torch.cat([L1, lam32.to(torch.float64)[:, None] * A], 1))
        L2 = _bf16_round(torch.cat([L2, Bm], 0))
    gx = pow2_tensor_scale(float(xh.abs().max())) if fmt == "nvfp4" else 1.0
    return {
        "residual": info,
        "lam": lam32.cpu().numpy(),
        "R_nk": R.T.contiguous().cpu().numpy(),
        "L1_rk": L1.T.contiguous().to(torch.float32).cpu().numpy(),
        "L2_nr": L2.T.contiguous().to(torch.float32).cpu().numpy(),
        "act_gscale": gx,
    }


def pack(fmt: str, prep: dict):
    """svdq_pack_weight on the prepared arrays (host)."""
    rank = prep["L1_rk"].shape[0]
    return B.pack_weight_np(fmt, prep["R_nk"], prep["L1_rk"] if rank else None,
                            prep["L2_nr"] if rank else None, prep["act_gscale"])
