"""Offline preparation of one layer with PyTorch (not on the timed path).

Follows "SVDQuant 阅读笔记" §3.1 eq.(4) (smoothing factor, alpha = 0.5),
eq.(3) (W_tilde = D W) and §5 eq.(10) (truncated SVD split, Sigma in L1),
with the factors materialised in bf16 before the residual is formed as in
"SVDQuant（实验性功能）" ("Residual iteration").  The LoRA concatenation is
eq.(13).  Used to build benchmark layers; the decomposition runs on the GPU
when one is present (torch.linalg.svd in fp64).
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


def prepare(fmt: str, X: np.ndarray, W: np.ndarray, rank: int, alpha: float = 0.5,
            lora: Optional[tuple] = None, device: Optional[str] = None):
    """Return lambda [K] fp32, R [N, K] fp32, L1 [r, K] fp32, L2 [N, r] fp32 and g_x."""
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
    U, S, Vh = torch.linalg.svd(Ws, full_matrices=False)
    L1 = _bf16_round(U[:, :rank] * S[:rank])                          # [K, r]
    L2 = _bf16_round(Vh[:rank, :])                                    # [r, N]
    R = (Ws - L1 @ L2).to(torch.float32)                              # [K, N]
    if lora is not None:
        A = torch.from_numpy(np.asarray(lora[0], np.float64)).to(dev)
        Bm = torch.from_numpy(np.asarray(lora[1], np.float64)).to(dev)
        L1 = _bf16_round(torch.cat([L1, lam32.to(torch.float64)[:, None] * A], 1))
        L2 = _bf16_round(torch.cat([L2, Bm], 0))
    xh = (Xt.to(torch.float32) / lam32[None, :]).to(torch.bfloat16).float()
    gx = pow2_tensor_scale(float(xh.abs().max())) if fmt == "nvfp4" else 1.0
    return {
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
