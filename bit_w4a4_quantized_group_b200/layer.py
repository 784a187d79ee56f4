"""A W4A4 + low-rank linear layer held on one GPU (thin wrapper over the C ABI).

``forward(X)`` makes the two device calls of include/svdq.h on the current
stream: the prologue (smooth, quantize, down-project) and the fused GEMM
(4-bit product + up-projection + bias).  Buffers are preallocated with
PyTorch; nothing here computes any part of the layer.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import binding as B


def _to_dev_u16_as_bf16(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)


class W4A4LowRankLinear:
    def __init__(self, fmt: str, N: int, K: int, packed: dict, lam: Optional[np.ndarray], act_gscale: float,
                 bias: Optional[np.ndarray] = None, device="cuda"):
        self.fmt = fmt
        self.device = torch.device(device)
        self.N, self.K = int(N), int(K)
        self.rank = packed["L1_bf16"].shape[0]
        self.w_codes = torch.from_numpy(packed["w_codes"]).to(self.device)
        self.w_scales = torch.from_numpy(packed["w_scales"]).to(self.device)
        self.w_gscale = float(packed["w_gscale"])
        self.act_gscale = float(act_gscale)
        self.L1 = _to_dev_u16_as_bf16(packed["L1_bf16"], self.device) if self.rank else None
        self.L2 = _to_dev_u16_as_bf16(packed["L2_bf16"], self.device) if self.rank else None
        if lam is not None:
            lam32 = np.ascontiguousarray(lam, np.float32)
            # the smoothing divide x / lambda is an IEEE divide only for finite, normal, positive
            # lambda (the C ABI's contract); anything else is rejected here, before any launch
            tiny = np.finfo(np.float32).tiny
            if lam32.shape != (self.K,) or not np.all(np.isfinite(lam32) & (lam32 >= tiny)):
                raise ValueError("lambda must hold K finite, normal, positive float32 values")
            self.lam = torch.from_numpy(lam32).to(self.device)
        else:
            self.lam = None
        self.bias = None
        if bias is not None:
            # bf16 by round-to-nearest-even (torch's conversion), like every other bf16 operand
            b32 = torch.from_numpy(np.ascontiguousarray(bias, np.float32).reshape(-1))
            self.bias = b32.to(torch.bfloat16).to(self.device)
        self._ws = {}

    def workspace(self, M: int):
        """Preallocated activation codes / scales / Z for M rows."""
        if M not in self._ws:
            sz = B.svdq_buffer_sizes(self.fmt, M, self.N, self.K, self.rank)
            self._ws[M] = {
                "a_codes": torch.empty(sz.a_codes, dtype=torch.uint8, device=self.device),
                "a_scales": torch.empty(sz.a_scales, dtype=torch.uint8, device=self.device),
                "Z": torch.empty((M, self.rank), dtype=torch.bfloat16, device=self.device) if self.rank else None,
            }
        return self._ws[M]

    def forward(self, X: torch.Tensor, Y: Optional[torch.Tensor] = None, check: bool = False) -> torch.Tensor:
        """Y = the layer applied to X (both calls on the current stream, asynchronous).

        With ``check=True`` the call also synchronizes the stream and reads the library's
        device error word: a kernel whose bounded wait ran out (for instance on a GPU that
        is time-sliced with other work) leaves Y undefined, and this raises instead of
        returning it.  Without it, callers that need the guarantee poll
        ``binding.svdq_get_last_device_error`` themselves.
        """
        M, K = X.shape
        ws = self.workspace(M)
        if Y is None:
            Y = torch.empty((M, self.N), dtype=torch.bfloat16, device=self.device)
        stream = torch.cuda.current_stream(self.device).cuda_stream     # one lookup for both calls
        B.quantize_act_lowrank_down_t(self.fmt, X, self.lam, self.act_gscale, self.L1,
                                      ws["a_codes"], ws["a_scales"], ws["Z"], stream)
        B.w4a4_gemm_lowrank_up_t(self.fmt, M, self.N, K, self.rank, ws["a_codes"], ws["a_scales"],
                                 self.act_gscale, self.w_codes, self.w_scales, self.w_gscale,
                                 ws["Z"], self.L2, self.bias, Y, stream)
        if check:
            st, site = B.svdq_get_last_device_error(torch.cuda.current_stream(self.device).cuda_stream)
            if st != B.SVDQ_OK:
                raise B.SvdqError(st, f"layer forward (device wait site {site})")
        return Y

    def gemm_only(self, M: int, Y: torch.Tensor, rank: Optional[int] = None):
        """The fused GEMM alone on the current workspace (rank 0 drops the branch)."""
        ws = self.workspace(M)
        r = self.rank if rank is None else rank
        B.w4a4_gemm_lowrank_up_t(self.fmt, M, self.N, self.K, r, ws["a_codes"], ws["a_scales"],
                                 self.act_gscale, self.w_codes, self.w_scales, self.w_gscale,
                                 ws["Z"] if r else None, self.L2 if r else None, self.bias, Y)

    def prologue_only(self, X: torch.Tensor, rank: Optional[int] = None):
        """The prologue alone (rank 0 quantizes without the down projection)."""
        M, _ = X.shape
        ws = self.workspace(M)
        r = self.rank if rank is None else rank
        B.quantize_act_lowrank_down_t(self.fmt, X, self.lam, self.act_gscale, self.L1 if r else None,
                                      ws["a_codes"], ws["a_scales"], ws["Z"] if r else None)
