"""Seeded synthetic inputs for the W4A4 + low-rank linear layer.

This module only draws random data with the shapes and value structure of
DiT-style linear layers.  It holds none of the method's arithmetic: no
smoothing factor, no decomposition, no quantizer.  Both the CPU reference
(under ``oracle/``) and the CUDA path consume what it returns.

Workload structure follows the layer shape and outlier description of
"SVDQuant 阅读笔记" §2.1 (X is b x m, W is m x n) and §3.1/§3.2 (a few
input channels carry very large activations; after smoothing the weight
gains a dominant low-rank component):

* ``X`` ~ N(0, 1) per element (GELU(N(0, 1)) for the MLP-down layer), with a
  random 1% of input channels multiplied by 30 (tiny layer: 8 channels x 50),
  rounded to bf16 because activations arrive as bf16.
* ``W`` ~ N(0, sigma_W) plus a planted rank-k "spike" ``U_s diag(s) V_s^T``
  whose singular vectors come from QR of Gaussian matrices.

Draw order is fixed (X, outlier channels, W, U_s, V_s, bias, LoRA A, LoRA B)
so that a seed fully determines a layer.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import ml_dtypes
import numpy as np


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    b: int            # tokens (GEMM M)
    m: int            # input features (GEMM K)
    n: int            # output features (GEMM N)
    rank: int         # low-rank branch rank r (after any LoRA concatenation)
    seed: int
    sigma_w: float = 0.02
    gelu_x: bool = False
    outlier_frac: float = 0.01
    outlier_count: Optional[int] = None   # overrides outlier_frac when set
    outlier_mult: float = 30.0
    spike_rank: int = 8
    spike_sigma: Optional[float] = None   # per-direction singular value; None: 2.5 x bulk edge
    lora_rank: int = 0                    # rank of a LoRA adapter concatenated onto the branch
    with_bias: bool = True

    @property
    def base_rank(self) -> int:
        return self.rank - self.lora_rank


def _dit(name, b, m, n, seed, rank=32, **kw):
    return LayerConfig(name=name, b=b, m=m, n=n, rank=rank, seed=seed, **kw)


# Named layers (sizes of DiT attention / MLP projections at 4096 image + 512 text tokens).
TINY = LayerConfig(name="tiny", b=256, m=512, n=512, rank=16, seed=0, outlier_count=8,
                   outlier_mult=50.0, spike_rank=4, spike_sigma=2.5)
QKV = _dit("qkv", 4608, 3072, 9216, seed=1)
MLP_UP = _dit("mlp_up", 4608, 3072, 12288, seed=2)
MLP_DOWN = _dit("mlp_down", 4608, 12288, 3072, seed=3, sigma_w=0.01, gelu_x=True)

NAMED = {c.name: c for c in (TINY, QKV, MLP_UP, MLP_DOWN)}


def sweep_configs():
    """Batch x shape x rank grid; rank 48 is a rank-16 LoRA concatenated onto rank 32."""
    out = []
    idx = 0
    for b in (256, 1024, 4096, 16384):
        for (m, n) in ((3072, 3072), (3072, 12288)):
            for r in (0, 16, 32, 48, 64, 128):
                lora = 16 if r == 48 else 0
                out.append(_dit(f"sweep_b{b}_m{m}_n{n}_r{r}", b, m, n, seed=100 + idx,
                                rank=r, lora_rank=lora))
                idx += 1
    return out


def to_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (library cast) and return the values as float32."""
    return np.asarray(x, dtype=np.float32).astype(ml_dtypes.bfloat16).astype(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already exact bf16 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _gelu_erf(x: np.ndarray) -> np.ndarray:
    from scipy.special import erf
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


@dataclasses.dataclass
class Layer:
    cfg: LayerConfig
    X: np.ndarray            # [b, m] float32 holding bf16 values
    W: np.ndarray            # [m, n] float64 (input-major, as in Y = X W)
    bias: Optional[np.ndarray]   # [n] float32 holding bf16 values
    lora_A: Optional[np.ndarray]  # [m, k] float64
    lora_B: Optional[np.ndarray]  # [k, n] float64
    outlier_channels: np.ndarray


def make_layer(cfg: LayerConfig, b: Optional[int] = None) -> Layer:
    """Draw one synthetic layer.  ``b`` overrides the token count (same weights)."""
    rng = np.random.default_rng(cfg.seed)
    rows = cfg.b if b is None else b
    m, n = cfg.m, cfg.n
    x = rng.standard_normal((rows, m))
    if cfg.gelu_x:
        x = _gelu_erf(x)
    n_out = cfg.outlier_count if cfg.outlier_count is not None else int(round(cfg.outlier_frac * m))
    ch = np.sort(rng.choice(m, size=n_out, replace=False)) if n_out > 0 else np.zeros(0, np.int64)
    x[:, ch] *= cfg.outlier_mult
    X = to_bf16(x)

    W = rng.standard_normal((m, n)) * cfg.sigma_w
    k = cfg.spike_rank
    if k > 0:
        us, _ = np.linalg.qr(rng.standard_normal((m, k)))
        vs, _ = np.linalg.qr(rng.standard_normal((n, k)))
        if cfg.spike_sigma is not None:
            s = cfg.spike_sigma
        else:
            s = 2.5 * cfg.sigma_w * (math.sqrt(m) + math.sqrt(n))
        W = W + (us * s) @ vs.T

    bias = to_bf16(rng.standard_normal(n) * 0.1) if cfg.with_bias else None
    lora_A = lora_B = None
    if cfg.lora_rank > 0:
        lora_A = rng.standard_normal((m, cfg.lora_rank)) / math.sqrt(m)
        lora_B = rng.standard_normal((cfg.lora_rank, n)) * cfg.sigma_w
    return Layer(cfg=cfg, X=X, W=W, bias=bias, lora_A=lora_A, lora_B=lora_B, outlier_channels=ch)


def make_activations(cfg: LayerConfig, rows: int, seed_offset: int) -> np.ndarray:
    """Extra activation batches with the same channel structure (outlier channels of ``cfg``)."""
    base = np.random.default_rng(cfg.seed)
    base.standard_normal((cfg.b, cfg.m))  # advance past the calibration batch
    n_out = cfg.outlier_count if cfg.outlier_count is not None else int(round(cfg.outlier_frac * cfg.m))
    ch = np.sort(base.choice(cfg.m, size=n_out, replace=False)) if n_out > 0 else np.zeros(0, np.int64)
    rng = np.random.default_rng([cfg.seed, seed_offset])
    x = rng.standard_normal((rows, cfg.m))
    if cfg.gelu_x:
        x = _gelu_erf(x)
    x[:, ch] *= cfg.outlier_mult
    return to_bf16(x)


def random_matrix(rng: np.random.Generator, shape, scale=1.0, dtype=np.float32) -> np.ndarray:
    return (rng.standard_normal(shape) * scale).astype(dtype)
