"""Helpers of the GPU parity tests: run the library through the C ABI on
seeded inputs and bring results back in canonical form."""
import numpy as np
import torch

from bit_w4a4_quantized_group_b200 import binding as B

from layouts import (bf16_bits_to_f32, blocked_scale_offsets, codes_canonical, f32_to_bf16_bits_exact,
                     scales_canonical, scales_padding)


def dev_bf16(x: np.ndarray) -> torch.Tensor:
    """float32 array of exact bf16 values -> device bf16 tensor (bit exact)."""
    bits = f32_to_bf16_bits_exact(np.ascontiguousarray(x, np.float32))
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def host_bf16(t: torch.Tensor) -> np.ndarray:
    return bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def check_device_error():
    torch.cuda.synchronize()
    st, site = B.svdq_get_last_device_error(None)
    assert st == B.SVDQ_OK, f"device error status {st} at wait site {site}"


def run_prologue(fmt, X, lam, gx, L1_rk, fill=0x5A):
    M, K = X.shape
    r = 0 if L1_rk is None else L1_rk.shape[0]
    sz = B.svdq_buffer_sizes(fmt, M, 128, K, r)
    Xd = dev_bf16(X)
    lam_d = None if lam is None else torch.from_numpy(np.ascontiguousarray(lam, np.float32)).cuda()
    L1d = dev_bf16(L1_rk) if r > 0 else None
    codes = torch.full((sz.a_codes,), fill, dtype=torch.uint8, device="cuda")
    scales = torch.full((sz.a_scales,), fill, dtype=torch.uint8, device="cuda")
    Z = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda") if r > 0 else None
    B.quantize_act_lowrank_down_t(fmt, Xd, lam_d, gx, L1d, codes, scales, Z)
    check_device_error()
    sc = scales.cpu().numpy()
    return {
        "codes": codes_canonical(fmt, codes.cpu().numpy(), M, K),
        "scales": scales_canonical(fmt, sc, M, K),
        "scale_padding": scales_padding(fmt, sc, M, K),
        "Z": host_bf16(Z) if r > 0 else np.zeros((M, 0), np.float32),
        "dev": {"codes": codes, "scales": scales, "Z": Z},
    }


def encode_scales(fmt, scale_bits: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Canonical scale bits [rows][G] -> library buffer bytes (padding rows zero)."""
    rp = (rows + 127) // 128 * 128
    if fmt == "w8a8":
        buf = np.zeros(rp, np.uint32)
        buf[:rows] = np.asarray(scale_bits, np.uint32).reshape(rows)
        return buf.view(np.uint8)
    if fmt in ("nvfp4", "mxfp4"):
        g = 16 if fmt == "nvfp4" else 32
        buf = np.zeros(rp * K // g, np.uint8)
        buf[blocked_scale_offsets(rows, K, g)] = scale_bits
        return buf
    buf = np.zeros((K // 64, rp), np.uint16)
    buf[:, :rows] = scale_bits.T
    return buf.view(np.uint8).reshape(-1)


def pack_codes_bytes(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8).reshape(-1)


def codes_bytes(fmt, codes: np.ndarray) -> np.ndarray:
    """Canonical codes -> library code buffer (nibble pairs, or one byte each for W8A8)."""
    if fmt == "w8a8":
        return np.ascontiguousarray(codes, np.uint8).reshape(-1)
    return pack_codes_bytes(codes)


def run_gemm(fmt, M, N, K, rank, a_codes, a_scales, gx, w_codes, w_scales, gw, Z, L2s, bias, y_offset=0):
    """All operand arguments are host NumPy buffers in library layout (or device tensors).
    y_offset: Y starts that many bf16 elements into a larger buffer (8: 16-byte but not
    32-byte aligned)."""
    def d(x):
        if x is None:
            return None
        if isinstance(x, torch.Tensor):
            return x
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()
    Ybuf = torch.full((M * N + y_offset,), float("nan"), dtype=torch.bfloat16, device="cuda")
    Y = Ybuf[y_offset:].view(M, N)
    B.w4a4_gemm_lowrank_up_t(fmt, M, N, K, rank, d(a_codes), d(a_scales), gx, d(w_codes), d(w_scales), gw,
                             None if rank == 0 else (Z if isinstance(Z, torch.Tensor) else dev_bf16(Z)),
                             None if rank == 0 else (L2s if isinstance(L2s, torch.Tensor) else dev_bf16(L2s)),
                             None if bias is None else (bias if isinstance(bias, torch.Tensor) else dev_bf16(bias)),
                             Y)
    check_device_error()
    return Y


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def y_elementwise_slack(qa, gx, qw, gw, Z, L2_nr, bias):
    """Sum of absolute terms of every output element, in fp64: the scale of the fp32
    accumulation error the GPU may add (g_x g_w |Q(X_hat)| |Q(R)|^T + |Z| |L2|^T + |bias|)."""
    import oracle as O
    fmt_g = qa["q"].shape[1] // qa["scale"].shape[1]
    xa = np.abs(qa["q"] * np.repeat(qa["scale"].astype(np.float64), fmt_g, axis=1))
    wb = np.abs(qw["q"] * np.repeat(qw["scale"].astype(np.float64), fmt_g, axis=1))
    S = gx * gw * (xa @ wb.T)
    if Z is not None and np.asarray(Z).shape[1] > 0:
        S = S + np.abs(np.asarray(Z, np.float64)) @ np.abs(np.asarray(L2_nr, np.float64)).T
    if bias is not None:
        S = S + np.abs(np.asarray(bias, np.float64))[None, :]
    return S


def assert_y_elementwise(Yg, Y64, S):
    """Every element within one bf16 ulp of the fp64 value plus 2^-16 of its absolute terms."""
    from layouts import bf16_ulp
    err = np.abs(np.asarray(Yg, np.float64) - Y64)
    tol = bf16_ulp(Y64) + 2.0 ** -16 * S
    assert np.all(err <= tol), f"max excess {np.max(err - tol)} at {np.unravel_index(np.argmax(err - tol), err.shape)}"
