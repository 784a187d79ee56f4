"""Decoders from the library's buffer layouts to canonical arrays.

Written from the layout text of include/svdq.h (index functions), separately
from the library and from the CPU reference; used only by tests.
"""
import numpy as np


def unpack_codes(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """[rows][K/2] bytes, element k in the low nibble of byte k/2 when k is even."""
    b = np.asarray(buf, np.uint8).reshape(rows, K // 2)
    out = np.empty((rows, K), np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def pack_codes(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def blocked_scale_offsets(rows: int, K: int, g: int = 16) -> np.ndarray:
    """Byte offset of (row, group) in the 128x4 blocked scale layout, groups of g elements."""
    r = np.arange(rows)[:, None]
    grp = np.arange(K // g)[None, :]
    return ((r // 128) * (K // (4 * g)) + grp // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + grp % 4


def nvfp4_scale_offsets(rows: int, K: int) -> np.ndarray:
    return blocked_scale_offsets(rows, K, 16)


def blocked_scales_canonical(buf: np.ndarray, rows: int, K: int, g: int = 16) -> np.ndarray:
    b = np.asarray(buf, np.uint8).reshape(-1)
    return b[blocked_scale_offsets(rows, K, g)]


def nvfp4_scales_canonical(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    return blocked_scales_canonical(buf, rows, K, 16)


def blocked_scales_padding(buf: np.ndarray, rows: int, K: int, g: int = 16) -> np.ndarray:
    """Bytes of the padding rows (rows .. ceil(rows/128)*128 - 1)."""
    rp = (rows + 127) // 128 * 128
    if rp == rows:
        return np.zeros(0, np.uint8)
    b = np.asarray(buf, np.uint8).reshape(-1)
    off = blocked_scale_offsets(rp, K, g)[rows:]
    return b[off]


def nvfp4_scales_padding(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    return blocked_scales_padding(buf, rows, K, 16)


def int4_scales_canonical(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """fp16 [K/64][Rp] group-major -> uint16 bits [rows][K/64]."""
    rp = (rows + 127) // 128 * 128
    b = np.asarray(buf).view(np.uint16).reshape(K // 64, rp)
    return b[:, :rows].T.copy()


def int4_scales_padding(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    rp = (rows + 127) // 128 * 128
    b = np.asarray(buf).view(np.uint16).reshape(K // 64, rp)
    return b[:, rows:].copy()


def row_scales_canonical(buf, rows: int) -> np.ndarray:
    """W8A8: fp32 [Rp] -> uint32 bits [rows][1]."""
    b = np.asarray(buf).reshape(-1).view(np.uint32)
    return b[:rows].reshape(rows, 1).copy()


def row_scales_padding(buf, rows: int) -> np.ndarray:
    rp = (rows + 127) // 128 * 128
    return np.asarray(buf).reshape(-1).view(np.uint32)[rows:rp].copy()


def codes_canonical(fmt: str, buf, rows: int, K: int) -> np.ndarray:
    """Codes as the reference returns them: nibbles for the 4-bit formats, bytes for W8A8."""
    if fmt == "w8a8":
        return np.asarray(buf, np.uint8).reshape(-1)[: rows * K].reshape(rows, K).copy()
    return unpack_codes(np.asarray(buf, np.uint8).reshape(-1)[: rows * K // 2], rows, K)


def scales_canonical(fmt: str, buf, rows: int, K: int) -> np.ndarray:
    if fmt == "int4":
        return int4_scales_canonical(buf, rows, K)
    if fmt == "w8a8":
        return row_scales_canonical(buf, rows)
    return blocked_scales_canonical(buf, rows, K, 16 if fmt == "nvfp4" else 32)


def scales_padding(fmt: str, buf, rows: int, K: int) -> np.ndarray:
    if fmt == "int4":
        return int4_scales_padding(buf, rows, K)
    if fmt == "w8a8":
        return row_scales_padding(buf, rows)
    return blocked_scales_padding(buf, rows, K, 16 if fmt == "nvfp4" else 32)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits_exact(x: np.ndarray) -> np.ndarray:
    """Bits of float32 values that are exact bf16 values (asserts exactness)."""
    x = np.ascontiguousarray(x, np.float32)
    u = x.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value is not a bf16 value"
    return (u >> 16).astype(np.uint16)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)
