"""The C ABI on the host: exports, argument checks, and the host pack (no GPU).

svdq_pack_weight runs on the CPU, so its codes and scales are compared bit
for bit with the CPU reference here.  Device calls are only made with
invalid arguments, which must be rejected before any launch.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from bit_w4a4_quantized_group_b200 import binding as B
from bit_w4a4_quantized_group_b200 import build as BUILD
from bit_w4a4_quantized_group_b200 import inputs as I

from layouts import (codes_canonical, int4_scales_canonical, nvfp4_scales_canonical, scales_canonical, scales_padding,
                     unpack_codes)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.load()


def _header_functions():
    txt = open(os.path.join(ROOT, "include", "svdq.h"), encoding="utf-8").read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol(lib):
    names = _header_functions()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTED)


def test_buffer_sizes(lib):
    s = B.svdq_buffer_sizes("nvfp4", 300, 640, 768, 32)
    assert s.a_codes == 300 * 384 and s.w_codes == 640 * 384
    assert s.a_scales == 384 * 768 // 16          # rows padded to 384
    assert s.w_scales == 640 * 768 // 16
    assert s.z == 300 * 32 * 2 and s.l1 == 32 * 768 * 2 and s.l2 == 640 * 32 * 2
    assert s.y == 300 * 640 * 2 and s.bias == 640 * 2
    s = B.svdq_buffer_sizes("int4", 300, 640, 768, 0)
    assert s.a_scales == 384 * (768 // 64) * 2 and s.z == 0
    s = B.svdq_buffer_sizes("w8a8", 300, 640, 768, 16)
    assert s.a_codes == 300 * 768 and s.w_codes == 640 * 768
    assert s.a_scales == 384 * 4 and s.w_scales == 640 * 4
    assert s.z == 300 * 16 * 2 and s.l2 == 640 * 16 * 2


@pytest.mark.parametrize("args", [
    ("nvfp4", 0, 256, 256, 16),      # M < 1
    ("nvfp4", 64, 200, 256, 16),     # N % 128
    ("nvfp4", 64, 256, 192, 16),     # K % 128
    ("nvfp4", 64, 256, 256, 24),     # rank % 16
    ("nvfp4", 64, 256, 256, 144),    # rank > 128
    (7, 64, 256, 256, 16),           # bad format
])
def test_buffer_sizes_rejects(lib, args):
    with pytest.raises(B.SvdqError) as e:
        B.svdq_buffer_sizes(*args)
    assert e.value.status == B.SVDQ_ERR_INVALID_ARG


def _bufs(n=8):
    return [np.zeros(1 << 16, np.uint8) for _ in range(n)]


def test_device_calls_reject_bad_arguments_without_launch(lib):
    b = _bufs()
    p = [x.ctypes.data for x in b]
    # bad K
    st = B.svdq_quantize_act_lowrank_down("nvfp4", 64, 200, 16, p[0], None, 1.0, p[1], p[2], p[3], p[4], None)
    assert st == B.SVDQ_ERR_INVALID_ARG and B.svdq_last_launch_count() == 0
    # NULL X
    st = B.svdq_quantize_act_lowrank_down("nvfp4", 64, 256, 16, None, None, 1.0, p[1], p[2], p[3], p[4], None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    # misaligned codes pointer
    st = B.svdq_quantize_act_lowrank_down("nvfp4", 64, 256, 16, p[0], None, 1.0, p[1], p[2] + 1, p[3], p[4], None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    # non power-of-two activation scale
    st = B.svdq_quantize_act_lowrank_down("nvfp4", 64, 256, 16, p[0], None, 3.0, p[1], p[2], p[3], p[4], None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    # INT4 requires unit tensor scales
    st = B.svdq_quantize_act_lowrank_down("int4", 64, 256, 16, p[0], None, 2.0, p[1], p[2], p[3], p[4], None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    # rank > 0 needs Z and L1
    st = B.svdq_quantize_act_lowrank_down("nvfp4", 64, 256, 16, p[0], None, 1.0, None, p[2], p[3], p[4], None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    # GEMM: bad N, missing Y, misaligned bias, non power-of-two weight scale
    args = dict(a=p[0], sa=p[1], w=p[2], sw=p[3], z=p[4], l2=p[5], bias=p[6], y=p[7])
    st = B.svdq_w4a4_gemm_lowrank_up("nvfp4", 64, 200, 256, 16, args["a"], args["sa"], 1.0, args["w"],
                                     args["sw"], 1.0, args["z"], args["l2"], args["bias"], args["y"], None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    st = B.svdq_w4a4_gemm_lowrank_up("nvfp4", 64, 256, 256, 16, args["a"], args["sa"], 1.0, args["w"],
                                     args["sw"], 1.0, args["z"], args["l2"], args["bias"], None, None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    st = B.svdq_w4a4_gemm_lowrank_up("nvfp4", 64, 256, 256, 16, args["a"], args["sa"], 1.0, args["w"],
                                     args["sw"], 1.0, args["z"], args["l2"], args["bias"] + 2, args["y"], None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    st = B.svdq_w4a4_gemm_lowrank_up("nvfp4", 64, 256, 256, 16, args["a"], args["sa"], 1.0, args["w"],
                                     args["sw"], 0.75, args["z"], args["l2"], args["bias"], args["y"], None)
    assert st == B.SVDQ_ERR_INVALID_ARG
    assert B.svdq_last_launch_count() == 0


def test_status_strings(lib):
    assert B.status_name(B.SVDQ_OK) == "ok"
    assert "timed out" in B.status_name(B.SVDQ_ERR_TIMEOUT)


# ----------------------------------------------------------------- host pack parity

def _check_pack(fmt, R_nk, L1_rk, L2_nr, gx):
    N, K = R_nk.shape
    got = B.pack_weight_np(fmt, R_nk, L1_rk, L2_nr, gx)
    ref = O.pack_weight(fmt, R_nk, L1_rk, L2_nr, gx)
    assert got["w_gscale"] == ref["gscale"]
    assert np.array_equal(codes_canonical(fmt, got["w_codes"], N, K), ref["q"]["codes"])
    assert np.array_equal(scales_canonical(fmt, got["w_scales"], N, K), ref["q"]["scale_bits"])
    assert np.all(scales_padding(fmt, got["w_scales"], N, K) == 0)
    if L1_rk is not None and L1_rk.shape[0] > 0:
        l1 = (got["L1_bf16"].astype(np.uint32) << 16).view(np.float32)
        l2 = (got["L2_bf16"].astype(np.uint32) << 16).view(np.float32)
        assert np.array_equal(l1, ref["L1_bf16"])
        assert np.array_equal(l2, ref["L2_scaled"])


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
def test_pack_weight_matches_reference_on_tiny_layer(lib, fmt):
    layer = I.make_layer(I.TINY)
    prep = O.prepare_layer(fmt, layer.X, layer.W, 16)
    _check_pack(fmt, prep["R_nk"], prep["L1_rk"].astype(np.float32), prep["L2_nr"].astype(np.float32),
                prep["act_gscale"])


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "w8a8"])
@pytest.mark.parametrize("scale_exp", [-12, -3, 0, 6])
def test_pack_weight_matches_reference_random(lib, fmt, scale_exp):
    rng = np.random.default_rng(100 + scale_exp)
    N, K, r = 256, 384, 32
    R = (rng.standard_normal((N, K)) * 2.0 ** scale_exp).astype(np.float32)
    # heavy-tailed entries, exact zeros and a zero group
    R[rng.random((N, K)) < 0.01] *= 40
    R[3, :] = 0.0
    R[5, 64:128] = 0.0
    L1 = rng.standard_normal((r, K)).astype(np.float32)
    L2 = (rng.standard_normal((N, r)) * 0.1).astype(np.float32)
    gx = 2.0 ** -7 if fmt == "nvfp4" else 1.0
    _check_pack(fmt, R, L1, L2, gx)


def test_pack_weight_rank0_and_ties(lib):
    # values placed exactly on E2M1 / INT4 rounding midpoints after scaling
    N, K = 128, 128
    R = np.zeros((N, K), np.float32)
    R[:, 0] = 6.0
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -2.5, -0.1], np.float32)
    R[:, 1:1 + len(mids)] = mids
    _check_pack("nvfp4", R, None, None, 1.0)
    R2 = np.zeros((N, K), np.float32)
    R2[:, 0] = 7.0
    R2[:, 1:6] = [0.5, 1.5, 2.5, -0.5, -3.5]
    _check_pack("int4", R2, None, None, 1.0)
    # MXFP4: amax 6 gives X = 1 and the same E2M1 midpoints; amax 7 saturates; a tiny group
    _check_pack("mxfp4", R, None, None, 1.0)
    R3 = np.zeros((N, K), np.float32)
    R3[:, 0] = 7.0
    R3[:, 1:5] = [0.25, -0.75, 3.5, 5.0]
    R3[:, 32] = 2.0 ** -140
    R3[:, 64] = -0.0
    _check_pack("mxfp4", R3, None, None, 1.0)
    # W8A8: max 127 gives s = 1 and the midpoints round to even; a tiny row has a subnormal scale
    R4 = np.zeros((N, K), np.float32)
    R4[:, 0] = 127.0
    R4[:, 1:7] = [0.5, 1.5, 2.5, -0.5, -126.5, 0.49]
    R4[5, :] = 0.0
    R4[6, :3] = [1e-40, -3e-41, 7e-42]
    R4[7, :] = -0.0
    _check_pack("w8a8", R4, None, None, 1.0)


def test_pack_weight_rejects(lib):
    N, K = 128, 128
    R = np.zeros((N, K), np.float32)
    with pytest.raises(B.SvdqError):
        B.pack_weight_np("nvfp4", R, None, None, 3.0)     # not a power of two
    with pytest.raises(B.SvdqError):
        B.pack_weight_np("int4", R, None, None, 0.5)      # INT4 needs g_x = 1
    with pytest.raises(B.SvdqError):
        B.pack_weight_np("mxfp4", R, None, None, 2.0)     # MXFP4 has no tensor scale
    with pytest.raises(B.SvdqError):
        B.pack_weight_np("w8a8", R, None, None, 2.0)      # nor has W8A8


def test_selftest_rejects_limits_out_of_range():
    # argument checks run before any CUDA call
    assert B.svdq_selftest_bounded_wait(10, None) == B.SVDQ_ERR_INVALID_ARG
    assert B.svdq_selftest_bounded_wait(10_000_000_000, None) == B.SVDQ_ERR_INVALID_ARG


# ------------------------------------------------------- randomized host pack parity

from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st


@settings(max_examples=30, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(fmt=st.sampled_from(["nvfp4", "int4", "mxfp4", "w8a8"]),
       nb=st.integers(1, 3), kb=st.integers(1, 4), rank=st.sampled_from([0, 16, 32]),
       exp=st.integers(-30, 20), dist=st.sampled_from(["normal", "heavy", "uniform", "sparse"]),
       seed=st.integers(0, 2 ** 31 - 1))
def test_pack_weight_matches_reference_randomized(lib, fmt, nb, kb, rank, exp, dist, seed):
    """Shapes, magnitudes and distributions drawn at random; codes, scales, g_w and the
    factors must match the CPU reference bit for bit."""
    rng = np.random.default_rng(seed)
    N, K = 128 * nb, 128 * kb
    if dist == "normal":
        R = rng.standard_normal((N, K))
    elif dist == "heavy":
        R = rng.standard_t(2.0, (N, K))
    elif dist == "uniform":
        R = rng.uniform(-1, 1, (N, K))
    else:
        R = rng.standard_normal((N, K)) * (rng.random((N, K)) < 0.05)
    R = (R * 2.0 ** exp).astype(np.float32)
    L1 = rng.standard_normal((rank, K)).astype(np.float32) if rank else None
    L2 = (rng.standard_normal((N, rank)) * 0.1).astype(np.float32) if rank else None
    gx = 2.0 ** int(rng.integers(-8, 3)) if fmt == "nvfp4" else 1.0
    _check_pack(fmt, R, L1, L2, gx)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """No CPU fallback: without the built library the binding raises instead of computing."""
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="libsvdq.so not found"):
        B.load(str(tmp_path / "libsvdq.so"))
    import oracle  # noqa: F401  (the reference is importable, but the product path never uses it)
    import bit_w4a4_quantized_group_b200.layer as L
    src = open(L.__file__, encoding="utf-8").read() + open(B.__file__, encoding="utf-8").read()
    assert "oracle" not in src
