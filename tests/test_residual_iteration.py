"""Residual iteration of the offline split (no GPU).

AutoRound "SVDQuant（实验性功能）", "Residual iteration": starting from the
plain SVD split, each outer iteration fits the low-rank branch to
W_tilde - Q(R_prev) and quantize-dequantizes the new residual as it is
deployed; early stop keeps the best candidate and stops once the target error
gets worse.  The target is the weight reconstruction error with smoothing off
and the calibration output error with smoothing on.

Pins of the CPU reference: the plain split at one iteration, Eckart-Young for
every refit (checked with scipy's singular values on the matrix the refit must
see), the target recomputed through the weight pack's quantizer, the early-stop
rule on a case where every candidate ties (rank 0), and an exactly
representable layer.  The PyTorch offline path is checked against the
reference: its quantize-dequantize bit for bit, its iteration to rounding.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as O
from bit_w4a4_quantized_group_b200 import inputs as I
from bit_w4a4_quantized_group_b200 import prepare as P

FMTS = ["int4", "nvfp4", "mxfp4", "w8a8"]


@pytest.fixture(scope="module")
def tiny():
    layer = I.make_layer(I.TINY)
    lam = O.smoothing_factors(layer.X, layer.W)
    return layer, lam, O.smooth_weight(layer.W, lam), O.smooth_activations(layer.X, lam)


def _deployed_qdq(fmt, R_kn):
    """Q(R) through the weight pack (per output channel along K), [K, N] fp64."""
    pk = O.pack_weight(fmt, np.ascontiguousarray(R_kn.T), None, None, 1.0)
    return O.dequantize(fmt, pk["q"]).T


# ----------------------------------------------------------- reference pins

@pytest.mark.parametrize("fmt", FMTS)
def test_one_iteration_is_the_plain_split(tiny, fmt):
    _, _, Wt, _ = tiny
    ri = O.residual_iteration(fmt, Wt, 16, 1)
    sp = O.svd_split(Wt, 16)
    assert np.array_equal(ri["L1_bf16"], sp["L1_bf16"])
    assert np.array_equal(ri["L2_bf16"], sp["L2_bf16"])
    assert np.array_equal(ri["R"], sp["R"])
    assert ri["chosen"] == 0 and len(ri["errors"]) == 1


@pytest.mark.parametrize("fmt", FMTS)
def test_each_refit_is_the_best_rank_r_fit_of_w_minus_qr(tiny, fmt):
    """Iteration i's branch is an optimal rank-r fit (to bf16 rounding) of W - Q(R_{i-1})."""
    _, _, Wt, _ = tiny
    r = 16
    prev = O.residual_iteration(fmt, Wt, r, 1)
    for it in (1, 2):
        QR = _deployed_qdq(fmt, prev["R"].astype(np.float64))
        T = Wt - QR
        s = scipy.linalg.svdvals(T)
        opt = np.sqrt(np.sum(s[r:] ** 2))
        cur = O.residual_iteration(fmt, Wt, r, it + 1)
        assert len(cur["errors"]) == it + 1 and cur["chosen"] == it
        fit = np.linalg.norm(T - cur["L1_bf16"] @ cur["L2_bf16"])
        # bf16 factors cost at most a few 2^-9 relative of the branch
        slack = 4 * 2.0 ** -9 * np.linalg.norm(cur["L1_bf16"] @ cur["L2_bf16"])
        assert opt <= fit + 1e-9 and fit <= opt + slack
        # a fit to W - R_{i-1} (Q dropped) would give back the previous branch (for the 4-bit
        # formats Q moves R far more than the bf16 rounding of the factors; for W8A8 it does not)
        stale = np.linalg.norm(T - prev["L1_bf16"] @ prev["L2_bf16"])
        if fmt != "w8a8":
            assert fit < stale
        # the new residual is W_tilde minus the new branch, in fp32
        assert np.array_equal(cur["R"], (Wt - cur["L1_bf16"] @ cur["L2_bf16"]).astype(np.float32))
        prev = cur


@pytest.mark.parametrize("fmt", FMTS)
def test_target_errors_recomputed_through_the_pack(tiny, fmt):
    _, _, Wt, Xh = tiny
    for iters in (1, 2, 3):
        for xh in (None, Xh):
            ri = O.residual_iteration(fmt, Wt, 16, iters, X_hat=xh)
            E = ri["L1_bf16"] @ ri["L2_bf16"] + _deployed_qdq(fmt, ri["R"].astype(np.float64)) - Wt
            want = np.linalg.norm(E if xh is None else xh.astype(np.float64) @ E)
            assert ri["errors"][-1] == pytest.approx(want, rel=1e-12)


def test_output_error_scales_with_the_calibration_set(tiny):
    _, _, Wt, _ = tiny
    eye = np.eye(Wt.shape[0])
    a = O.residual_iteration("nvfp4", Wt, 16, 3)
    b = O.residual_iteration("nvfp4", Wt, 16, 3, X_hat=4.0 * eye)
    assert np.allclose(b["errors"], 4.0 * np.asarray(a["errors"]), rtol=1e-12)


@pytest.mark.parametrize("fmt", FMTS)
def test_early_stop_on_ties_keeps_the_first_candidate(tiny, fmt):
    """Rank 0: every candidate is the same, so the second is not better and the loop stops."""
    _, _, Wt, _ = tiny
    es = O.residual_iteration(fmt, Wt, 0, 6, early_stop=True)
    assert es["chosen"] == 0 and len(es["errors"]) == 2
    assert es["errors"][0] == es["errors"][1]
    assert es["errors"][0] == pytest.approx(np.linalg.norm(_deployed_qdq(fmt, Wt) - Wt), rel=1e-12)
    full = O.residual_iteration(fmt, Wt, 0, 6, early_stop=False)
    assert full["chosen"] == 5 and len(full["errors"]) == 6


@pytest.mark.parametrize("fmt", FMTS)
def test_early_stop_keeps_the_best_prefix_candidate(tiny, fmt):
    _, _, Wt, Xh = tiny
    for xh in (None, Xh):
        es = O.residual_iteration(fmt, Wt, 16, 6, early_stop=True, X_hat=xh)
        e = np.asarray(es["errors"])
        assert es["chosen"] == int(np.argmin(e))
        assert np.all(np.diff(e[:-1]) < 0)                        # improved until the last one
        assert len(e) == 6 or e[-1] >= e[-2]                       # stopped only on a worse one
        assert e[es["chosen"]] <= e[0]


def test_exactly_representable_layer_has_zero_error():
    """W_tilde = L1 L2 with bf16 factors and orthogonal structure: the split is exact to SVD rounding."""
    K, N, r = 128, 128, 4
    L1 = np.zeros((K, r))
    L2 = np.zeros((r, N))
    for i, (row, col, s) in enumerate([(3, 70, 8.0), (40, 5, 4.0), (90, 100, 2.0), (127, 0, 1.0)]):
        L1[row, i] = s
        L2[i, col] = 1.0
    Wt = L1 @ L2
    for fmt in FMTS:
        es = O.residual_iteration(fmt, Wt, r, 4, early_stop=True)
        assert max(es["errors"]) <= 1e-13 * np.linalg.norm(Wt)
        assert np.abs(es["L1_bf16"] @ es["L2_bf16"] - Wt).max() <= 2.0 ** -8 * 8.0
        assert np.abs(es["R"]).max() <= 1e-13


def test_iterations_lower_the_target_on_a_seeded_layer(tiny):
    """The purpose of the iteration: a better weight and output fit than the plain split."""
    _, _, Wt, Xh = tiny
    for fmt in FMTS:
        w = O.residual_iteration(fmt, Wt, 16, 4, early_stop=True)
        o = O.residual_iteration(fmt, Wt, 16, 4, early_stop=True, X_hat=Xh)
        assert w["errors"][w["chosen"]] < 0.97 * w["errors"][0]
        assert o["errors"][o["chosen"]] < 0.97 * o["errors"][0]


def test_prepare_layer_uses_output_error_when_smoothing(tiny):
    layer, lam, Wt, Xh = tiny
    prep = O.prepare_layer("nvfp4", layer.X, layer.W, 16, residual_iters=3, early_stop=True)
    ri = O.residual_iteration("nvfp4", Wt, 16, 3, True, Xh)
    assert prep["split"]["residual"]["errors"] == ri["errors"]
    assert np.array_equal(prep["R_nk"], np.ascontiguousarray(ri["R"].T))
    prep_w = O.prepare_layer("nvfp4", layer.X, layer.W, 16, smooth=False, residual_iters=3)
    ri_w = O.residual_iteration("nvfp4", layer.W, 16, 3)
    assert prep_w["split"]["residual"]["errors"] == ri_w["errors"]


# ------------------------------------------------------ PyTorch offline path

def _qdq_cases(fmt):
    rng = np.random.default_rng(7)
    N, K = 128, 256
    out = []
    for e in (-20, -6, 0, 5):
        R = (rng.standard_normal((N, K)) * 2.0 ** e).astype(np.float32)
        R[rng.random((N, K)) < 0.02] *= 50
        out.append(R)
    R = np.zeros((N, K), np.float32)
    R[:, 0] = 6.0
    R[:, 1:11] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -2.5, -5.0]
    R[1, :] = -0.0
    R[2, 0:64] = 7.0
    R[2, 1:6] = [0.5, 1.5, 2.5, -0.5, -3.5]
    R[4, :] = 2.0 ** -140
    R[5, 32:64] = 3.0e38
    R[6, :16] = np.float32(6.0 * 448.0 * 2.0 ** -10) * np.linspace(-1, 1, 16, dtype=np.float32)
    out.append(R)
    return out


@pytest.mark.parametrize("fmt", FMTS)
def test_torch_qdq_is_the_pack_quantizer_bit_for_bit(fmt):
    for R in _qdq_cases(fmt):
        if fmt == "int4" and np.abs(R).max() > 1e30:
            R = np.where(np.abs(R) > 1e30, np.float32(1e4), R)
        want = _deployed_qdq(fmt, R.T.astype(np.float64)).T
        gw = O.pow2_global_scale(np.abs(R).max()) if fmt == "nvfp4" else 1.0
        want2 = O.dequantize(fmt, O.quantize(fmt, R, gw))
        got = P.qdq_weight(fmt, torch.from_numpy(R)).numpy()
        assert np.array_equal(want, want2)
        assert np.array_equal(np.signbit(got), np.signbit(want))        # signed zeros too
        assert np.array_equal(got, want), np.abs(got - want).max()


@pytest.mark.parametrize("fmt", FMTS)
def test_torch_iteration_follows_the_reference(tiny, fmt):
    _, _, Wt, Xh = tiny
    ref = O.residual_iteration(fmt, Wt, 16, 3, early_stop=True, X_hat=Xh)
    L1, L2, R, chosen, errs = P.residual_iteration(fmt, torch.from_numpy(Wt), 16, 3, True,
                                                   torch.from_numpy(Xh.astype(np.float64)))
    assert chosen == ref["chosen"] and len(errs) == len(ref["errors"])
    assert np.allclose(errs, ref["errors"], rtol=2e-4)
    # the returned residual is W_tilde minus the returned branch
    assert torch.equal(R, (torch.from_numpy(Wt) - L1 @ L2).to(torch.float32))
    d = np.linalg.norm((L1 @ L2).numpy() - ref["L1_bf16"] @ ref["L2_bf16"])
    assert d <= 1e-2 * np.linalg.norm(ref["L1_bf16"] @ ref["L2_bf16"])


def test_torch_prepare_one_iteration_unchanged(tiny):
    layer = tiny[0]
    a = P.prepare("nvfp4", layer.X, layer.W, 16, device="cpu")
    b = P.prepare("nvfp4", layer.X, layer.W, 16, device="cpu", residual_iters=3, early_stop=True)
    assert a["residual"] == {} and b["residual"]["chosen"] >= 1
    ref = O.prepare_layer("nvfp4", layer.X, layer.W, 16)
    assert np.array_equal(a["lam"], ref["lam"])
    assert a["act_gscale"] == b["act_gscale"] == ref["act_gscale"]
    # the iterated split packs to a layer with a smaller calibration output error
    errs = b["residual"]["errors"]
    assert errs[b["residual"]["chosen"]] < errs[0]


def test_planted_dropped_quantizer_is_caught(tiny):
    """An iteration that refits to W_tilde - R_prev (Q dropped) returns the previous branch;
    the refit pin (strictly better than the stale branch) catches it."""
    _, _, Wt, _ = tiny
    fmt, r = "nvfp4", 16
    prev = O.residual_iteration(fmt, Wt, r, 1)
    # the planted mistake, written out: refit to W_tilde - R instead of W_tilde - Q(R)
    wrong = O.svd_split(Wt - prev["R"].astype(np.float64), r)
    T = Wt - _deployed_qdq(fmt, prev["R"].astype(np.float64))
    fit_wrong = np.linalg.norm(T - wrong["L1_bf16"] @ wrong["L2_bf16"])
    stale = np.linalg.norm(T - prev["L1_bf16"] @ prev["L2_bf16"])
    assert not fit_wrong < stale * (1 - 1e-3)          # the pin would fail on it
    cur = O.residual_iteration(fmt, Wt, r, 2)
    assert np.linalg.norm(T - cur["L1_bf16"] @ cur["L2_bf16"]) < stale


def test_offline_tensor_scale_matches_the_reference():
    """prepare.py's power-of-two tensor scale (reading 4) against the reference's, at the
    exact boundaries 6 * 448 * 2^e, one ulp either side of them, zero and random values."""
    rng = np.random.default_rng(55)
    vals = [0.0, 1e-30, 3.0e38]
    for e in range(-40, 40, 3):
        b = 6.0 * 448.0 * 2.0 ** e
        vals += [b, float(np.nextafter(np.float32(b), np.float32(np.inf))),
                 float(np.nextafter(np.float32(b), np.float32(0)))]
    vals += list(np.exp(rng.uniform(-60, 60, 200)))
    for v in vals:
        v32 = float(np.float32(v))
        assert P.pow2_tensor_scale(v32) == O.pow2_global_scale(v32), v32


def test_offline_prepare_matches_the_reference_split(tiny):
    """prepare.py (PyTorch, fp64 SVD) against the reference's prepare_layer on the same layer:
    lambda and g_x bit for bit, the bf16 factors' product and the residual to SVD rounding."""
    layer = tiny[0]
    for fmt in FMTS:
        a = P.prepare(fmt, layer.X, layer.W, 16, device="cpu")
        ref = O.prepare_layer(fmt, layer.X, layer.W, 16)
        assert np.array_equal(a["lam"], ref["lam"]) and a["act_gscale"] == ref["act_gscale"]
        prod = a["L2_nr"].astype(np.float64) @ a["L1_rk"].astype(np.float64)
        prod_ref = ref["L2_nr"] @ ref["L1_rk"]
        assert np.linalg.norm(prod - prod_ref) <= 1e-2 * np.linalg.norm(prod_ref)
        assert np.linalg.norm(a["R_nk"] - ref["R_nk"]) <= 2e-2 * np.linalg.norm(ref["R_nk"]) + 1e-6
