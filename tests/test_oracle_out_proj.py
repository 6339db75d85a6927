"""Pins of the SSD-epilogue oracle (RMSNorm + INT8 out projection + mean correction), CPU."""
import numpy as np
import pytest

from oracle import out_proj as O


def _data(seed, T=256, K=128, D=48, outliers=True):
    rs = np.random.default_rng(seed)
    y = rs.standard_normal((T, K))
    if outliers:
        y[:, rs.choice(K, 3, replace=False)] *= 20.0
    gamma = rs.uniform(0.5, 1.5, K)
    W = rs.standard_normal((D, K)) / np.sqrt(K)
    return y, gamma, W


def test_rmsnorm_closed_forms():
    y = np.array([[3.0, 4.0], [0.0, 0.0], [-2.0, 2.0]])
    u = O.rmsnorm(y, eps=0.0 + 1e-300)
    np.testing.assert_allclose(u[0], [3 / np.sqrt(12.5), 4 / np.sqrt(12.5)])
    np.testing.assert_allclose(u[2], [-1.0, 1.0])
    np.testing.assert_array_equal(O.rmsnorm(np.zeros((1, 4))), np.zeros((1, 4)))   # eps keeps 0 finite
    # scale invariance (up to eps)
    y2, _, _ = _data(0, outliers=False)
    np.testing.assert_allclose(O.rmsnorm(7.0 * y2, eps=0.0 + 1e-300), O.rmsnorm(y2, eps=0.0 + 1e-300), rtol=1e-12)


def test_gamma_migration_is_an_identity_in_fp64():
    y, gamma, W = _data(1)
    np.testing.assert_allclose(O.out_proj_fp64(y, gamma, W), O.rmsnorm(y) @ (W * gamma[None, :]).T, rtol=1e-12)


def test_mean_correction_is_the_least_squares_shift():
    y, gamma, W = _data(2)
    cal = O.calibrate_out_proj(y, gamma, W, coef=1.0)
    Y = O.out_proj_fp64(y, gamma, W)
    Yq = O.out_proj_i8(y, cal, correct=False)["y"]
    loss = lambda c: np.sum((Y - (Yq + c[None, :])) ** 2)
    best = loss(cal["c_star"])
    rs = np.random.default_rng(3)
    for _ in range(20):                                   # any other shift is worse
        assert loss(cal["c_star"] + 1e-3 * rs.standard_normal(cal["c_star"].shape)) > best
    assert loss(np.zeros_like(cal["c_star"])) >= best
    # and the corrected output has zero mean error per channel on the calibration set
    np.testing.assert_allclose((Y - O.out_proj_i8(y, cal)["y"]).mean(axis=0), 0.0, atol=1e-12)


def test_coefficient_scales_the_correction():
    y, gamma, W = _data(4)
    full = O.calibrate_out_proj(y, gamma, W, coef=1.0)
    part = O.calibrate_out_proj(y, gamma, W)
    np.testing.assert_allclose(part["c"], 0.15 * full["c_star"], rtol=1e-15)
    d = O.out_proj_i8(y, part)["y"] - O.out_proj_i8(y, part, correct=False)["y"]
    np.testing.assert_allclose(d, np.broadcast_to(part["c"], d.shape), rtol=0, atol=1e-15)


def test_exact_integers_on_representable_inputs():
    # rows of ±a with equal magnitudes: RMSNorm gives exactly ±1, s_a = 1/127; weights are codes × 2^-7
    rs = np.random.default_rng(5)
    K, D = 64, 16
    y = rs.choice([-2.0, 2.0], size=(32, K))
    Wc = rs.integers(-127, 128, (D, K)).astype(np.float64)
    Wc[:, 0] = 127.0                                      # every output channel reaches the amax
    W = Wc / 128.0
    gamma = np.ones(K)
    cal = O.calibrate_out_proj(y, gamma, W)
    np.testing.assert_array_equal(cal["Wq"], Wc.astype(np.int8))
    r = O.out_proj_i8(y, cal, correct=False)
    np.testing.assert_array_equal(r["Aq"], (np.sign(y) * 127).astype(np.int8))
    np.testing.assert_array_equal(r["acc"], (np.sign(y) * 127).astype(np.int64) @ Wc.astype(np.int64).T)
    np.testing.assert_allclose(r["y"], O.out_proj_fp64(y, gamma, W), rtol=0, atol=1e-12)   # exact
    np.testing.assert_allclose(cal["c_star"], 0.0, atol=1e-12)


def test_correction_removes_a_systematic_error_out_of_sample():
    # features that are the same on every token (after RMSNorm) are rounded the same way on every
    # token: a systematic error that the calibration mean estimates and removes on unseen tokens
    rs = np.random.default_rng(6)
    T, K, D = 2048, 128, 32
    y = 0.05 * rs.standard_normal((T, K))
    y[:, :8] = rs.uniform(0.5, 3.0, 8)[None, :]          # constant features carry most of the norm
    gamma = np.ones(K)
    W = rs.standard_normal((D, K)) / np.sqrt(K)
    cal = O.calibrate_out_proj(y[:1024], gamma, W, coef=1.0)
    Y = O.out_proj_fp64(y[1024:], gamma, W)
    e0 = np.linalg.norm(Y - O.out_proj_i8(y[1024:], cal, correct=False)["y"])
    e1 = np.linalg.norm(Y - O.out_proj_i8(y[1024:], cal)["y"])
    assert e1 < 0.9 * e0
