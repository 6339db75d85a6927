"""SSD epilogue: RMSNorm + INT8 output projection with mean correction — TEST
INFRASTRUCTURE ONLY.

Follows "SSDi8: Accurate and Efficient 8-bit Quantization for State Space Duality"
(ICLR 2026 paper notes): key design 4 (the quantisation error of Y = XW is
compensated by the per-channel mean c*_p = (1/N) Σ_i (Y - Y')_{i,p}, the closed-form
minimiser of ‖Y - (Y' + c)‖_F², applied to the output projection only), the
training strategy (symmetric static W8A8; γ migration for the RMSNorm outliers;
mean-correction coefficient 0.15).  Readings where the notes are silent:
* RMSNorm over the d_inner = H·P features of a token, eps = 1e-5, no gating (the
  scan has none): u = y / sqrt(mean(y²) + eps);
* γ migration: the RMSNorm weight γ is folded into the projection, W' = W·diag(γ),
  so the quantised activation is u itself;
* activation scale: one static symmetric step s_a = amax|u| / 127 over the
  calibration tokens; weights: one step per output channel, s_w[d] = amax_k |W'[d,k]| / 127;
  q = clamp(rint(v / s), ±127) (as the scan's quantiser);
* Y'[t,d] = s_a·s_w[d]·Σ_k Aq[t,k]·Wq[d,k]  (exact int64 accumulation), and the
  corrected output Y'' = Y' + 0.15·c*, c* the per-channel mean of Y - Y' over the
  calibration tokens, Y = u·W'ᵀ in float64.

Functions: `rmsnorm`, `calibrate_out_proj` (scales, codes and c*), `out_proj_i8`
(the quantised epilogue), `out_proj_fp64` (the definition).  Pins in
tests/test_oracle_out_proj.py: c* is the least-squares optimum (no other constant
shift lowers ‖Y - (Y' + c)‖ on the calibration set), exact integer results on
representable inputs, RMSNorm's closed forms, γ migration as an identity.
"""
from __future__ import annotations

import numpy as np

QMAX = 127
EPS = 1e-5
MEAN_CORRECTION_COEF = 0.15


def rmsnorm(y: np.ndarray, eps: float = EPS) -> np.ndarray:
    """y [T, K] → y / sqrt(mean_k y² + eps), float64."""
    y = np.asarray(y, np.float64)
    return y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)


def _q(v: np.ndarray, s) -> np.ndarray:
    return np.clip(np.rint(np.asarray(v, np.float64) / s), -QMAX, QMAX).astype(np.int64)


def _step(amax):
    amax = np.asarray(amax, np.float64)
    return np.where(amax > 0, amax / QMAX, 1.0)


def out_proj_fp64(y, gamma, W) -> np.ndarray:
    """The definition: RMSNorm(y)·γ projected by W [D, K]: [T, D], float64."""
    return (rmsnorm(y) * np.asarray(gamma, np.float64)) @ np.asarray(W, np.float64).T


def calibrate_out_proj(y_cal, gamma, W, coef: float = MEAN_CORRECTION_COEF) -> dict:
    """Static scales, weight codes and the mean correction from calibration tokens y_cal [N, K]."""
    Wg = np.asarray(W, np.float64) * np.asarray(gamma, np.float64)[None, :]       # γ migration
    s_w = _step(np.abs(Wg).max(axis=1))                                            # [D]
    Wq = _q(Wg, s_w[:, None])
    u = rmsnorm(y_cal)
    s_a = float(_step(np.abs(u).max()))
    Yq = (_q(u, s_a) @ Wq.T) * s_a * s_w[None, :]
    c_star = (u @ Wg.T - Yq).mean(axis=0)                                          # per-channel mean error
    return {"s_a": s_a, "s_w": s_w, "Wq": Wq.astype(np.int8), "c_star": c_star, "c": coef * c_star}


def out_proj_i8(y, cal: dict, correct: bool = True) -> dict:
    """The quantised epilogue on tokens y [T, K]: RMSNorm, static INT8 activation codes, INT32
    (exact) products with the weight codes, dequantisation, + c (if `correct`)."""
    u = rmsnorm(y)
    Aq = _q(u, cal["s_a"])
    acc = Aq @ cal["Wq"].astype(np.int64).T
    assert np.abs(acc).max(initial=0) < 2 ** 31, "int32 accumulator overflow"
    out = acc * cal["s_a"] * cal["s_w"][None, :]
    if correct:
        out = out + cal["c"][None, :]
    return {"y": out, "Aq": Aq.astype(np.int8), "acc": acc.astype(np.int32)}
