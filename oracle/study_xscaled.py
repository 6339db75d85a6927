"""Quantisation error of the ChunkState reconstruction — TEST INFRASTRUCTURE ONLY.

"SSDi8: Accurate and Efficient 8-bit Quantization for State Space Duality" (key
design 1) moves the state decay from B onto X, X_scaled = LUT_state ⊙ X with
LUT_state[j] = dt_j·exp(Acs_{Q-1} - Acs_j), and quantises X_scaled once per (h,p);
its appendix A (the proof is not on the page) states that under mild conditions
this has a smaller quantisation error than quantising X and applying the LUT
afterwards.  This module measures both, in float64, on given inputs:

  "xscaled"    X̂ = Q(X_s; s_xs)·s_xs                 s_xs[h,p] = amax |X_s[.,h,p]| / 127
  "x_then_lut" X̂ = (Q(X; s_x)·s_x) ⊙ LUT_state        s_x[h,p]  = amax |x[.,h,p]| / 127

with Q(v; s) = clamp(rint(v / s), ±127) (amax over the whole input, so nothing
saturates), and reports ‖X̂ - X_s‖ / ‖X_s‖ over all elements and the same
relative error of the chunk states S_c = X̂ᵀB against the exact S_c.  It uses
`ssd_fp64.ssd_chunked` for X_s, LUT_state and S_c.
"""
from __future__ import annotations

import numpy as np

from . import ssd_fp64 as F

QMAX = 127


def _q(v: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Symmetric quantise-dequantise with step s (broadcast), float64."""
    return np.clip(np.rint(v / s), -QMAX, QMAX) * s


def _scale(amax: np.ndarray) -> np.ndarray:
    return np.where(amax > 0, amax / QMAX, 1.0)


def study(x, dt, A, B, chunk: int) -> dict:
    """x [Bt,L,H,P], dt [Bt,L,H], A [H], B [Bt,L,G,N] (values as float); L a multiple of chunk.

    Returns {"xs_err": {scheme: rel. L2}, "state_err": {scheme: rel. L2}, "lut_spread": median over
    (b,c,h) of max/min LUT_state within a chunk, "xs_outlier_ratio": amax |X_s| / its 99.9th percentile}."""
    x = np.asarray(x, np.float64)
    dt = np.asarray(dt, np.float64)
    Bt, L, H, P = x.shape
    Q = int(chunk)
    assert L % Q == 0, "whole chunks only"
    nc = L // Q
    _, _, parts = F.ssd_chunked(x, dt, A, B, B, np.zeros(H), Q, states_only=True)
    Acs = parts["Acs"]                                                  # [Bt,nc,Q,H]
    lut = dt.reshape(Bt, nc, Q, H) * np.exp(Acs[:, :, Q - 1:Q, :] - Acs)   # LUT_state
    Xs = parts["Xs"]                                                    # [Bt,nc,Q,H,P] = lut ⊙ x
    xc = x.reshape(Bt, nc, Q, H, P)
    s_xs = _scale(np.abs(Xs).max(axis=(0, 1, 2)))                       # [H,P]
    s_x = _scale(np.abs(xc).max(axis=(0, 1, 2)))
    est = {"xscaled": _q(Xs, s_xs), "x_then_lut": _q(xc, s_x) * lut[..., None]}
    Bh = np.asarray(B, np.float64)[:, :, np.arange(H) // (H // B.shape[2]), :].reshape(Bt, nc, Q, H, -1)
    S = parts["S"]                                                      # [Bt,nc,H,P,N]
    rel = lambda a, b: float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
    xs_err = {k: rel(v, Xs) for k, v in est.items()}
    st_err = {k: rel(np.einsum("bcjhp,bcjhn->bchpn", v, Bh, optimize=True), S) for k, v in est.items()}
    spread = lut.max(axis=2) / np.maximum(lut.min(axis=2), 1e-300)
    a = np.abs(Xs).reshape(-1)
    return {"xs_err": xs_err, "state_err": st_err, "lut_spread": float(np.median(spread)),
            "xs_outlier_ratio": float(a.max() / max(np.quantile(a, 0.999), 1e-300))}
