"""fp64 oracle of the SSD scan: the definition, a brute force, and the chunked form.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Shapes follow the library: x [Bt,L,H,P], dt [Bt,L,H], A [H], B and C [Bt,L,G,N],
D [H]; head h reads group g(h) = h // (H/G) (SSDi8 notes, "background": B and C
are stored along G and broadcast to the heads).  All arithmetic is float64.

Functions and what pins them (tests/test_oracle_fp64.py):
* ssd_sequential — the recurrence itself, from a given initial state (zero by
  default).  Pinned by the brute force, the closed forms at L=1 and A=0, dt=0,
  and the hand-derived golden fixture.
* ssd_quadratic  — y = (L∘CBᵀ)(dt⊙x) + Dx with every segment sum formed afresh,
  plus the decayed initial state.  Pinned against the sequential form and the
  golden fixture.
* ssd_chunked    — ChunkCumsum, ChunkState (eq. 4 after the reconstruction),
  StatePassing (eq. 6 read as H_{c+1} = d_c·H_c + S_c, H_0 the initial state),
  ChunkBMM, ChunkScan1/2.  Pinned by chunk-size invariance against the
  sequential form and by splitting a sequence at a chunk boundary.
* calibrate      — static symmetric scales over a prefix.  Pinned by invariants
  (amax maps to 127, zero tensors give scale 1).
"""
from __future__ import annotations

import numpy as np

QMAX = 127


def _heads_view(M: np.ndarray, H: int) -> np.ndarray:
    """Broadcast a [Bt,L,G,N] tensor to its heads: [Bt,L,H,N]."""
    G = M.shape[2]
    return M[:, :, np.arange(H) // (H // G), :]


def ssd_sequential(x, dt, A, B, C, D, state0=None):
    """Sequential recurrence, token by token.

    h_t = exp(dt_t·A_h)·h_{t-1} + dt_t·x_t ⊗ B_{g(h),t}   (h_t is [P,N])
    y_t = h_t·C_{g(h),t} + D_h·x_t
    Returns (y [Bt,L,H,P], final state h_L [Bt,H,P,N]).
    """
    x = np.asarray(x, np.float64)
    dt = np.asarray(dt, np.float64)
    A = np.asarray(A, np.float64)
    D = np.asarray(D, np.float64)
    Bt, L, H, P = x.shape
    Bh = _heads_view(np.asarray(B, np.float64), H)
    Ch = _heads_view(np.asarray(C, np.float64), H)
    N = Bh.shape[-1]
    h = np.zeros((Bt, H, P, N)) if state0 is None else np.array(state0, np.float64)
    y = np.empty((Bt, L, H, P))
    for t in range(L):
        decay = np.exp(dt[:, t, :] * A[None, :])                       # [Bt,H]
        inject = (dt[:, t, :, None] * x[:, t, :, :])[..., None] * Bh[:, t, :, None, :]
        h = decay[:, :, None, None] * h + inject
        y[:, t] = np.einsum("bhpn,bhn->bhp", h, Ch[:, t]) + D[None, :, None] * x[:, t]
    return y, h


def ssd_quadratic(x, dt, A, B, C, D, state0=None):
    """Brute-force "attention form" for small inputs.

    y[t] = Σ_{s≤t} (C_t·B_s)·exp(Σ_{k=s+1..t} dt_k·A)·dt_s·x_s + D·x_t
           + exp(Σ_{k=0..t} dt_k·A)·h0·C_t,
    final = Σ_s exp(Σ_{k=s+1..L-1} dt_k·A)·dt_s·x_s ⊗ B_s + exp(Σ_{k=0..L-1} dt_k·A)·h0,
    h0 the initial state (zero by default).  Every segment sum is accumulated from
    scratch (no cumulative-sum differences).
    """
    x = np.asarray(x, np.float64)
    dt = np.asarray(dt, np.float64)
    A = np.asarray(A, np.float64)
    D = np.asarray(D, np.float64)
    Bt, L, H, P = x.shape
    Bh = _heads_view(np.asarray(B, np.float64), H)
    Ch = _heads_view(np.asarray(C, np.float64), H)
    N = Bh.shape[-1]
    y = np.empty((Bt, L, H, P))
    final = np.zeros((Bt, H, P, N))
    h0 = None if state0 is None else np.asarray(state0, np.float64)
    for b in range(Bt):
        for h in range(H):
            a = dt[b, :, h] * A[h]
            seg = np.full((L, L), -np.inf)                 # seg[t,s] = Σ_{k=s+1..t} a_k
            for s in range(L):
                seg[s, s] = 0.0
                acc = 0.0
                for t in range(s + 1, L):
                    acc += a[t]
                    seg[t, s] = acc
            Lmat = np.exp(seg)                             # 0 above the diagonal
            CB = Ch[b, :, h, :] @ Bh[b, :, h, :].T         # CB[t,s] = C_t·B_s
            u = dt[b, :, h, None] * x[b, :, h, :]
            y[b, :, h, :] = (Lmat * CB) @ u + D[h] * x[b, :, h, :]
            w = Lmat[L - 1, :] if L else np.zeros(0)       # decay from s to the end
            final[b, h] = (w[:, None] * u).T @ Bh[b, :, h, :]
            if h0 is not None:
                for t in range(L):
                    acc = 0.0
                    for k in range(t + 1):
                        acc += a[k]
                    y[b, t, h, :] += np.exp(acc) * (h0[b, h] @ Ch[b, t, h, :])
                acc = 0.0
                for k in range(L):
                    acc += a[k]
                final[b, h] += np.exp(acc) * h0[b, h]
    return y, final


def ssd_chunked(x, dt, A, B, C, D, chunk: int, return_parts: bool = False, states_only: bool = False,
                state0=None):
    """The five SSD sub-modules in fp64, chunk length Q = `chunk`.

    A final partial chunk is padded with tokens of dt = 0 and x = B = C = 0,
    which leave the state and the cumulative sums unchanged.
      ChunkCumsum : Acs[j] = Σ_{i≤j} dt_i·A          (inclusive, per chunk)
      ChunkState  : S_c = Σ_j (dt_j·exp(Acs_{Q-1}-Acs_j)·x_j) ⊗ B_j   (eq. 4 with X_scaled)
      StatePassing: H_0 = state0 (or 0), H_{c+1} = exp(Acs_{Q-1})·H_c + S_c   (eq. 6)
      ChunkBMM    : CB[j,i] = C_j·B_i
      ChunkScan2  : y_d[j] = Σ_{i≤j} CB[j,i]·exp(Acs_j-Acs_i)·dt_i·x_i
      ChunkScan1  : y_o[j] = exp(Acs_j)·H_c·C_j
      y = y_d + y_o + D·x
    """
    x = np.asarray(x, np.float64)
    dt = np.asarray(dt, np.float64)
    A = np.asarray(A, np.float64)
    D = np.asarray(D, np.float64)
    Bt, L, H, P = x.shape
    Bh = _heads_view(np.asarray(B, np.float64), H)
    Ch = _heads_view(np.asarray(C, np.float64), H)
    N = Bh.shape[-1]
    Q = int(chunk)
    nc = (L + Q - 1) // Q
    Lp = nc * Q

    def pad(a):
        w = [(0, 0)] * a.ndim
        w[1] = (0, Lp - L)
        return np.pad(a, w)

    xc = pad(x).reshape(Bt, nc, Q, H, P)
    dtc = pad(dt).reshape(Bt, nc, Q, H)
    Bc = pad(Bh).reshape(Bt, nc, Q, H, N)
    Cc = pad(Ch).reshape(Bt, nc, Q, H, N)

    # ChunkCumsum
    Acs = np.cumsum(dtc * A[None, None, None, :], axis=2)            # [Bt,nc,Q,H]
    last = Acs[:, :, Q - 1:Q, :]                                       # [Bt,nc,1,H]
    # ChunkState: decay moved from B onto x (the reconstruction), then X_scaledᵀ·B
    lut_state = dtc * np.exp(last - Acs)                               # [Bt,nc,Q,H]
    Xs = lut_state[..., None] * xc                                     # [Bt,nc,Q,H,P]
    S = np.einsum("bcjhp,bcjhn->bchpn", Xs, Bc, optimize=True)          # [Bt,nc,H,P,N]
    # StatePassing
    d = np.exp(last[:, :, 0, :])                                       # [Bt,nc,H]
    Hs = np.zeros((Bt, nc + 1, H, P, N))
    if state0 is not None:
        Hs[:, 0] = np.asarray(state0, np.float64)
    for c in range(nc):
        Hs[:, c + 1] = d[:, c, :, None, None] * Hs[:, c] + S[:, c]
    if states_only:
        return None, Hs[:, nc], {"Acs": Acs, "S": S, "H": Hs[:, :nc], "d": d, "Xs": Xs}
    # ChunkBMM and the masked intra-chunk product (ChunkScan2)
    CB = np.einsum("bcjhn,bcihn->bchji", Cc, Bc, optimize=True)         # [Bt,nc,H,Q,Q]
    Acs_h = np.moveaxis(Acs, 3, 2)                                     # [Bt,nc,H,Q]
    diff = Acs_h[..., :, None] - Acs_h[..., None, :]                   # Acs_j - Acs_i
    causal = np.tril(np.ones((Q, Q), dtype=bool))
    decay_ji = np.where(causal, np.exp(np.where(causal, diff, 0.0)), 0.0)
    dt_h = np.moveaxis(dtc, 3, 2)                                      # [Bt,nc,H,Q]
    Mmat = CB * decay_ji * dt_h[..., None, :]
    y_d = np.einsum("bchji,bcihp->bcjhp", Mmat, xc, optimize=True)
    # ChunkScan1: contribution of the state entering the chunk
    y_o = np.einsum("bcjhn,bchpn->bcjhp", Cc, Hs[:, :nc], optimize=True) * np.exp(Acs)[..., None]
    y = y_d + y_o + D[None, None, None, :, None] * xc
    y = y.reshape(Bt, Lp, H, P)[:, :L]
    final = Hs[:, nc]
    if not return_parts:
        return y, final
    return y, final, {"Acs": Acs, "S": S, "H": Hs[:, :nc], "d": d, "Xs": Xs, "CB": CB}


def calibrate(x, dt, A, B, C, chunk: int, prefix: int = 512):
    """Static symmetric INT8 scales from the first min(prefix, L) tokens of each row.

    Step-size convention (real value = code·scale, codes in [-127, 127]):
      s_B[g], s_C[g] = amax over the prefix of |B|, |C| in group g / 127
      s_x[h,p]       = amax of |X_scaled| (fp64) over the prefix chunks / 127
      s_s[h,p]       = amax over n of |S_c| and of the passed states H_1..H_nc (fp64)
                       over the prefix chunks / 127
    An all-zero slice gets scale 1.  Each scale is rounded once to float32.
    Per-G scales for B and C, per-(H,P) scales for X_scaled and the state with the
    state axis N left unquantised (SSDi8 notes, key designs 2 and 3).
    """
    x = np.asarray(x, np.float64)
    T = min(int(prefix), x.shape[1])
    xs, dts = x[:, :T], np.asarray(dt, np.float64)[:, :T]
    Bs, Cs = np.asarray(B, np.float64)[:, :T], np.asarray(C, np.float64)[:, :T]
    Bt, _, H, P = xs.shape

    def scale(amax):
        amax = np.asarray(amax, np.float64)
        return np.where(amax > 0, amax / QMAX, 1.0).astype(np.float32)

    s_B = scale(np.abs(Bs).max(axis=(0, 1, 3)) if T else np.zeros(Bs.shape[2]))
    s_C = scale(np.abs(Cs).max(axis=(0, 1, 3)) if T else np.zeros(Cs.shape[2]))
    if T == 0:
        one = np.ones(H * P, np.float32)
        return {"s_B": s_B, "s_C": s_C, "s_x": one, "s_s": one.copy()}
    _, final, parts = ssd_chunked(xs, dts, A, Bs, Cs, np.zeros(H), chunk, states_only=True)
    Xs = parts["Xs"]                                                   # [Bt,nc,Q,H,P]
    s_x = scale(np.abs(Xs).max(axis=(0, 1, 2)).reshape(-1))
    st = np.maximum(np.abs(parts["S"]).max(axis=(0, 1, 4)), np.abs(parts["H"]).max(axis=(0, 1, 4)))
    st = np.maximum(st, np.abs(final).max(axis=(0, 3)))
    s_s = scale(st.reshape(-1))
    return {"s_B": s_B, "s_C": s_C, "s_x": s_x, "s_s": s_s}


def rel_l2(got, ref) -> float:
    """‖got − ref‖₂ / ‖ref‖₂ over the whole tensor (0 when both are zero)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((got - ref).ravel())
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)
