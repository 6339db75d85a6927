"""Pins of the fp64 oracle against closed forms, brute force and invariants (CPU only)."""
import json
import math
import os

import numpy as np
import pytest

from harness import Workload, make_inputs, as_float
from oracle import ssd_fp64 as F
from oracle.ssd_fp64 import rel_l2

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _inputs(seed, Bt, L, H, P, N, G, Q=64, **kw):
    w = Workload("t", Bt, L, H, P, N, G, Q, seed=seed, **kw)
    d = make_inputs(w)
    return (as_float(d["x"]), d["dt"].astype(np.float64), d["A"].astype(np.float64),
            as_float(d["B"]), as_float(d["C"]), d["D"].astype(np.float64))


def _hand_L3():
    with open(os.path.join(GOLDEN, "hand_L3.json")) as f:
        g = json.load(f)
    x = np.array(g["x"]).reshape(1, 3, 1, 1)
    dt = np.array(g["dt"]).reshape(1, 3, 1)
    A = np.array([g["A"]])
    B = np.array(g["B"]).reshape(1, 3, 1, 2)
    C = np.array(g["C"]).reshape(1, 3, 1, 2)
    D = np.array([g["D"]])
    return x, dt, A, B, C, D


def _hand_L3_expected():
    # Written out by hand from the recurrence (see tests/golden/hand_L3.json):
    # h0 = [0.5, 0];  h1 = [0.5 e1, -0.5];  h2 = [0.5 e1 e2 + 3, -0.5 e2 + 3]
    e1, e2 = math.exp(-0.25), math.exp(-1.0)
    y = np.array([1.0, 1.5 * e1 - 0.5, e1 * e2 - 2.5 * e2 + 22.5]).reshape(1, 3, 1, 1)
    final = np.array([0.5 * e1 * e2 + 3.0, -0.5 * e2 + 3.0]).reshape(1, 1, 1, 2)
    return y, final


@pytest.mark.parametrize("fn", ["sequential", "quadratic", "chunked1", "chunked2", "chunked3"])
def test_golden_hand_L3(fn):
    x, dt, A, B, C, D = _hand_L3()
    if fn == "sequential":
        y, fin = F.ssd_sequential(x, dt, A, B, C, D)
    elif fn == "quadratic":
        y, fin = F.ssd_quadratic(x, dt, A, B, C, D)
    else:
        y, fin = F.ssd_chunked(x, dt, A, B, C, D, chunk=int(fn[-1]))
    ey, ef = _hand_L3_expected()
    np.testing.assert_allclose(y, ey, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(fin, ef, rtol=1e-13, atol=1e-13)


def test_golden_detects_planted_mistakes():
    """Each plausible slip in the recurrence changes the hand example's answer."""
    x, dt, A, B, C, D = _hand_L3()
    ey, ef = _hand_L3_expected()
    wrong = {
        "B and C swapped": F.ssd_sequential(x, dt, A, C, B, D),
        "D term dropped": F.ssd_sequential(x, dt, A, B, C, 0 * D),
        "dt missing on the input": F.ssd_sequential(x, np.ones_like(dt), A, B, C, D),
        "decay uses the previous dt": F.ssd_sequential(x, np.roll(dt, 1, axis=1), A, B, C, D),
        "A with the wrong sign": F.ssd_sequential(x, dt, -A, B, C, D),
    }
    for name, (y, fin) in wrong.items():
        assert not (np.allclose(y, ey, rtol=1e-9) and np.allclose(fin, ef, rtol=1e-9)), name


@pytest.mark.parametrize("L", [1, 2, 7, 64, 100])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_sequential_equals_bruteforce(L, seed):
    args = _inputs(seed, 2, L, 4, 3, 5, 2)
    ys, fs = F.ssd_sequential(*args)
    yq, fq = F.ssd_quadratic(*args)
    assert rel_l2(ys, yq) < 1e-12
    assert rel_l2(fs, fq) < 1e-12


def test_L1_closed_form():
    x, dt, A, B, C, D = _inputs(3, 2, 1, 4, 3, 5, 2)
    y, fin = F.ssd_sequential(x, dt, A, B, C, D)
    g = np.arange(4) // 2
    for b in range(2):
        for h in range(4):
            cb = float(C[b, 0, g[h]] @ B[b, 0, g[h]])
            np.testing.assert_allclose(y[b, 0, h], dt[b, 0, h] * cb * x[b, 0, h] + D[h] * x[b, 0, h],
                                       rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(fin[b, h], dt[b, 0, h] * np.outer(x[b, 0, h], B[b, 0, g[h]]),
                                       rtol=1e-13, atol=1e-14)


def test_dt_zero_gives_skip_only():
    x, dt, A, B, C, D = _inputs(4, 2, 33, 4, 3, 5, 1)
    for fn in (F.ssd_sequential, F.ssd_quadratic, lambda *a: F.ssd_chunked(*a, chunk=8)):
        y, fin = fn(x, 0 * dt, A, B, C, D)
        np.testing.assert_allclose(y, D[None, None, :, None] * x, rtol=0, atol=1e-15)
        assert np.all(fin == 0)


def test_A_zero_is_dt_weighted_cumsum():
    x, dt, A, B, C, D = _inputs(5, 2, 50, 4, 3, 5, 2)
    A0 = np.zeros_like(A)
    y, fin = F.ssd_sequential(x, dt, A0, B, C, D)
    g = np.arange(4) // 2
    Bh, Ch = B[:, :, g], C[:, :, g]
    inject = (dt[..., None] * x)[..., None] * Bh[:, :, :, None, :]          # [Bt,L,H,P,N]
    h = np.cumsum(inject, axis=1)
    ey = np.einsum("blhpn,blhn->blhp", h, Ch) + D[None, None, :, None] * x
    assert rel_l2(y, ey) < 1e-12
    assert rel_l2(fin, h[:, -1]) < 1e-12
    yc, fc = F.ssd_chunked(x, dt, A0, B, C, D, chunk=16)
    assert rel_l2(yc, ey) < 1e-12 and rel_l2(fc, h[:, -1]) < 1e-12


@pytest.mark.parametrize("L,chunks", [(64, [1, 2, 4, 8, 16, 32, 64]), (100, [3, 7, 16, 64, 128]),
                                      (257, [64, 128, 256])])
def test_chunked_is_chunk_size_invariant(L, chunks):
    args = _inputs(6, 2, L, 4, 3, 5, 2)
    ys, fs = F.ssd_sequential(*args)
    for Q in chunks:
        yc, fc = F.ssd_chunked(*args, chunk=Q)
        assert rel_l2(yc, ys) < 1e-12, Q
        assert rel_l2(fc, fs) < 1e-12, Q


def test_chunk_equal_to_L_is_the_quadratic_form():
    args = _inputs(7, 1, 48, 2, 4, 6, 1)
    yq, fq = F.ssd_quadratic(*args)
    yc, fc = F.ssd_chunked(*args, chunk=48)
    assert rel_l2(yc, yq) < 1e-13 and rel_l2(fc, fq) < 1e-13


def test_group_broadcast_identical_groups_equal_one_group():
    x, dt, A, B, C, D = _inputs(8, 2, 40, 4, 3, 5, 1)
    B2 = np.repeat(B, 2, axis=2)
    C2 = np.repeat(C, 2, axis=2)
    y1, f1 = F.ssd_sequential(x, dt, A, B, C, D)
    y2, f2 = F.ssd_sequential(x, dt, A, B2, C2, D)
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(f1, f2)
    yc, fc = F.ssd_chunked(x, dt, A, B2, C2, D, chunk=16)
    assert rel_l2(yc, y1) < 1e-12


def test_group_assignment_is_contiguous_blocks():
    """Head h reads group h // (H/G): perturbing group 1 changes heads 2,3 only (H=4, G=2)."""
    x, dt, A, B, C, D = _inputs(9, 1, 20, 4, 3, 5, 2)
    y0, _ = F.ssd_sequential(x, dt, A, B, C, D)
    B2 = B.copy()
    B2[:, :, 1] += 0.5
    y1, _ = F.ssd_sequential(x, dt, A, B2, C, D)
    assert np.array_equal(y0[:, :, :2], y1[:, :, :2])
    assert not np.allclose(y0[:, :, 2:], y1[:, :, 2:])


def test_reconstruction_identity():
    """X×(B⊙LUT) = (LUT⊙X)×B along the shared chunk axis (SSDi8 notes, key design 1)."""
    rs = np.random.default_rng(0)
    X = rs.standard_normal((64, 16))
    Bm = rs.standard_normal((64, 32))
    lut = rs.random(64)
    lhs = X.T @ (Bm * lut[:, None])
    rhs = (X * lut[:, None]).T @ Bm
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    Xi = rs.integers(-8, 9, (64, 16))
    Bi = rs.integers(-8, 9, (64, 32))
    li = rs.integers(0, 5, 64)
    assert np.array_equal(Xi.T @ (Bi * li[:, None]), (Xi * li[:, None]).T @ Bi)


def test_chunked_parts_match_definitions():
    """Chunk states and passed states agree with the sequential recurrence at chunk ends."""
    x, dt, A, B, C, D = _inputs(10, 1, 96, 2, 3, 4, 1)
    _, _, parts = F.ssd_chunked(x, dt, A, B, C, D, chunk=32, return_parts=True)
    for c in range(3):
        _, hc = F.ssd_sequential(x[:, :32 * c], dt[:, :32 * c], A, B[:, :32 * c], C[:, :32 * c], D)
        np.testing.assert_allclose(parts["H"][:, c], hc, rtol=1e-12, atol=1e-14)
        # S_c is the state reached from zero over chunk c alone
        sl = slice(32 * c, 32 * (c + 1))
        _, sc = F.ssd_sequential(x[:, sl], dt[:, sl], A, B[:, sl], C[:, sl], D)
        np.testing.assert_allclose(parts["S"][:, c], sc, rtol=1e-12, atol=1e-14)


def test_calibrate_invariants():
    x, dt, A, B, C, D = _inputs(11, 2, 300, 4, 8, 16, 2)
    sc = F.calibrate(x, dt, A, B, C, chunk=64, prefix=128)
    pre = slice(0, 128)
    for g in range(2):
        assert sc["s_B"][g] == np.float32(np.abs(B[:, pre, g]).max() / 127)
        assert sc["s_C"][g] == np.float32(np.abs(C[:, pre, g]).max() / 127)
    # the largest prefix |X_scaled| of every (h,p) maps onto code 127
    _, _, parts = F.ssd_chunked(x[:, pre], dt[:, pre], A, B[:, pre], C[:, pre], D, 64, states_only=True)
    amax = np.abs(parts["Xs"]).max(axis=(0, 1, 2)).reshape(-1)
    np.testing.assert_allclose(amax / sc["s_x"].astype(np.float64), 127.0, rtol=1e-6)
    z = F.calibrate(0 * x, dt, A, 0 * B, 0 * C, chunk=64)
    assert np.all(z["s_B"] == 1) and np.all(z["s_x"] == 1) and np.all(z["s_s"] == 1)


# ---------------------------------------------------------------- initial state
def _state0(seed, Bt, H, P, N):
    return np.random.default_rng(100 + seed).standard_normal((Bt, H, P, N))


@pytest.mark.parametrize("L", [1, 2, 7, 64])
@pytest.mark.parametrize("seed", [0, 1])
def test_initial_state_sequential_equals_bruteforce(L, seed):
    args = _inputs(seed, 2, L, 4, 3, 5, 2)
    h0 = _state0(seed, 2, 4, 3, 5)
    ys, fs = F.ssd_sequential(*args, state0=h0)
    yq, fq = F.ssd_quadratic(*args, state0=h0)
    assert rel_l2(ys, yq) < 1e-12 and rel_l2(fs, fq) < 1e-12
    # the initial state really enters: both forms differ from the zero-state result
    y0, _ = F.ssd_sequential(*args)
    assert rel_l2(ys, y0) > 1e-3


def test_initial_state_is_linear_superposition():
    # the recurrence is linear in the state: y(h0) = y(0) + (decayed h0)·C
    x, dt, A, B, C, D = _inputs(3, 1, 9, 2, 3, 4, 1)
    h0 = _state0(3, 1, 2, 3, 4)
    y, fin = F.ssd_sequential(x, dt, A, B, C, D, state0=h0)
    y0, fin0 = F.ssd_sequential(x, dt, A, B, C, D)
    acs = np.cumsum(dt * A[None, None, :], axis=1)                        # Σ_{k≤t} a_k   [1,L,H]
    Ch = C[:, :, np.arange(2) // 2]
    extra = np.exp(acs)[..., None] * np.einsum("bhpn,blhn->blhp", h0, Ch)
    assert rel_l2(y, y0 + extra) < 1e-12
    assert rel_l2(fin, fin0 + np.exp(acs[:, -1])[..., None, None] * h0) < 1e-12


@pytest.mark.parametrize("Q", [16, 64])
def test_initial_state_chunked_equals_sequential(Q):
    args = _inputs(4, 2, 150, 4, 3, 5, 2)
    h0 = _state0(4, 2, 4, 3, 5)
    ys, fs = F.ssd_sequential(*args, state0=h0)
    yc, fc = F.ssd_chunked(*args, chunk=Q, state0=h0)
    assert rel_l2(yc, ys) < 1e-12 and rel_l2(fc, fs) < 1e-12


def test_split_at_a_chunk_boundary_equals_the_whole():
    x, dt, A, B, C, D = _inputs(8, 2, 192, 4, 3, 5, 2)
    y, fin = F.ssd_chunked(x, dt, A, B, C, D, chunk=64)
    y1, f1 = F.ssd_chunked(x[:, :128], dt[:, :128], A, B[:, :128], C[:, :128], D, chunk=64)
    y2, f2 = F.ssd_chunked(x[:, 128:], dt[:, 128:], A, B[:, 128:], C[:, 128:], D, chunk=64, state0=f1)
    assert rel_l2(np.concatenate([y1, y2], axis=1), y) < 1e-12
    assert rel_l2(f2, fin) < 1e-12


def test_A_zero_with_initial_state_closed_form():
    x, dt, A, B, C, D = _inputs(9, 2, 40, 4, 3, 5, 2)
    A0 = np.zeros_like(A)
    h0 = _state0(9, 2, 4, 3, 5)
    y, fin = F.ssd_sequential(x, dt, A0, B, C, D, state0=h0)
    g = np.arange(4) // 2
    inject = (dt[..., None] * x)[..., None] * B[:, :, g][:, :, :, None, :]
    h = h0[:, None] + np.cumsum(inject, axis=1)                           # h_t = h0 + Σ_{s≤t} dt x Bᵀ
    ey = np.einsum("blhpn,blhn->blhp", h, C[:, :, g]) + D[None, None, :, None] * x
    assert rel_l2(y, ey) < 1e-12 and rel_l2(fin, h[:, -1]) < 1e-12


def test_calibrate_state_scale_counts_the_passed_states():
    """s_s must take the amax over the passed states too: with A = 0 every chunk adds
    S_c = Q * dt * x * B = 1, so H_c = c and the final state is nc = 4 while every S_c is
    1 -> s_s = 4/127 (dropping the passed states would give 1/127, dropping the final one
    3/127); s_x = amax |dt x| / 127 = (1/32)/127 in closed form."""
    Q, nc = 32, 4
    L = Q * nc
    x = np.ones((1, L, 1, 1))
    dt = np.full((1, L, 1), 1.0 / Q)
    A = np.zeros(1)
    B = np.ones((1, L, 1, 1))
    C = np.ones((1, L, 1, 1))
    sc = F.calibrate(x, dt, A, B, C, chunk=Q, prefix=L)
    assert sc["s_s"][0] == np.float32(4.0 / 127)
    assert sc["s_x"][0] == np.float32((1.0 / Q) / 127)
    # a single large chunk state that decays away: the amax is that S_c itself
    x2 = np.zeros((1, L, 1, 1))
    x2[:, Q:2 * Q] = -3.0                                   # chunk 1 only
    A2 = np.array([-64.0])                                  # dt*A = -2 per token: decays to ~0 in a chunk
    sc2 = F.calibrate(x2, dt, A2, B, C, chunk=Q, prefix=L)
    _, _, parts = F.ssd_chunked(x2, dt, A2, B, C, np.zeros(1), Q, states_only=True)
    s1 = abs(parts["S"][0, 1].max()) if abs(parts["S"][0, 1].max()) > abs(parts["S"][0, 1].min()) else abs(parts["S"][0, 1].min())
    assert sc2["s_s"][0] == np.float32(s1 / 127)
    assert np.abs(parts["H"]).max() <= s1 + 1e-12
