"""Pins of the integer W8A8 oracle (CPU only)."""
import numpy as np
import pytest

from harness import Workload, make_inputs, as_float, WORKLOADS
from oracle import ssd_fp64 as F
from oracle import ssd_w8a8 as W
from oracle.ssd_fp64 import rel_l2

F32 = np.float32


def _ulp_err(got32, ref64):
    got = got32.astype(np.float64)
    ulp = np.spacing(np.abs(ref64).astype(np.float32)).astype(np.float64)
    return np.abs(got - ref64) / ulp


def test_exp_f32_error_bound():
    x = np.linspace(-87.0, 0.0, 2_000_001).astype(F32)
    x = np.concatenate([x, -np.logspace(-30, 1.9, 100_000).astype(F32), np.float32([0.0, -0.0, 1e-3, 2.0])])
    err = _ulp_err(W.exp_f32(x), np.exp(x.astype(np.float64)))
    assert err.max() <= 2.0, err.max()
    assert W.exp_f32(F32(0.0)) == F32(1.0)
    assert W.exp_f32(F32(-0.0)) == F32(1.0)
    assert W.exp_f32(F32(-87.5)) == 0.0
    assert np.all(W.exp_f32(np.float32([-1e30, -100.0])) == 0.0)


def test_chunk_cumsum_exact_on_dyadic_inputs():
    rs = np.random.default_rng(1)
    for Q in (64, 128, 256):
        a = -(rs.integers(0, 1 << 10, (5, Q)) / 1024.0).astype(F32)   # all partial sums exact
        np.testing.assert_array_equal(W.chunk_cumsum_f32(a), np.cumsum(a.astype(np.float64), axis=-1))


def test_chunk_cumsum_order_is_the_specified_one():
    """Bit-for-bit check of the 32-lane order on a case where other orders round differently."""
    rs = np.random.default_rng(2)
    a = (-rs.random((3, 64)) * 0.1).astype(F32)
    got = W.chunk_cumsum_f32(a)
    m = 2
    ref = np.empty_like(a)
    for r in range(3):
        loc = [[a[r, l * m]] for l in range(32)]
        for l in range(32):
            loc[l].append(F32(loc[l][0] + a[r, l * m + 1]))
        tot = [loc[l][-1] for l in range(32)]
        v = list(tot)
        for off in (1, 2, 4, 8, 16):
            v = [F32(v[l - off] + v[l]) if l >= off else v[l] for l in range(32)]
        for l in range(32):
            e = F32(0.0) if l == 0 else v[l - 1]
            for i in range(m):
                ref[r, l * m + i] = F32(e + loc[l][i])
    np.testing.assert_array_equal(got, ref)
    seq = np.cumsum(a, axis=-1, dtype=np.float32)
    assert not np.array_equal(got, seq)          # the order matters for the bits
    np.testing.assert_allclose(got, np.cumsum(a.astype(np.float64), axis=-1), rtol=1e-5)


def test_quantizer_rounds_half_even_and_never_emits_minus_128():
    v = np.float32([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 1e9, -1e9, 126.5, -127.49])
    q = W.quantize_sym(v, F32(1.0))
    np.testing.assert_array_equal(q, np.int8([0, 2, 2, 0, -2, -2, 127, -127, 126, -127]))


def test_fixed_point_decay_shift_worked_values():
    """eq. 6 with S = 2^7: Q(H) ← S8 + (dq·H + 64) >> 7, saturated to ±127."""
    cases = [  # (dq, H_prev, S8, expected) — by hand: 99·100/128 = 77.34 → 77, etc.
        (99, 100, 5, 82), (99, -100, 5, -72), (128, 57, -3, 54), (0, 120, 7, 7),
        (64, 1, 0, 1), (64, -1, 0, 0), (128, 127, 100, 127), (128, -127, -100, -127),
    ]
    for dq, hp, s8, exp in cases:
        # two chunks: the first leaves state hp (from zero), the second adds s8
        S8 = np.int8([hp, s8]).reshape(1, 2, 1, 1, 1)
        dqs = np.int32([0, dq]).reshape(1, 1, 2)
        Hs = W.state_passing_i8(S8, dqs, 7)
        assert Hs[0, 1, 0, 0, 0] == hp
        assert Hs[0, 2, 0, 0, 0] == exp, (dq, hp, s8, Hs[0, 2, 0, 0, 0], exp)


def _exact_case(seed, L=192, Q=64, G=2, H=4, P=8, N=16, Bt=2):
    """Inputs on which every W8A8 rounding is exact: A = 0, dt = 1/8, sparse ternary x, B, C."""
    rs = np.random.default_rng(seed)

    def tern(shape, p):
        return (rs.choice([-1.0, 0.0, 1.0], size=shape, p=[p / 2, 1 - p, p / 2])).astype(F32)

    x = tern((Bt, L, H, P), 0.06)
    Bv = tern((Bt, L, G, N), 0.06)
    Cv = tern((Bt, L, G, N), 0.3)
    dt = np.full((Bt, L, H), 0.125, F32)
    A = np.zeros(H, F32)
    D = rs.integers(-2, 3, H).astype(F32)
    s_B = np.ones(G, F32)
    s_C = np.ones(G, F32)
    s_x = np.full(H * P, 0.125, F32)     # X_scaled = x/8 → Xq = x
    s_s = np.full(H * P, 0.125, F32)     # M = s_x·s_B/s_s = 1 → S8 = acc
    return x, dt, A, Bv, Cv, D, s_B, s_C, s_x, s_s, Q


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_w8a8_equals_fp64_exactly_when_representable(seed):
    x, dt, A, Bv, Cv, D, s_B, s_C, s_x, s_s, Q = _exact_case(seed)
    Bq, Cq = W.quantize_inputs(Bv, Cv, s_B, s_C)
    assert np.array_equal(Bq, Bv.astype(np.int8)) and np.array_equal(Cq, Cv.astype(np.int8))
    r = W.ssd_w8a8(x, dt, A, Bq, Cq, D, s_B, s_C, s_x, s_s, Q)
    assert np.all(r["dq"] == 128)
    assert np.abs(r["H8"]).max() < 127 and np.abs(r["final8"]).max() < 127, "case must not saturate"
    ys, fs = F.ssd_sequential(x, dt, A, Bv, Cv, D)
    np.testing.assert_allclose(r["y"], ys, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["final"], fs, rtol=0, atol=1e-12)
    # the INT32 ChunkState accumulator is 8·S_c exactly
    _, _, parts = F.ssd_chunked(x, dt, A, Bv, Cv, D, Q, return_parts=True)
    np.testing.assert_array_equal(r["acc_state"], np.rint(8 * parts["S"]).astype(np.int64))


def test_w8a8_ragged_tail_matches_exact_definition():
    x, dt, A, Bv, Cv, D, s_B, s_C, s_x, s_s, Q = _exact_case(5, L=150)
    Bq, Cq = W.quantize_inputs(Bv, Cv, s_B, s_C)
    r = W.ssd_w8a8(x, dt, A, Bq, Cq, D, s_B, s_C, s_x, s_s, Q)
    ys, fs = F.ssd_sequential(x, dt, A, Bv, Cv, D)
    np.testing.assert_allclose(r["y"], ys, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["final"], fs, rtol=0, atol=1e-12)


def test_w8a8_A_zero_recursion_is_saturating_prefix_sum():
    w = Workload("t", 2, 640, 4, 8, 16, 1, 64, seed=3)
    d = make_inputs(w)
    x, Bv, Cv = as_float(d["x"]).astype(F32), as_float(d["B"]).astype(F32), as_float(d["C"]).astype(F32)
    A = np.zeros(4, F32)
    sc = F.calibrate(x, d["dt"], A, Bv, Cv, 64, prefix=64)   # short prefix: later chunks saturate
    Bq, Cq = W.quantize_inputs(Bv, Cv, sc["s_B"], sc["s_C"])
    r = W.ssd_w8a8(x, d["dt"], A, Bq, Cq, d["D"], sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 64)
    assert np.all(r["dq"] == 128)
    H = np.zeros_like(r["S8"][:, 0], dtype=np.int64)
    for c in range(r["S8"].shape[1]):
        np.testing.assert_array_equal(r["H8"][:, c], H)
        H = np.clip(H + r["S8"][:, c], -127, 127)
    np.testing.assert_array_equal(r["final8"], H)
    assert (np.abs(H) == 127).any(), "the test must exercise saturation"


def test_w8a8_saturation_and_int32_headroom():
    # worst case ChunkState accumulator: Q·127·127 < 2^24, so float32(acc) is exact
    assert 256 * 127 * 127 < 2 ** 24
    assert int(F32(256 * 127 * 127)) == 256 * 127 * 127
    w = Workload("t", 1, 128, 2, 8, 16, 1, 64, seed=4)
    d = make_inputs(w)
    x, Bv, Cv = as_float(d["x"]).astype(F32), as_float(d["B"]).astype(F32), as_float(d["C"]).astype(F32)
    s_x = np.full(16, 1e-6, F32)
    s_s = np.full(16, 1e-12, F32)            # requant multiplier s_x·s_B/s_s = 1: S8 = acc saturates
    r = W.ssd_w8a8(x, d["dt"], d["A"], *W.quantize_inputs(Bv, Cv, np.full(1, 1e-6, F32), np.full(1, 1e-6, F32)),
                   d["D"], np.full(1, 1e-6, F32), np.full(1, 1e-6, F32), s_x, s_s, 64)
    for k in ("Xq", "S8", "H8", "final8"):
        assert r[k].min() >= -127 and r[k].max() <= 127
        assert (np.abs(r[k]) == 127).any(), k


def test_w8a8_requant_matches_definition():
    """S8 = clamp(rint(float32(acc)·M)), M = (s_x·s_B)/s_s in float32 (key design 2)."""
    w = WORKLOADS["tiny"]
    d = make_inputs(w)
    x, Bv, Cv = as_float(d["x"]).astype(F32), as_float(d["B"]).astype(F32), as_float(d["C"]).astype(F32)
    sc = F.calibrate(x, d["dt"], d["A"], Bv, Cv, 64)
    Bq, Cq = W.quantize_inputs(Bv, Cv, sc["s_B"], sc["s_C"])
    r = W.ssd_w8a8(x, d["dt"], d["A"], Bq, Cq, d["D"], sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 64)
    acc = r["acc_state"].astype(np.float64)
    M64 = (sc["s_x"].astype(np.float64) * sc["s_B"][0]) / sc["s_s"].astype(np.float64)
    real = acc * M64.reshape(4, 16)[None, None, :, :, None]
    # the float32 requantisation differs from the exact one by at most one code, on ties only
    assert np.abs(r["S8"] - np.clip(np.rint(real), -127, 127)).max() <= 1
    # and the stored states dequantise to the fp64 chunk states within one step per element
    _, _, parts = F.ssd_chunked(x, d["dt"], d["A"], Bv, Cv, d["D"], 64, return_parts=True)
    deq = r["S8"] * sc["s_s"].reshape(4, 16)[None, None, :, :, None]
    assert rel_l2(deq, parts["S"]) < 0.05


@pytest.mark.parametrize("name", ["tiny"])
def test_w8a8_output_within_tolerance_of_fp64(name):
    w = WORKLOADS[name]
    d = make_inputs(w)
    x, Bv, Cv = as_float(d["x"]), as_float(d["B"]), as_float(d["C"])
    sc = F.calibrate(x, d["dt"], d["A"], Bv, Cv, w.chunk, w.calib_prefix)
    Bq, Cq = W.quantize_inputs(Bv.astype(F32), Cv.astype(F32), sc["s_B"], sc["s_C"])
    r = W.ssd_w8a8(x.astype(F32), d["dt"], d["A"], Bq, Cq, d["D"], sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"],
                   w.chunk)
    ys, _ = F.ssd_sequential(x, d["dt"], d["A"], Bv, Cv, d["D"])
    assert rel_l2(r["y"], ys) <= 5e-2


# ---------------------------------------------------------------- initial state and decode step
def _calibrated(w, prefix=64):
    d = make_inputs(w)
    x, Bv, Cv = as_float(d["x"]).astype(F32), as_float(d["B"]).astype(F32), as_float(d["C"]).astype(F32)
    sc = F.calibrate(x, d["dt"], d["A"], Bv, Cv, w.chunk, prefix=prefix)
    Bq, Cq = W.quantize_inputs(Bv, Cv, sc["s_B"], sc["s_C"])
    return d, x, Bq, Cq, sc


def test_w8a8_split_at_a_chunk_boundary_is_bit_exact():
    w = Workload("t", 2, 320, 4, 8, 16, 2, 64, seed=11, head_scale=True, outliers=True)
    d, x, Bq, Cq, sc = _calibrated(w)
    args = (d["A"], d["D"], sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 64)
    whole = W.ssd_w8a8(x, d["dt"], Bq=Bq, Cq=Cq, **dict(zip(("A", "D", "s_B", "s_C", "s_x", "s_s", "chunk"), args)))
    cut = 192
    kw = dict(zip(("A", "D", "s_B", "s_C", "s_x", "s_s", "chunk"), args))
    r1 = W.ssd_w8a8(x[:, :cut], d["dt"][:, :cut], Bq=Bq[:, :cut], Cq=Cq[:, :cut], **kw)
    r2 = W.ssd_w8a8(x[:, cut:], d["dt"][:, cut:], Bq=Bq[:, cut:], Cq=Cq[:, cut:], init8=r1["final8"], **kw)
    assert (r1["final8"] != 0).any(), "the carried state must be non-trivial"
    np.testing.assert_array_equal(np.concatenate([r1["H8"], r2["H8"]], axis=1), whole["H8"])
    np.testing.assert_array_equal(np.concatenate([r1["S8"], r2["S8"]], axis=1), whole["S8"])
    np.testing.assert_array_equal(np.concatenate([r1["acc_scan1"], r2["acc_scan1"]], axis=1), whole["acc_scan1"])
    np.testing.assert_array_equal(r2["final8"], whole["final8"])
    np.testing.assert_array_equal(np.concatenate([r1["y"], r2["y"]], axis=1), whole["y"])


@pytest.mark.parametrize("seed", [0, 1])
def test_w8a8_with_initial_state_equals_fp64_exactly_when_representable(seed):
    x, dt, A, Bv, Cv, D, s_B, s_C, s_x, s_s, Q = _exact_case(seed)
    Bq, Cq = W.quantize_inputs(Bv, Cv, s_B, s_C)
    Bt, L, H, P = x.shape
    init8 = np.random.default_rng(50 + seed).integers(-20, 21, (Bt, H, P, Bv.shape[-1])).astype(np.int8)
    r = W.ssd_w8a8(x, dt, A, Bq, Cq, D, s_B, s_C, s_x, s_s, Q, init8=init8)
    assert np.abs(r["final8"]).max() < 127, "case must not saturate"
    h0 = init8.astype(np.float64) * s_s.reshape(H, P)[None, :, :, None].astype(np.float64)
    ys, fs = F.ssd_sequential(x, dt, A, Bv, Cv, D, state0=h0)
    np.testing.assert_allclose(r["y"], ys, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["final"], fs, rtol=0, atol=1e-12)


def test_decode_step_equals_a_one_token_scan():
    w = Workload("t", 2, 257, 4, 8, 16, 2, 64, seed=12, head_scale=True, outliers=True)
    d, x, Bq, Cq, sc = _calibrated(w)
    kw = dict(A=d["A"], D=d["D"], s_B=sc["s_B"], s_C=sc["s_C"], s_x=sc["s_x"], s_s=sc["s_s"])
    r0 = W.ssd_w8a8(x[:, :256], d["dt"][:, :256], Bq=Bq[:, :256], Cq=Cq[:, :256], chunk=64, **kw)
    t = 256
    step = W.decode_step_i8(x[:, t], d["dt"][:, t], Bq=Bq[:, t], Cq=Cq[:, t], state8=r0["final8"], **kw)
    one = W.ssd_w8a8(x[:, t:t + 1], d["dt"][:, t:t + 1], Bq=Bq[:, t:t + 1], Cq=Cq[:, t:t + 1], chunk=32,
                     init8=r0["final8"], **kw)
    np.testing.assert_array_equal(step["state8"], one["final8"])
    np.testing.assert_array_equal(step["Xq"], one["Xq"][:, 0])
    np.testing.assert_array_equal(step["S8"], one["S8"][:, 0])
    np.testing.assert_array_equal(step["acc_state"], one["acc_state"][:, 0])
    np.testing.assert_array_equal(step["dq"], one["dq"][:, :, 0])
    np.testing.assert_array_equal(step["acc_scan1"], one["acc_scan1"][:, 0])
    np.testing.assert_array_equal(step["CB"], one["CB"][:, 0, :, 0, 0])
    np.testing.assert_allclose(step["y"], one["y"][:, 0], rtol=1e-13, atol=1e-12)
    # the scan over all 257 tokens (the last one alone in a padded chunk) ends in the same state
    full = W.ssd_w8a8(x, d["dt"], Bq=Bq, Cq=Cq, chunk=64, **kw)
    np.testing.assert_array_equal(full["final8"], step["state8"])
    assert not np.array_equal(step["state8"], r0["final8"])


def test_decode_steps_equal_fp64_exactly_when_representable():
    x, dt, A, Bv, Cv, D, s_B, s_C, s_x, s_s, Q = _exact_case(3, L=24)
    Bq, Cq = W.quantize_inputs(Bv, Cv, s_B, s_C)
    Bt, L, H, P = x.shape
    N = Bv.shape[-1]
    st = np.zeros((Bt, H, P, N), np.int8)
    ys, fs = F.ssd_sequential(x, dt, A, Bv, Cv, D)
    for t in range(L):
        r = W.decode_step_i8(x[:, t], dt[:, t], A, Bq[:, t], Cq[:, t], D, s_B, s_C, s_x, s_s, st)
        np.testing.assert_allclose(r["y"], ys[:, t], rtol=0, atol=1e-12)
        st = r["state8"]
    assert np.abs(st).max() < 127
    np.testing.assert_allclose(st.astype(np.float64) * s_s.reshape(H, P)[None, :, :, None], fs, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- the notes' storage variant (study switches)
def test_fp16_acs_is_exact_when_acs_is_representable_in_half():
    x, dt, A, Bv, Cv, D, s_B, s_C, s_x, s_s, Q = _exact_case(6)
    A = np.full_like(A, -0.5)                                 # a = -1/16: every Acs is k/16, |Acs| <= 12
    Bq, Cq = W.quantize_inputs(Bv, Cv, s_B, s_C)
    r0 = W.ssd_w8a8(x, dt, A, Bq, Cq, D, s_B, s_C, s_x, s_s, Q)
    r1 = W.ssd_w8a8(x, dt, A, Bq, Cq, D, s_B, s_C, s_x, s_s, Q, acs_fp16=True)
    assert np.array_equal(r0["Acs"], r1["Acs"].astype(np.float16).astype(np.float32))
    for k in ("Xq", "S8", "H8", "final8", "dq", "acc_scan1"):
        np.testing.assert_array_equal(r0[k], r1[k])
    np.testing.assert_array_equal(r0["y"], r1["y"])


def test_fp16_acs_changes_codes_when_not_representable():
    w = Workload("t", 1, 512, 4, 8, 16, 1, 256, seed=7)
    d, x, Bq, Cq, sc = _calibrated(w)
    kw = dict(A=d["A"], D=d["D"], s_B=sc["s_B"], s_C=sc["s_C"], s_x=sc["s_x"], s_s=sc["s_s"], chunk=256)
    r0 = W.ssd_w8a8(x, d["dt"], Bq=Bq, Cq=Cq, **kw)
    r1 = W.ssd_w8a8(x, d["dt"], Bq=Bq, Cq=Cq, acs_fp16=True, **kw)
    assert not np.array_equal(r0["Acs"], r1["Acs"])
    assert rel_l2(r1["y"], r0["y"]) < 1e-2


def test_int8_cb_is_a_per_tile_symmetric_requantisation():
    w = Workload("t", 2, 512, 4, 8, 16, 2, 256, seed=8)
    d, x, Bq, Cq, sc = _calibrated(w)
    kw = dict(A=d["A"], D=d["D"], s_B=sc["s_B"], s_C=sc["s_C"], s_x=sc["s_x"], s_s=sc["s_s"], chunk=256)
    r = W.ssd_w8a8(x, d["dt"], Bq=Bq, Cq=Cq, cb_int8=True, **kw)
    CB, CB8, s = r["CB"].astype(np.float64), r["CB8"].astype(np.float64), r["s_cb"]
    assert np.all(np.abs(CB8 * s - CB) <= s / 2 + 1e-9)            # rounding to the nearest step
    assert np.all(np.abs(CB8).max(axis=(-2, -1)) == 127)            # every tile's amax maps to 127
    r0 = W.ssd_w8a8(x, d["dt"], Bq=Bq, Cq=Cq, **kw)
    for k in ("Xq", "S8", "H8", "final8", "acc_scan1"):              # only ChunkScan2 reads CB
        np.testing.assert_array_equal(r0[k], r[k])
    assert rel_l2(r["y"], r0["y"]) < 1e-2
