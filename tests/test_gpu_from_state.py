"""GPU parity of the scan continued from a given state (ssd_scan_fwd_*_from_state).

bf16: y and the final state within 5e-3 (relative L2) of the fp64 recurrence started
from the same state.  W8A8: the final INT8 state bit-exact with the integer oracle
started from the same codes, y within 1e-2 of that oracle and 5e-2 of fp64.  Both
paths: a sequence split at a chunk boundary, the second call continuing from the
first call's final state, reproduces one call over the whole sequence bit for bit.
"""
import numpy as np
import pytest

from harness import Workload, make_inputs, as_float
from oracle import ssd_fp64 as F
from oracle import ssd_w8a8 as W
from oracle.ssd_fp64 import rel_l2
from tests.gpu_common import TOL_BF16, TOL_I8_Y, bf16_to_np, host, oracle_scales

pytestmark = pytest.mark.gpu

CASES = {
    "ragged-q256": Workload("ragged-q256", 2, 1000, 6, 64, 128, 2, 256, head_scale=True, outliers=True),
    "ragged-q128": Workload("ragged-q128", 1, 700, 4, 64, 128, 1, 128, seed=1),
    "tiny-ragged": Workload("tiny-ragged", 3, 77, 8, 16, 16, 2, 64, seed=3),
}
F32 = np.float32


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import int8_quant_b200 as iq
    iq.library()
    return torch


def _problem(inp, chunk):
    from int8_quant_b200.runner import SsdProblem, to_device
    return SsdProblem(to_device(inp), chunk)


def _slice(inp, a, b):
    return {k: (np.ascontiguousarray(v[:, a:b]) if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}


@pytest.mark.parametrize("name", list(CASES))
def test_bf16_from_state_matches_fp64(torch_cuda, name):
    w = CASES[name]
    inp = make_inputs(w)
    pb = _problem(inp, w.chunk)
    h0 = (0.5 * np.random.default_rng(7).standard_normal(tuple(pb.final32.shape))).astype(F32)
    pb.run_bf16(initial_state=torch_cuda.from_numpy(h0).cuda())
    torch_cuda.cuda.synchronize()
    ey, ef = F.ssd_sequential(as_float(inp["x"]), inp["dt"], inp["A"], as_float(inp["B"]), as_float(inp["C"]),
                              inp["D"], state0=h0.astype(np.float64))
    y, fin = bf16_to_np(pb.y), host(pb.final32).astype(np.float64)
    assert rel_l2(y, ey) <= TOL_BF16, rel_l2(y, ey)
    assert rel_l2(fin, ef) <= TOL_BF16, rel_l2(fin, ef)
    y0, _ = F.ssd_sequential(as_float(inp["x"]), inp["dt"], inp["A"], as_float(inp["B"]), as_float(inp["C"]),
                             inp["D"])
    assert rel_l2(y[:, :64], y0[:, :64]) > 10 * TOL_BF16     # the state made a visible difference


@pytest.mark.parametrize("name", list(CASES))
def test_i8_from_state_bit_exact(torch_cuda, name):
    w = CASES[name]
    inp = make_inputs(w)
    pb = _problem(inp, w.chunk)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
    init8 = np.random.default_rng(8).integers(-60, 61, tuple(pb.final8.shape)).astype(np.int8)
    pb.run_i8(initial_state=torch_cuda.from_numpy(init8).cuda())
    torch_cuda.cuda.synchronize()
    Bv, Cv = as_float(inp["B"]).astype(F32), as_float(inp["C"]).astype(F32)
    Bq, Cq = W.quantize_inputs(Bv, Cv, sc["s_B"], sc["s_C"])
    r = W.ssd_w8a8(as_float(inp["x"]).astype(F32), inp["dt"], inp["A"], Bq, Cq, inp["D"], sc["s_B"], sc["s_C"],
                   sc["s_x"], sc["s_s"], w.chunk, 7, init8=init8)
    np.testing.assert_array_equal(host(pb.final8), r["final8"])
    y = bf16_to_np(pb.y)
    assert rel_l2(y, r["y"]) <= 1e-2, rel_l2(y, r["y"])
    H, P = w.nheads, w.headdim
    h0 = init8.astype(np.float64) * np.asarray(sc["s_s"], np.float64).reshape(H, P)[None, :, :, None]
    ey, _ = F.ssd_sequential(as_float(inp["x"]), inp["dt"], inp["A"], as_float(inp["B"]), as_float(inp["C"]),
                             inp["D"], state0=h0)
    assert rel_l2(y, ey) <= TOL_I8_Y, rel_l2(y, ey)


@pytest.mark.parametrize("path", ["bf16", "w8a8"])
def test_split_at_a_chunk_boundary_is_bit_exact(torch_cuda, path):
    torch = torch_cuda
    w = Workload("split", 2, 1024, 6, 64, 128, 2, 256, seed=4, head_scale=True, outliers=True)
    inp = make_inputs(w)
    cut = 512
    parts = [_problem(inp, w.chunk), _problem(_slice(inp, 0, cut), w.chunk), _problem(_slice(inp, cut, w.seqlen),
                                                                                      w.chunk)]
    if path == "w8a8":
        sc = oracle_scales(inp, w.chunk, w.calib_prefix)
        for pb in parts:
            pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
        whole, first, second = parts
        whole.run_i8()
        first.run_i8()
        second.run_i8(initial_state=first.final8)
        fin_w, fin_s = whole.final8, second.final8
    else:
        whole, first, second = parts
        whole.run_bf16()
        first.run_bf16()
        second.run_bf16(initial_state=first.final32)
        fin_w, fin_s = whole.final32, second.final32
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([first.y, second.y], dim=1), whole.y)
    assert torch.equal(fin_s, fin_w)


def test_zero_length_returns_the_initial_state(torch_cuda):
    torch = torch_cuda
    w = Workload("L0", 2, 0, 4, 64, 128, 1, 256)
    pb = _problem(make_inputs(w), w.chunk)
    h0 = torch.randn(tuple(pb.final32.shape), device="cuda")
    pb.run_bf16(initial_state=h0)
    pb.set_scales(np.ones(1), np.ones(1), np.ones(4 * 64), np.ones(4 * 64))
    s0 = torch.randint(-127, 128, tuple(pb.final8.shape), device="cuda", dtype=torch.int8)
    pb.run_i8(initial_state=s0)
    torch.cuda.synchronize()
    assert torch.equal(pb.final32, h0) and torch.equal(pb.final8, s0)
