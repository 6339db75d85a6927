"""GPU parity of the one-token decode step (ssd_decode_step_bf16 / _i8).

bf16: token by token from a random fp32 state, y and the state within 5e-3
(relative L2) of the fp64 recurrence; continuing a scan's final state, the next
token matches the recurrence over the whole sequence.  W8A8: every INT8 state
code bit-exact with the integer oracle's one-token step (and with the scan over
the same tokens when each token ends a chunk), y within 1e-2 of the oracle and
5e-2 of fp64.
"""
import numpy as np
import pytest

from harness import Workload, make_inputs, as_float
from oracle import ssd_fp64 as F
from oracle import ssd_w8a8 as W
from oracle.ssd_fp64 import rel_l2
from tests.gpu_common import TOL_BF16, TOL_I8_Y, bf16_to_np, host, oracle_scales

pytestmark = pytest.mark.gpu
F32 = np.float32

CASES = {
    "2.7b-shape": Workload("dec", 3, 264, 6, 64, 128, 2, 256, seed=21, head_scale=True, outliers=True),
    "small": Workload("dec-small", 2, 70, 8, 16, 16, 2, 64, seed=22),
}


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import int8_quant_b200 as iq
    iq.library()
    return torch


def _token(dev, t):
    return {k: (v[:, t].contiguous() if k in ("x", "dt", "B", "C") else v) for k, v in dev.items()}


@pytest.mark.parametrize("name", list(CASES))
def test_bf16_decode_steps_match_fp64(torch_cuda, name):
    torch = torch_cuda
    from int8_quant_b200.runner import Decoder, to_device
    w = CASES[name]
    inp = make_inputs(w)
    dev = to_device(inp)
    h0 = (0.3 * np.random.default_rng(3).standard_normal((w.batch, w.nheads, w.headdim, w.dstate))).astype(F32)
    dec = Decoder(torch.from_numpy(h0).cuda(), dev["A"], dev["D"], "bf16")
    T = 6
    ys = []
    for t in range(T):
        tk = _token(dev, t)
        ys.append(bf16_to_np(dec.step(tk["x"], tk["dt"], tk["B"], tk["C"]).clone()))
    torch.cuda.synchronize()
    ey, ef = F.ssd_sequential(as_float(inp["x"])[:, :T], inp["dt"][:, :T], inp["A"], as_float(inp["B"])[:, :T],
                              as_float(inp["C"])[:, :T], inp["D"], state0=h0.astype(np.float64))
    for t in range(T):
        assert rel_l2(ys[t], ey[:, t]) <= TOL_BF16, (t, rel_l2(ys[t], ey[:, t]))
    fin = host(dec.state).astype(np.float64)
    assert rel_l2(fin, ef) <= TOL_BF16, rel_l2(fin, ef)


def test_bf16_decode_continues_a_scan(torch_cuda):
    from int8_quant_b200.runner import Decoder, SsdProblem, to_device
    w = CASES["2.7b-shape"]
    inp = make_inputs(w)
    L0 = 256
    pre = {k: (np.ascontiguousarray(v[:, :L0]) if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    pb = SsdProblem(to_device(pre), w.chunk, with_i8=False)
    pb.run_bf16()
    dev = to_device(inp)
    dec = Decoder(pb.final32, dev["A"], dev["D"], "bf16")
    ys = []
    for t in range(L0, w.seqlen):
        tk = _token(dev, t)
        ys.append(bf16_to_np(dec.step(tk["x"], tk["dt"], tk["B"], tk["C"]).clone()))
    torch_cuda.cuda.synchronize()
    ey, ef = F.ssd_sequential(as_float(inp["x"]), inp["dt"], inp["A"], as_float(inp["B"]), as_float(inp["C"]),
                              inp["D"])
    got = np.stack(ys, axis=1)
    assert rel_l2(got, ey[:, L0:]) <= TOL_BF16, rel_l2(got, ey[:, L0:])
    assert rel_l2(host(dec.state).astype(np.float64), ef) <= TOL_BF16


@pytest.mark.parametrize("name,shift", [("2.7b-shape", 7), ("2.7b-shape", 5), ("2.7b-shape", 9), ("small", 7)])
def test_i8_decode_steps_bit_exact(torch_cuda, name, shift):
    """Shifts 5 and 7 take the (P, N) = (64, 128) kernel's two-codes-per-word carry, 9 its
    code-at-a-time one; the (16, 16) shape runs the row kernel."""
    torch = torch_cuda
    from int8_quant_b200.runner import Decoder, to_device
    w = CASES[name]
    inp = make_inputs(w)
    dev = to_device(inp)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    scd = {k: torch.from_numpy(np.asarray(v, F32)).cuda() for k, v in sc.items() if k.startswith("s_")}
    st8 = np.random.default_rng(4).integers(-90, 91, (w.batch, w.nheads, w.headdim, w.dstate)).astype(np.int8)
    dec = Decoder(torch.from_numpy(st8.copy()).cuda(), dev["A"], dev["D"], "w8a8", scd, shift=shift)
    x, Bv, Cv = as_float(inp["x"]).astype(F32), as_float(inp["B"]).astype(F32), as_float(inp["C"]).astype(F32)
    Bq, Cq = W.quantize_inputs(Bv, Cv, sc["s_B"], sc["s_C"])
    ref = st8
    for t in range(8):
        tk = _token(dev, t)
        y = bf16_to_np(dec.step(tk["x"], tk["dt"], tk["B"], tk["C"]).clone())
        torch.cuda.synchronize()
        r = W.decode_step_i8(x[:, t], inp["dt"][:, t], inp["A"], Bq[:, t], Cq[:, t], inp["D"], sc["s_B"], sc["s_C"],
                             sc["s_x"], sc["s_s"], ref, k=shift)
        np.testing.assert_array_equal(host(dec.state), r["state8"])
        assert rel_l2(y, r["y"]) <= 1e-2, (t, rel_l2(y, r["y"]))
        ref = r["state8"]
    if shift != 7:                                  # coarser or finer decay codes: the integers decide
        return
    H, P = w.nheads, w.headdim
    ss = np.asarray(sc["s_s"], np.float64).reshape(H, P)[None, :, :, None]
    ey, _ = F.ssd_sequential(as_float(inp["x"])[:, :8], inp["dt"][:, :8], inp["A"], as_float(inp["B"])[:, :8],
                             as_float(inp["C"])[:, :8], inp["D"], state0=st8.astype(np.float64) * ss)
    assert rel_l2(y, ey[:, 7]) <= TOL_I8_Y, rel_l2(y, ey[:, 7])


def test_i8_decode_after_a_scan_equals_the_longer_scan(torch_cuda):
    torch = torch_cuda
    from int8_quant_b200.runner import Decoder, SsdProblem, to_device
    w = CASES["2.7b-shape"]                       # chunk 256; tokens 256.. each end a chunk of their own
    inp = make_inputs(w)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    L0 = 256
    cut = lambda n: {k: (np.ascontiguousarray(v[:, :n]) if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    pb0 = SsdProblem(to_device(cut(L0)), w.chunk, with_bf16=False)
    pb1 = SsdProblem(to_device(cut(L0 + 1)), w.chunk, with_bf16=False)
    for pb in (pb0, pb1):
        pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
        pb.run_i8()
    dev = to_device(inp)
    dec = Decoder(pb0.final8, dev["A"], dev["D"], "w8a8", pb0.scales)
    tk = _token(dev, L0)
    y = dec.step(tk["x"], tk["dt"], tk["B"], tk["C"])
    torch.cuda.synchronize()
    assert torch.equal(dec.state, pb1.final8)
    assert rel_l2(bf16_to_np(y), bf16_to_np(pb1.y[:, L0])) <= 1e-2
