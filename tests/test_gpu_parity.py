"""GPU parity: the CUDA path against the oracle, element by element (bf16 and W8A8).

Sizes span several chunks, heads and groups, with a ragged final chunk; edge
cases cover L=1, L shorter than a chunk, L=0 and batch 0.  bf16: relative L2 of
y and the final state <= 5e-3 against the fp64 recurrence.  W8A8: every integer
intermediate bit-exact against the integer oracle, y within 5e-2 of fp64.
"""
import numpy as np
import pytest

from harness import Workload, WORKLOADS, make_inputs
from oracle.ssd_fp64 import rel_l2
from tests.gpu_common import (TOL_BF16, TOL_I8_Y, bf16_to_np, host, oracle_fp64, oracle_i8, oracle_scales, poison)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": WORKLOADS["tiny"],
    "ragged-q256": Workload("ragged-q256", 2, 1000, 6, 64, 128, 2, 256, head_scale=True, outliers=True),
    "ragged-q128": Workload("ragged-q128", 1, 700, 4, 64, 128, 1, 128, seed=1),
    "ragged-q64": Workload("ragged-q64", 2, 333, 4, 64, 128, 4, 64, seed=2),
    "tiny-ragged": Workload("tiny-ragged", 3, 77, 8, 16, 16, 2, 64, seed=3),
    "L1": Workload("L1", 2, 1, 4, 64, 128, 1, 256, seed=4),
    "L63": Workload("L63", 1, 63, 4, 16, 16, 1, 64, seed=5),
    # 20 heads: the tensor-core ChunkScan takes them in blocks of 8, 8 and 4
    "ragged-heads": Workload("ragged-heads", 1, 512, 20, 64, 128, 1, 256, seed=6),
}


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import int8_quant_b200 as iq
    iq.library()            # the CUDA library must be present: no fallback
    return torch


def _problem(torch_cuda, w):
    """Inputs and device buffers; the outputs start as NaN bit patterns (y, fp32 state) and
    code -128 (INT8 state), so that an element the kernels never write fails the checks."""
    from int8_quant_b200.runner import SsdProblem, to_device
    inp = make_inputs(w)
    pb = SsdProblem(to_device(inp), w.chunk)
    poison(torch_cuda, pb)
    return inp, pb


@pytest.mark.parametrize("name", list(CASES))
def test_bf16_matches_fp64(torch_cuda, name):
    w = CASES[name]
    inp, pb = _problem(torch_cuda, w)
    pb.run_bf16()
    torch_cuda.cuda.synchronize()
    y = bf16_to_np(pb.y)
    fin = host(pb.final32).astype(np.float64)
    ey, ef = oracle_fp64(inp)
    assert rel_l2(y, ey) <= TOL_BF16, rel_l2(y, ey)
    assert rel_l2(fin, ef) <= TOL_BF16, rel_l2(fin, ef)


@pytest.mark.parametrize("name", list(CASES))
def test_i8_bit_exact_and_within_tolerance(torch_cuda, name):
    w = CASES[name]
    inp, pb = _problem(torch_cuda, w)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
    dbg = pb.run_i8_debug()
    torch_cuda.cuda.synchronize()
    r = oracle_i8(inp, sc, w.chunk)
    np.testing.assert_array_equal(host(pb.Bq), r["Bq"])
    np.testing.assert_array_equal(host(pb.Cq), r["Cq"])
    np.testing.assert_array_equal(host(dbg["Acs"]), r["Acs"])
    np.testing.assert_array_equal(host(dbg["dq"]), r["dq"])
    np.testing.assert_array_equal(host(dbg["Xq"]), r["Xq"])
    np.testing.assert_array_equal(host(dbg["acc_state"]), r["acc_state"])
    np.testing.assert_array_equal(host(dbg["S8"]), r["S8"])
    np.testing.assert_array_equal(host(dbg["H8"]), r["H8"])
    np.testing.assert_array_equal(host(pb.final8), r["final8"])
    np.testing.assert_array_equal(host(dbg["acc_scan1"]), r["acc_scan1"])
    cb = host(dbg["cb"])
    low = np.tril(np.ones((w.chunk, w.chunk), dtype=bool))
    np.testing.assert_array_equal(cb[..., low], r["CB"][..., low])
    y = bf16_to_np(pb.y)
    assert rel_l2(y, r["y"]) <= 1e-2, rel_l2(y, r["y"])        # float tail vs the integer oracle
    ey, _ = oracle_fp64(inp)
    assert rel_l2(y, ey) <= TOL_I8_Y, rel_l2(y, ey)


@pytest.mark.parametrize("shift", [5, 9])
def test_i8_other_decay_shifts_bit_exact(torch_cuda, shift):
    """Decay shift 5 takes StatePassing's two-codes-per-field carry, 9 its code-at-a-time one."""
    w = CASES["ragged-q256"]
    inp, pb = _problem(torch_cuda, w)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], shift)
    dbg = pb.run_i8_debug()
    torch_cuda.cuda.synchronize()
    r = oracle_i8(inp, sc, w.chunk, shift)
    for k in ("dq", "S8", "H8", "acc_scan1"):
        np.testing.assert_array_equal(host(dbg[k]), r[k], err_msg=k)
    np.testing.assert_array_equal(host(pb.final8), r["final8"])
    assert rel_l2(bf16_to_np(pb.y), r["y"]) <= 1e-2


def test_i8_production_call_equals_debug_call(torch_cuda):
    w = CASES["ragged-q256"]
    inp, pb = _problem(torch_cuda, w)
    sc = oracle_scales(inp, w.chunk)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"])
    pb.run_i8_debug()
    y1, f1 = pb.y.clone(), pb.final8.clone()
    pb.y.zero_()
    pb.final8.zero_()
    pb.run_i8()
    torch_cuda.cuda.synchronize()
    assert torch_cuda.equal(y1, pb.y) and torch_cuda.equal(f1, pb.final8)


@pytest.mark.parametrize("name", ["tiny", "ragged-q256", "ragged-q64"])
def test_calibration_matches_oracle(torch_cuda, name):
    w = CASES[name]
    inp, pb = _problem(torch_cuda, w)
    got = pb.calibrate(w.calib_prefix)
    torch_cuda.cuda.synchronize()
    ref = oracle_scales(inp, w.chunk, w.calib_prefix)
    for k in ("s_B", "s_C"):
        np.testing.assert_allclose(host(got[k]), ref[k], rtol=1e-6)
    for k in ("s_x", "s_s"):
        np.testing.assert_allclose(host(got[k]), ref[k], rtol=1e-4)


def test_seqlen_zero_and_batch_zero(torch_cuda):
    torch = torch_cuda
    from int8_quant_b200.runner import SsdProblem, to_device
    w = Workload("L0", 2, 0, 4, 64, 128, 1, 256)
    inp = make_inputs(w)
    pb = SsdProblem(to_device(inp), w.chunk)
    pb.final32.fill_(7.0)
    pb.run_bf16()
    pb.set_scales(np.ones(1), np.ones(1), np.ones(4 * 64), np.ones(4 * 64))
    pb.final8.fill_(7)
    pb.run_i8()
    torch.cuda.synchronize()
    assert torch.count_nonzero(pb.final32) == 0 and torch.count_nonzero(pb.final8) == 0
    w0 = Workload("B0", 0, 128, 4, 64, 128, 1, 256)
    pb0 = SsdProblem(to_device(make_inputs(w0)), w0.chunk)
    pb0.run_bf16()
    torch.cuda.synchronize()


def test_chunk_size_invariance_bf16(torch_cuda):
    """bf16 results at chunk 64, 128 and 256 agree within tolerance (the method is exact in chunking)."""
    base = Workload("inv", 1, 768, 4, 64, 128, 1, 64, seed=9)
    outs = []
    for q in (64, 128, 256):
        inp, pb = _problem(torch_cuda, base.with_(chunk=q))
        pb.run_bf16()
        torch_cuda.cuda.synchronize()
        outs.append((bf16_to_np(pb.y), host(pb.final32).astype(np.float64)))
    for y, f in outs[1:]:
        assert rel_l2(y, outs[0][0]) <= TOL_BF16 and rel_l2(f, outs[0][1]) <= TOL_BF16


def test_workspace_status_is_ok_after_a_run(torch_cuda):
    import int8_quant_b200 as iq
    inp, pb = _problem(torch_cuda, CASES["tiny"])
    pb.run_bf16()
    assert iq.ssd_workspace_status(pb.ws_bf16) == 0


@pytest.mark.parametrize("path", ["bf16", "w8a8"])
@pytest.mark.parametrize("name", ["ragged-q256", "ragged-q64"])
def test_streamed_segments_equal_whole_batch(torch_cuda, name, path):
    """Host-resident batch streamed one row's segment of 2 chunks at a time, each segment
    continuing from the previous one's state (the last one ragged): y and the final
    state equal the whole-batch call bit for bit."""
    from int8_quant_b200.runner import StreamedScan
    torch = torch_cuda
    w = CASES[name].with_(batch=3)
    inp, pb = _problem(torch_cuda, w)
    if path == "w8a8":
        sc = oracle_scales(inp, w.chunk, w.calib_prefix)
        pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
        pb.run_i8()
        fin = pb.final8
    else:
        pb.run_bf16()
        fin = pb.final32
    torch.cuda.synchronize()
    host = {k: pb.inp[k].to("cpu").pin_memory() for k in ("x", "dt", "B", "C")}
    host["y"] = torch.empty_like(pb.y, device="cpu").pin_memory()
    host["final"] = torch.empty_like(fin, device="cpu").pin_memory()
    run = StreamedScan(host, pb.inp["A"], pb.inp["D"], w.chunk, path, rows_per_group=1,
                       scales=pb.scales if path == "w8a8" else None, seg_len=2 * w.chunk)
    assert len(run.groups) == 3 * ((w.seqlen + 2 * w.chunk - 1) // (2 * w.chunk)) > 3
    for _ in range(2):
        host["y"].view(torch.int16).fill_(-1)
        run.run()
        torch.cuda.synchronize()
        assert torch.equal(host["y"].view(torch.int16), pb.y.cpu().view(torch.int16))
        assert torch.equal(host["final"], fin.cpu())


@pytest.mark.parametrize("path", ["bf16", "w8a8"])
@pytest.mark.parametrize("name", ["ragged-q256", "tiny-ragged"])
def test_streamed_batch_equals_whole_batch(torch_cuda, name, path):
    """Host-resident batch run group by group with overlapped copies (two rows per group,
    so the last group is partial for an odd batch) gives the whole-batch results bit for bit."""
    from int8_quant_b200.runner import StreamedScan
    torch = torch_cuda
    w = CASES[name].with_(batch=3)
    inp, pb = _problem(torch_cuda, w)
    if path == "w8a8":
        sc = oracle_scales(inp, w.chunk, w.calib_prefix)
        pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
        pb.run_i8()
        fin = pb.final8
    else:
        pb.run_bf16()
        fin = pb.final32
    torch.cuda.synchronize()
    host = {k: pb.inp[k].to("cpu").pin_memory() for k in ("x", "dt", "B", "C")}
    host["y"] = torch.empty_like(pb.y, device="cpu").pin_memory()
    host["final"] = torch.empty_like(fin, device="cpu").pin_memory()
    run = StreamedScan(host, pb.inp["A"], pb.inp["D"], w.chunk, path, rows_per_group=2,
                       scales=pb.scales if path == "w8a8" else None)
    for _ in range(2):                      # a second pass reuses the slots behind the first
        host["y"].zero_()
        run.run()
        torch.cuda.synchronize()
        assert torch.equal(host["y"].view(torch.int16), pb.y.cpu().view(torch.int16))
        assert torch.equal(host["final"], fin.cpu())
