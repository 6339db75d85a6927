"""GPU parity of the single-kernel W8A8 scan (fused_i8.cu, selected with SSD_I8_FUSED=1).

The fused kernel runs ChunkCumsum, ChunkState, StatePassing (as a link inside each work
item, passed between items through flags), ChunkBMM and ChunkScan in one persistent
launch.  It must give the integer oracle's intermediates bit for bit (every chunk's
Acs, decay code, Xq, INT32 ChunkState accumulator, S8, passed INT8 state, ChunkBMM and
ChunkScan1 accumulators, and the final state), and y and the final state identical to
the five-launch path (same floating-point operations in the same order).  Cases cover
chunks 64/128/256, ragged final chunks, several groups, a ragged last head block, decay
shifts 5 and 9 (the packed and the generic StatePassing link), a scan continued from a
state across a chunk boundary, and sampled chains at full size.
"""
import os

import numpy as np
import pytest

from harness import Workload, WORKLOADS, make_inputs, as_float
from oracle import ssd_w8a8 as W
from oracle.ssd_fp64 import rel_l2
from tests.gpu_common import (TOL_I8_Y, bf16_to_np, host, oracle_fp64, oracle_i8, oracle_scales, chain_oracle,
                              chain_oracle_i8, full_size_scales, poison)

pytestmark = pytest.mark.gpu

CASES = {
    "ragged-q256": Workload("ragged-q256", 2, 1000, 6, 64, 128, 2, 256, head_scale=True, outliers=True),
    "ragged-q128": Workload("ragged-q128", 1, 700, 4, 64, 128, 1, 128, seed=1),
    "ragged-q64": Workload("ragged-q64", 2, 333, 4, 64, 128, 4, 64, seed=2),
    "L1": Workload("L1", 2, 1, 4, 64, 128, 1, 256, seed=4),
    "ragged-heads": Workload("ragged-heads", 1, 512, 20, 64, 128, 1, 256, seed=6),
    "g1-ragged": Workload("g1-ragged", 2, 1000, 6, 64, 128, 1, 256, seed=7, head_scale=True, outliers=True),
}
F32 = np.float32


@pytest.fixture
def fused(monkeypatch):
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import int8_quant_b200 as iq
    iq.library()
    monkeypatch.setenv("SSD_I8_FUSED", "1")
    return torch


def _problem(w, inp=None):
    import torch
    from int8_quant_b200.runner import SsdProblem, to_device
    inp = make_inputs(w) if inp is None else inp
    pb = SsdProblem(to_device(inp), w.chunk, with_bf16=False)
    poison(torch, pb)
    return inp, pb


def _check_against_oracle(torch, w, shift=7):
    inp, pb = _problem(w)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], shift)
    dbg = pb.run_i8_debug()
    torch.cuda.synchronize()
    r = oracle_i8(inp, sc, w.chunk, shift)
    for k in ("Acs", "dq", "Xq", "acc_state", "S8", "H8", "acc_scan1"):
        np.testing.assert_array_equal(host(dbg[k]), r[k], err_msg=k)
    np.testing.assert_array_equal(host(pb.final8), r["final8"])
    low = np.tril(np.ones((w.chunk, w.chunk), dtype=bool))
    np.testing.assert_array_equal(host(dbg["cb"])[..., low], r["CB"][..., low])
    y = bf16_to_np(pb.y)
    assert rel_l2(y, r["y"]) <= 1e-2, rel_l2(y, r["y"])
    ey, _ = oracle_fp64(inp)
    assert rel_l2(y, ey) <= TOL_I8_Y, rel_l2(y, ey)
    return inp, pb


@pytest.mark.parametrize("name", ["ragged-q256", "ragged-q128", "ragged-q64", "L1"])
def test_fused_bit_exact(fused, name):
    _check_against_oracle(fused, CASES[name])


def test_fused_ragged_last_head_block(fused, monkeypatch):
    """20 heads in items of 8: blocks of 8, 8 and 4 heads."""
    monkeypatch.setenv("SSD_FUSED_HEADS", "8")
    _check_against_oracle(fused, CASES["ragged-heads"])


@pytest.mark.parametrize("shift", [5, 9])
def test_fused_other_decay_shifts(fused, shift):
    """k = 5 runs the packed StatePassing link, k = 9 the code-at-a-time one."""
    _check_against_oracle(fused, CASES["ragged-q256"], shift)


@pytest.mark.parametrize("name", ["ragged-q256", "ragged-q64", "ragged-heads", "g1-ragged"])
def test_fused_equals_staged(fused, name, monkeypatch):
    """Same y and final state, bit for bit, as the five-launch path; every output written
    (y starts as NaN bit patterns, the state as an out-of-range code, before each run)."""
    torch = fused
    w = CASES[name]
    inp, pb = _problem(w)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
    out = []
    for flag in ("1", "0"):
        monkeypatch.setenv("SSD_I8_FUSED", flag)
        pb.y.view(torch.int16).fill_(-1)
        pb.final8.fill_(-128)
        pb.run_i8()
        torch.cuda.synchronize()
        out.append((pb.y.view(torch.int16).clone(), pb.final8.clone()))
    for y, fin in out:
        assert not bool((y == -1).any()) and not bool((fin == -128).any())
    assert torch.equal(out[0][1], out[1][1])
    assert torch.equal(out[0][0], out[1][0]), int((out[0][0] != out[1][0]).sum())


def test_fused_production_equals_debug(fused):
    torch = fused
    w = CASES["ragged-q256"]
    inp, pb = _problem(w)
    sc = oracle_scales(inp, w.chunk)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"])
    pb.run_i8_debug()
    y1, f1 = pb.y.clone(), pb.final8.clone()
    pb.y.zero_()
    pb.final8.zero_()
    pb.run_i8()
    torch.cuda.synchronize()
    assert torch.equal(y1, pb.y) and torch.equal(f1, pb.final8)


def test_fused_split_at_a_chunk_boundary(fused):
    """The second half started from the first half's INT8 state equals one call."""
    torch = fused
    w = Workload("split", 2, 1024, 6, 64, 128, 2, 256, seed=4, head_scale=True, outliers=True)
    inp = make_inputs(w)
    cut = 512
    sl = lambda a, b: {k: (np.ascontiguousarray(v[:, a:b]) if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    parts = [_problem(w, inp)[1], _problem(w, sl(0, cut))[1], _problem(w, sl(cut, w.seqlen))[1]]
    for pb in parts:
        pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
    whole, first, second = parts
    whole.run_i8()
    first.run_i8()
    second.run_i8(initial_state=first.final8)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([first.y, second.y], dim=1), whole.y)
    assert torch.equal(second.final8, whole.final8)


@pytest.mark.parametrize("name", ["mamba2-2.7b", "long-16k"])
def test_fused_fullsize_sampled_chains_bit_exact(fused, name):
    torch = fused
    w = WORKLOADS[name]
    sc = full_size_scales(w)
    inp, pb = _problem(w)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
    dbg = pb.run_i8_debug()
    torch.cuda.synchronize()
    rs = np.random.default_rng(54321)
    pts = {(0, 0), (w.batch - 1, w.nheads - 1), (int(rs.integers(w.batch)), int(rs.integers(w.nheads)))}
    for b, h in sorted(pts):
        r = chain_oracle_i8(w, b, h, sc)
        np.testing.assert_array_equal(host(dbg["Xq"][b, :, h, :]), r["Xq"][0, :, 0, :])
        np.testing.assert_array_equal(host(dbg["S8"][b, :, h]), r["S8"][0, :, 0])
        np.testing.assert_array_equal(host(dbg["H8"][b, :, h]), r["H8"][0, :, 0])
        np.testing.assert_array_equal(host(dbg["acc_scan1"][b, :, h, :]), r["acc_scan1"][0, :, 0, :])
        np.testing.assert_array_equal(host(pb.final8[b, h]), r["final8"][0, 0])
        y = bf16_to_np(pb.y[b, :, h, :])
        assert rel_l2(y, r["y"][0, :, 0, :]) <= 1e-2, (b, h, rel_l2(y, r["y"][0, :, 0, :]))
        ey, _, _ = chain_oracle(w, b, h)
        assert rel_l2(y, ey) <= TOL_I8_Y, (b, h, rel_l2(y, ey))
    del pb, dbg
    torch.cuda.empty_cache()
