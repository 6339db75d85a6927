"""GPU parity at the full workload sizes, on sampled (batch, head) chains.

Each test runs the whole workload through the same entry points the bench times;
the oracle then regenerates only the sampled chains' inputs (the generator is
counter-based) and recomputes them on the host:
* bf16: y and the final state of each sampled chain within 5e-3 (relative L2)
  of the fp64 recurrence;
* W8A8 (scales from the oracle's calibration on the 512-token prefix): every
  integer intermediate of the sampled chains bit-exact (Acs, decay codes, Xq,
  ChunkState INT32 accumulators, S8, passed INT8 states, ChunkScan1 INT32
  accumulators, ChunkBMM accumulators of the chain's group, final INT8 state),
  y within 1e-2 of the integer oracle's dequantised y and within 5e-2 of fp64;
* the library's GPU calibration agrees with the oracle's within 1e-4.
The long-context sweeps (B = 1, L = 64K and 256K: 256 and 1024 chunks through
StatePassing) run by default; their inputs take a minute or two to generate, once per
workload for both paths.  SSD_FULLSIZE_LONG=0 leaves them out.
"""
import functools
import os

import numpy as np
import pytest

from harness import WORKLOADS, make_inputs
from oracle.ssd_fp64 import rel_l2
from tests.gpu_common import (TOL_BF16, TOL_I8_Y, bf16_to_np, host, chain_oracle, chain_oracle_i8,
                              full_size_scales)

pytestmark = pytest.mark.gpu

LONG = os.environ.get("SSD_FULLSIZE_LONG", "1") == "1"
BF16_WORKLOADS = ["mamba2-1.3b", "mamba2-2.7b", "long-16k"] + (["long-64k", "long-256k"] if LONG else [])
I8_WORKLOADS = ["mamba2-2.7b", "mamba2-8b", "long-16k"] + (["long-64k", "long-256k"] if LONG else [])


def _samples(w, n=3):
    rs = np.random.default_rng(12345)
    pts = {(0, 0), (w.batch - 1, w.nheads - 1)}
    while len(pts) < n:
        pts.add((int(rs.integers(w.batch)), int(rs.integers(w.nheads))))
    return sorted(pts)


@pytest.fixture(scope="module")
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import int8_quant_b200 as iq
    iq.library()
    return torch


@functools.lru_cache(maxsize=None)
def _inputs(name):
    """Host inputs of a workload, generated once for both paths."""
    return make_inputs(WORKLOADS[name])


def _run(cuda, w, i8: bool, scales=None, debug=False):
    from int8_quant_b200.runner import SsdProblem, to_device
    pb = SsdProblem(to_device(_inputs(w.name)), w.chunk, with_i8=i8, with_bf16=not i8)
    dbg = None
    if not i8:
        pb.run_bf16()
    else:
        pb.set_scales(scales["s_B"], scales["s_C"], scales["s_x"], scales["s_s"], 7)
        dbg = pb.run_i8_debug() if debug else None
        if not debug:
            pb.run_i8()
    cuda.cuda.synchronize()
    return pb, dbg


@pytest.mark.parametrize("name", BF16_WORKLOADS)
def test_fullsize_bf16_sampled_chains(cuda, name):
    w = WORKLOADS[name]
    pb, _ = _run(cuda, w, i8=False)
    for b, h in _samples(w):
        ey, ef, _ = chain_oracle(w, b, h)
        y = bf16_to_np(pb.y[b, :, h, :])
        fin = host(pb.final32[b, h]).astype(np.float64)
        assert rel_l2(y, ey) <= TOL_BF16, (b, h, rel_l2(y, ey))
        assert rel_l2(fin, ef) <= TOL_BF16, (b, h, rel_l2(fin, ef))
    del pb
    cuda.cuda.empty_cache()


@pytest.mark.parametrize("name", I8_WORKLOADS)
def test_fullsize_w8a8_sampled_chains_bit_exact(cuda, name):
    w = WORKLOADS[name]
    sc = full_size_scales(w)
    pb, dbg = _run(cuda, w, i8=True, scales=sc, debug=True)
    Q, P = w.chunk, w.headdim
    L, nc = w.seqlen, w.nchunks
    low = np.tril(np.ones((Q, Q), dtype=bool))
    for b, h in _samples(w):
        r = chain_oracle_i8(w, b, h, sc)
        g = r["g"]
        np.testing.assert_array_equal(host(pb.Bq[b, :, g, :]), r["Bq"][0, :, 0, :])
        np.testing.assert_array_equal(host(pb.Cq[b, :, g, :]), r["Cq"][0, :, 0, :])
        np.testing.assert_array_equal(host(dbg["Acs"][b, h]), r["Acs"][0, 0])
        np.testing.assert_array_equal(host(dbg["dq"][b, h]), r["dq"][0, 0])
        np.testing.assert_array_equal(host(dbg["Xq"][b, :, h, :]), r["Xq"][0, :, 0, :])
        np.testing.assert_array_equal(host(dbg["acc_state"][b, :, h]), r["acc_state"][0, :, 0])
        np.testing.assert_array_equal(host(dbg["S8"][b, :, h]), r["S8"][0, :, 0])
        np.testing.assert_array_equal(host(dbg["H8"][b, :, h]), r["H8"][0, :, 0])
        np.testing.assert_array_equal(host(dbg["acc_scan1"][b, :, h, :]), r["acc_scan1"][0, :, 0, :])
        np.testing.assert_array_equal(host(pb.final8[b, h]), r["final8"][0, 0])
        cb = host(dbg["cb"][b, :, g])
        np.testing.assert_array_equal(cb[:, low], r["CB"][0, :, 0][:, low])
        y = bf16_to_np(pb.y[b, :, h, :])
        assert rel_l2(y, r["y"][0, :, 0, :]) <= 1e-2, (b, h, rel_l2(y, r["y"][0, :, 0, :]))
        ey, _, _ = chain_oracle(w, b, h)
        assert rel_l2(y, ey) <= TOL_I8_Y, (b, h, rel_l2(y, ey))
    del pb, dbg
    cuda.cuda.empty_cache()


@pytest.mark.parametrize("name", ["mamba2-2.7b", "mamba2-8b"])
def test_fullsize_gpu_calibration_matches_oracle(cuda, name):
    from int8_quant_b200.runner import SsdProblem, to_device
    w = WORKLOADS[name]
    pb = SsdProblem(to_device(make_inputs(w)), w.chunk, with_i8=True, with_bf16=False)
    got = pb.calibrate(w.calib_prefix)
    cuda.cuda.synchronize()
    ref = full_size_scales(w)
    for k in ("s_B", "s_C"):
        np.testing.assert_allclose(host(got[k]), ref[k], rtol=1e-6)
    for k in ("s_x", "s_s"):
        np.testing.assert_allclose(host(got[k]), ref[k], rtol=1e-4)
    del pb
    cuda.cuda.empty_cache()
