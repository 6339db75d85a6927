"""GPU parity of the notes' storage variant (`ssd_i8_params.storage`).

SSD_STORAGE_ACS_FP16 keeps the cumulative sums Acs as IEEE half and SSD_STORAGE_CB_INT8
requantises each (b, c, g) CB tile to INT8 in HBM ("SSDi8" notes, overall framework and
key design 2).  The integer oracle takes the same two readings as switches (acs_fp16,
cb_int8), so every integer is compared bit for bit: the half-rounded Acs, the decay
codes, Xq, the ChunkState accumulators and codes, the passed and final states, the
ChunkScan1 accumulators, the full INT32 CB tiles, their INT8 codes and fp64 steps; y
is held to the oracle's dequantised y (1e-2) and to the fp64 definition (5e-2).  The
variant's outputs start as values no kernel writes, so an unwritten element fails.
"""
import numpy as np
import pytest

from harness import Workload, make_inputs
from oracle.ssd_fp64 import rel_l2
from tests.gpu_common import TOL_I8_Y, bf16_to_np, host, oracle_fp64, oracle_i8, oracle_scales, poison

pytestmark = pytest.mark.gpu

CASES = {
    "ragged-g2": Workload("ragged-g2", 2, 1000, 6, 64, 128, 2, 256, head_scale=True, outliers=True),
    "g1": Workload("g1", 1, 600, 4, 64, 128, 1, 256, seed=8),
}


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import int8_quant_b200 as iq
    iq.library()
    return torch


@pytest.mark.parametrize("storage", [1, 2, 3])
@pytest.mark.parametrize("name", list(CASES))
def test_storage_variant_bit_exact(torch_cuda, name, storage):
    from int8_quant_b200.runner import SsdProblem, to_device
    torch = torch_cuda
    w = CASES[name]
    inp = make_inputs(w)
    pb = SsdProblem(to_device(inp), w.chunk, with_bf16=False)
    poison(torch, pb)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7, storage)
    dbg = pb.run_i8_debug()
    torch.cuda.synchronize()
    r = oracle_i8(inp, sc, w.chunk, 7, acs_fp16=bool(storage & 1), cb_int8=bool(storage & 2))
    for k in ("Acs", "dq", "Xq", "acc_state", "S8", "H8", "acc_scan1"):
        np.testing.assert_array_equal(host(dbg[k]), r[k], err_msg=k)
    np.testing.assert_array_equal(host(pb.final8), r["final8"])
    cb = host(dbg["cb"])
    if storage & 2:
        np.testing.assert_array_equal(cb, r["CB"])                      # every entry of the tile
        np.testing.assert_array_equal(host(dbg["cb8"]), r["CB8"])
        np.testing.assert_array_equal(host(dbg["s_cb"]), r["s_cb"][..., 0, 0])
    else:
        low = np.tril(np.ones((w.chunk, w.chunk), dtype=bool))
        np.testing.assert_array_equal(cb[..., low], r["CB"][..., low])
    y = bf16_to_np(pb.y)
    assert rel_l2(y, r["y"]) <= 1e-2, rel_l2(y, r["y"])
    ey, _ = oracle_fp64(inp)
    assert rel_l2(y, ey) <= TOL_I8_Y, rel_l2(y, ey)


def test_storage_variant_production_equals_debug(torch_cuda):
    torch = torch_cuda
    from int8_quant_b200.runner import SsdProblem, to_device
    w = CASES["ragged-g2"]
    inp = make_inputs(w)
    pb = SsdProblem(to_device(inp), w.chunk, with_bf16=False)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7, 3)
    pb.run_i8_debug()
    y1, f1 = pb.y.clone(), pb.final8.clone()
    poison(torch, pb)
    pb.run_i8()
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), pb.y.view(torch.int16)) and torch.equal(f1, pb.final8)


def test_storage_variant_needs_chunk_256(torch_cuda):
    import int8_quant_b200 as iq
    from int8_quant_b200.runner import SsdProblem, to_device
    w = Workload("q128", 1, 300, 4, 64, 128, 1, 128, seed=9)
    inp = make_inputs(w)
    pb = SsdProblem(to_device(inp), w.chunk, with_bf16=False)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7, 3)
    with pytest.raises(iq.SsdError) as e:
        pb.run_i8()
    assert e.value.status == 2                                            # SSD_ERR_UNSUPPORTED
