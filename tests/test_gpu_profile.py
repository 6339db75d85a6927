"""The library's per-kernel timing (instrumentation used by the bench): with a stage filter only
that kernel is timed; without it every stage of a W8A8 step is, once per step."""
import pytest

from harness import Workload, make_inputs
from tests.gpu_common import oracle_scales

pytestmark = pytest.mark.gpu


def test_profile_filter_times_only_the_named_kernel():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import int8_quant_b200 as iq
    from int8_quant_b200.runner import SsdProblem, to_device
    w = Workload("prof", 1, 512, 4, 64, 128, 1, 256, seed=12)
    inp = make_inputs(w)
    pb = SsdProblem(to_device(inp), w.chunk, with_bf16=False)
    sc = oracle_scales(inp, w.chunk, w.calib_prefix)
    pb.set_scales(sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"], 7)
    try:
        iq.ssd_profile_filter(None)
        iq.ssd_profile_reset()
        iq.ssd_profile_enable(True)
        for _ in range(3):
            pb.run_i8()
        torch.cuda.synchronize()
        iq.ssd_profile_enable(False)
        every = {k: v for k, v in iq.ssd_profile_read().items() if v[1]}
        assert set(every) == {"quantize_inputs", "chunk_cumsum", "chunk_state", "state_passing", "chunk_scan"}
        assert all(c == 3 and t > 0 for t, c in every.values())
        iq.ssd_profile_reset()
        iq.ssd_profile_filter("chunk_scan")
        iq.ssd_profile_enable(True)
        for _ in range(2):
            pb.run_i8()
        torch.cuda.synchronize()
        iq.ssd_profile_enable(False)
        one = {k: v for k, v in iq.ssd_profile_read().items() if v[1]}
        assert set(one) == {"chunk_scan"} and one["chunk_scan"][1] == 2
    finally:
        iq.ssd_profile_enable(False)
        iq.ssd_profile_filter(None)
        iq.ssd_profile_reset()
