"""ssd_scan_fwd_bf16_static: the bf16 scan for callers that cannot allocate device memory.

Such callers (an arena that owns all device memory, a plugin that may not call
cudaMalloc) cannot pass a workspace, so this entry point uses the library's fixed
32 MiB device scratch instead.  The test calls it through the C ABI twice in a row,
on two different problems (the larger first, so that stale scratch contents would show),
and checks each result against the regular ssd_scan_fwd_bf16 with a caller-allocated
workspace: the same kernels on the same inputs, so the results must be identical bit for
bit; the scratch's status word reads SSD_OK after each call.  Then it checks that a
problem too large for the scratch is refused.
"""
import ctypes

import pytest

from harness import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _static_call(lib, pb):
    i = pb.inp
    import torch
    st = torch.cuda.current_stream().cuda_stream
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.ssd_scan_fwd_bf16_static(ctypes.byref(pb.shape), p(i["x"]), p(i["dt"]), p(i["A"]), p(i["B"]),
                                        p(i["C"]), p(i["D"]), p(pb.y), p(pb.final32), ctypes.c_void_p(st))


def test_static_scratch_matches_workspace_call_twice_in_a_row():
    import torch
    assert torch.cuda.is_available()
    import int8_quant_b200 as iq
    from int8_quant_b200.runner import SsdProblem, to_device
    lib = iq.library()
    problems = [Workload("s1", 2, 1000, 6, 64, 128, 2, 256, head_scale=True, outliers=True, seed=11),
                Workload("s2", 3, 77, 8, 16, 16, 2, 64, seed=12)]
    for w in problems:
        shape = iq.SsdShape.of(w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk)
        assert iq.ssd_workspace_bytes(shape, False) <= 32 << 20
    for w in problems:
        pb = SsdProblem(to_device(make_inputs(w)), w.chunk, with_i8=False)
        pb.run_bf16()                          # regular entry point, caller workspace
        torch.cuda.synchronize()
        y_ref, f_ref = pb.y.clone(), pb.final32.clone()
        pb.y.fill_(float("nan"))
        pb.final32.fill_(float("nan"))
        assert _static_call(lib, pb) == 0
        assert lib.ssd_static_scratch_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
        torch.cuda.synchronize()
        assert torch.equal(pb.y.view(torch.int16), y_ref.view(torch.int16))
        assert torch.equal(pb.final32, f_ref)


def test_static_scratch_rejects_problems_that_do_not_fit():
    import torch
    import int8_quant_b200 as iq
    lib = iq.library()
    big = iq.SsdShape.of(8, 8192, 80, 64, 1, 128, 256)       # needs ~1 GB of scratch
    assert iq.ssd_workspace_bytes(big, False) > 32 << 20
    y = torch.full((4,), 7.0, device="cuda")
    fake = ctypes.c_void_p(y.data_ptr())
    st = lib.ssd_scan_fwd_bf16_static(ctypes.byref(big), fake, fake, fake, fake, fake, fake, fake, fake,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 3                                           # SSD_ERR_WORKSPACE, nothing enqueued
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
