"""Device-side bounded waits on the GPU, without a fault: a wait that nothing will
ever satisfy must end with SSD_ERR_TIMEOUT in the status word, a second wait in the
same CTA must leave early through the CTA's abort flag, and the context must stay
usable for the scan afterwards."""
import pytest

from harness import WORKLOADS

pytestmark = pytest.mark.gpu

LIMIT = 2_000_000            # cycles, about a millisecond at the B200 clocks
FULL_LIMIT = 4_000_000_000   # the kernels' own limit (about two seconds)


def test_expired_wait_reports_timeout_and_aborts_the_rest_of_the_cta():
    import torch
    import int8_quant_b200 as iq
    iq.library()
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    cycles = torch.zeros(2, dtype=torch.int64, device="cuda")
    iq.ssd_selftest_bounded_wait(LIMIT, status, cycles)
    torch.cuda.synchronize()
    assert int(status.item()) == 5                      # SSD_ERR_TIMEOUT
    c0, c1 = (int(v) for v in cycles.cpu())
    assert c0 >= LIMIT                                  # warp 0 waited out its own limit ...
    assert c0 < FULL_LIMIT // 4                         # ... and not much more
    assert c1 < FULL_LIMIT // 4                         # warp 1 left on the abort flag, far before its limit


def test_context_is_usable_after_a_timeout():
    import torch
    import int8_quant_b200 as iq
    from harness import make_inputs
    from int8_quant_b200.runner import SsdProblem, to_device
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cycles = torch.zeros(2, dtype=torch.int64, device="cuda")
    iq.ssd_selftest_bounded_wait(LIMIT, status, cycles)
    torch.cuda.synchronize()
    assert int(status.item()) == 5
    w = WORKLOADS["tiny"]
    pb = SsdProblem(to_device(make_inputs(w)), w.chunk)
    pb.run_bf16()
    torch.cuda.synchronize()
    assert iq.ssd_workspace_status(pb.ws_bf16) == 0
    assert bool(torch.isfinite(pb.y.float()).all())
