"""The C-ABI library loads and exports what include/ssd.h declares; host-side validation (no GPU)."""
import ctypes
import os
import re

import pytest

import int8_quant_b200 as iq
from int8_quant_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "ssd.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_the_binding_names():
    assert sorted(ssd.EXPORTS) == _declared()


def test_library_exports_every_declared_symbol():
    lib = iq.library()
    for name in _declared():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings():
    lib = iq.library()
    for code, name in ssd.STATUS_NAMES.items():
        assert lib.ssd_status_string(code).decode().startswith(name)


@pytest.mark.parametrize("shape,ok", [
    ((8, 8192, 80, 64, 1, 128, 256), True),
    ((1, 256, 4, 16, 1, 16, 64), True),
    ((1, 100, 4, 64, 2, 128, 128), True),
    ((0, 0, 4, 64, 1, 128, 256), True),
    ((1, 256, 4, 32, 1, 16, 64), False),     # unsupported (P, N)
    ((1, 256, 4, 64, 1, 128, 96), False),    # unsupported chunk
    ((1, 256, 6, 64, 4, 128, 256), False),   # H % G != 0
    ((-1, 256, 4, 64, 1, 128, 256), False),
])
def test_workspace_bytes_validates_shapes(shape, ok):
    s = iq.SsdShape.of(*shape)
    assert (iq.ssd_workspace_bytes(s, False) > 0) == ok
    assert (iq.ssd_workspace_bytes(s, True) > 0) == ok


def test_workspace_grows_with_the_problem_and_i8_is_smaller():
    a = iq.ssd_workspace_bytes(iq.SsdShape.of(1, 1024, 8, 64, 1, 128, 256), False)
    b = iq.ssd_workspace_bytes(iq.SsdShape.of(2, 1024, 8, 64, 1, 128, 256), False)
    c = iq.ssd_workspace_bytes(iq.SsdShape.of(2, 1024, 8, 64, 1, 128, 256), True)
    assert b > a and c < b


def _fake(n=0x10000):
    return ctypes.c_void_p(n)        # aligned, never dereferenced: every call below fails validation


def test_invalid_arguments_fail_before_any_launch():
    lib = iq.library()
    s = iq.SsdShape.of(1, 256, 4, 64, 1, 128, 256)
    f = _fake()
    ws = iq.ssd_workspace_bytes(s, False)
    # null x
    st = lib.ssd_scan_fwd_bf16(ctypes.byref(s), None, f, f, f, f, f, f, f, f, ws, None)
    assert st == 1
    # misaligned y
    st = lib.ssd_scan_fwd_bf16(ctypes.byref(s), f, f, f, f, f, f, _fake(0x10002), f, f, ws, None)
    assert st == 1
    # workspace too small / missing
    assert lib.ssd_scan_fwd_bf16(ctypes.byref(s), f, f, f, f, f, f, f, f, f, ws - 1, None) == 3
    assert lib.ssd_scan_fwd_bf16(ctypes.byref(s), f, f, f, f, f, f, f, f, None, ws, None) == 3
    # unsupported shape
    s2 = iq.SsdShape.of(1, 256, 4, 32, 1, 16, 64)
    assert lib.ssd_scan_fwd_bf16(ctypes.byref(s2), f, f, f, f, f, f, f, f, f, 1 << 30, None) == 2
    # W8A8: missing params, bad shift
    wsi = iq.ssd_workspace_bytes(s, True)
    assert lib.ssd_scan_fwd_i8(ctypes.byref(s), f, f, f, f, f, f, None, f, f, f, wsi, None) == 1
    p = iq.SsdI8Params(0x10000, 0x10000, 0x10000, 0x10000, 0)
    assert lib.ssd_scan_fwd_i8(ctypes.byref(s), f, f, f, f, f, f, ctypes.byref(p), f, f, f, wsi, None) == 1
    p.decay_shift = 15
    assert lib.ssd_scan_fwd_i8(ctypes.byref(s), f, f, f, f, f, f, ctypes.byref(p), f, f, f, wsi, None) == 1
    # the storage variant: unknown flags; a chunk other than 256 or the (16, 16) shape is unsupported
    p.decay_shift = 7
    p.storage = 4
    assert lib.ssd_scan_fwd_i8(ctypes.byref(s), f, f, f, f, f, f, ctypes.byref(p), f, f, f, wsi, None) == 1
    p.storage = iq.SSD_STORAGE_ACS_FP16 | iq.SSD_STORAGE_CB_INT8
    s128 = iq.SsdShape.of(1, 256, 4, 64, 1, 128, 128)
    assert lib.ssd_scan_fwd_i8(ctypes.byref(s128), f, f, f, f, f, f, ctypes.byref(p), f, f, f, 1 << 30, None) == 2
    s16 = iq.SsdShape.of(1, 256, 4, 16, 1, 16, 256)
    assert lib.ssd_scan_fwd_i8(ctypes.byref(s16), f, f, f, f, f, f, ctypes.byref(p), f, f, f, 1 << 30, None) == 2
    # quantize: null outputs
    assert lib.ssd_quantize_inputs(ctypes.byref(s), f, f, f, f, None, f, None) == 1
    # calibration: workspace too small
    cw = iq.ssd_calibrate_workspace_bytes(s, 512)
    assert cw > 0
    assert lib.ssd_calibrate_i8(ctypes.byref(s), 512, f, f, f, f, f, f, f, f, f, f, cw - 1, None) == 3
    assert lib.ssd_calibrate_i8(ctypes.byref(s), -1, f, f, f, f, f, f, f, f, f, f, cw, None) == 1


def test_null_shape_is_rejected():
    lib = iq.library()
    assert lib.ssd_workspace_bytes(None, 0) == 0
    f = _fake()
    assert lib.ssd_scan_fwd_bf16(None, f, f, f, f, f, f, f, f, f, 1 << 20, None) == 1


def test_bounded_wait_selftest_validates_before_any_launch():
    lib = iq.library()
    f = _fake()
    assert lib.ssd_selftest_bounded_wait(0, f, f, None) == 1            # limit out of range
    assert lib.ssd_selftest_bounded_wait(-5, f, f, None) == 1
    assert lib.ssd_selftest_bounded_wait(1 << 40, f, f, None) == 1      # beyond the kernels' own limit
    assert lib.ssd_selftest_bounded_wait(1000, None, f, None) == 1      # null status
    assert lib.ssd_selftest_bounded_wait(1000, f, None, None) == 1      # null cycles


def test_decode_step_validates_before_any_launch():
    lib = iq.library()
    f = _fake()
    one = iq.SsdShape.of(2, 1, 4, 64, 1, 128, 256)
    two = iq.SsdShape.of(2, 2, 4, 64, 1, 128, 256)                    # seqlen must be 1
    bad = iq.SsdShape.of(2, 1, 4, 32, 1, 64, 256)                     # unsupported (P, N)
    assert lib.ssd_decode_step_bf16(ctypes.byref(two), f, f, f, f, f, f, f, f, None) == 1
    assert lib.ssd_decode_step_bf16(ctypes.byref(bad), f, f, f, f, f, f, f, f, None) == 2
    assert lib.ssd_decode_step_bf16(ctypes.byref(one), f, f, f, f, f, f, None, f, None) == 1     # null state
    assert lib.ssd_decode_step_bf16(ctypes.byref(one), f, f, f, f, f, f, f, _fake(0x10004), None) == 1
    p = iq.SsdI8Params(0x10000, 0x10000, 0x10000, 0x10000, 7)
    assert lib.ssd_decode_step_i8(ctypes.byref(one), f, f, f, f, f, f, None, f, f, None) == 1    # no params
    p.decay_shift = 0
    assert lib.ssd_decode_step_i8(ctypes.byref(one), f, f, f, f, f, f, ctypes.byref(p), f, f, None) == 1
    assert lib.ssd_decode_step_bf16(None, f, f, f, f, f, f, f, f, None) == 1


def test_out_proj_validates_before_any_launch():
    lib = iq.library()
    f = _fake()
    ws = lib.ssd_out_proj_workspace_bytes(256, 512)
    assert ws >= 256 * 512
    assert lib.ssd_out_proj_workspace_bytes(-1, 512) == 0
    # unsupported sizes
    assert lib.ssd_out_proj_i8(256, 500, 512, f, 0.1, f, f, None, f, None, f, ws, None) == 2
    assert lib.ssd_out_proj_i8(256, 512, 500, f, 0.1, f, f, None, f, None, f, ws, None) == 2
    assert lib.ssd_out_proj_i8(200, 512, 512, f, 0.1, f, f, None, f, None, f, ws, None) == 2
    # bad scale, null weights, small workspace
    assert lib.ssd_out_proj_i8(256, 512, 512, f, 0.0, f, f, None, f, None, f, ws, None) == 1
    assert lib.ssd_out_proj_i8(256, 512, 512, f, 0.1, None, f, None, f, None, f, ws, None) == 1
    assert lib.ssd_out_proj_i8(256, 512, 512, f, 0.1, f, f, None, f, None, f, ws - 1, None) == 3
