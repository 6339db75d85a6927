"""Device buffers for one SSD problem and the call sequence of each path.

torch allocates memory and provides the stream; every step of the scan is a call
into libssd.so.
"""
from __future__ import annotations

import numpy as np
import torch

from . import ssd


def to_device(inputs: dict, device="cuda") -> dict:
    """Host arrays (bf16 as uint16 bits) → device tensors with the library's dtypes."""
    out = {}
    for k, v in inputs.items():
        if isinstance(v, np.ndarray):
            if v.dtype == np.uint16:
                t = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16)
            else:
                t = torch.from_numpy(np.ascontiguousarray(v))
            out[k] = t.to(device, non_blocking=False).contiguous()
        else:
            out[k] = v
    return out


class SsdProblem:
    """Inputs on the device plus every buffer the two paths write."""

    def __init__(self, dev_inputs: dict, chunk: int, with_i8: bool = True, with_bf16: bool = True):
        self.inp = dev_inputs
        x, B = dev_inputs["x"], dev_inputs["B"]
        self.shape = ssd.shape_of(x, B, chunk)
        b, L, H, P = x.shape
        G, N = B.shape[2], B.shape[3]
        dev = x.device
        self.dims = (b, L, H, P, G, N, chunk)
        self.y = torch.empty_like(x)
        if with_bf16:
            self.final32 = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
            self.ws_bf16 = torch.empty(max(ssd.ssd_workspace_bytes(self.shape, False), 256), dtype=torch.uint8,
                                       device=dev)
        if with_i8:
            self.Bq = torch.empty(B.shape, dtype=torch.int8, device=dev)
            self.Cq = torch.empty(B.shape, dtype=torch.int8, device=dev)
            self.final8 = torch.empty((b, H, P, N), dtype=torch.int8, device=dev)
            self.ws_i8 = torch.empty(max(ssd.ssd_workspace_bytes(self.shape, True), 256), dtype=torch.uint8,
                                     device=dev)
        self.scales = None
        self.params = None

    # -- bf16
    def run_bf16(self, stream=None):
        i = self.inp
        ssd.ssd_scan_fwd_bf16(self.shape, i["x"], i["dt"], i["A"], i["B"], i["C"], i["D"], self.y,
                              self.final32, self.ws_bf16, stream)

    # -- W8A8
    def set_scales(self, s_B, s_C, s_x, s_s, shift: int = 7):
        dev = self.inp["x"].device
        f = lambda a: torch.as_tensor(np.asarray(a, np.float32) if not torch.is_tensor(a) else a,
                                      dtype=torch.float32).to(dev).contiguous()
        self.scales = {"s_B": f(s_B), "s_C": f(s_C), "s_x": f(s_x), "s_s": f(s_s)}
        self.params = ssd.i8_params(self.scales["s_B"], self.scales["s_C"], self.scales["s_x"],
                                    self.scales["s_s"], shift)

    def calibrate(self, prefix: int = 512, shift: int = 7, stream=None):
        b, L, H, P, G, N, Q = self.dims
        dev = self.inp["x"].device
        out = {k: torch.empty(n, dtype=torch.float32, device=dev)
               for k, n in (("s_B", G), ("s_C", G), ("s_x", H * P), ("s_s", H * P))}
        ws = torch.empty(max(ssd.ssd_calibrate_workspace_bytes(self.shape, prefix), 256), dtype=torch.uint8,
                         device=dev)
        i = self.inp
        ssd.ssd_calibrate_i8(self.shape, prefix, i["x"], i["dt"], i["A"], i["B"], i["C"], out["s_B"],
                             out["s_C"], out["s_x"], out["s_s"], ws, stream)
        self.set_scales(out["s_B"], out["s_C"], out["s_x"], out["s_s"], shift)
        return out

    def quantize(self, stream=None):
        i = self.inp
        ssd.ssd_quantize_inputs(self.shape, i["B"], i["C"], self.scales["s_B"], self.scales["s_C"], self.Bq,
                                self.Cq, stream)

    def run_i8(self, stream=None, quantize=True):
        if quantize:
            self.quantize(stream)
        i = self.inp
        ssd.ssd_scan_fwd_i8(self.shape, i["x"], i["dt"], i["A"], self.Bq, self.Cq, i["D"], self.params, self.y,
                            self.final8, self.ws_i8, stream)

    def run_i8_debug(self, stream=None):
        b, L, H, P, G, N, Q = self.dims
        nc = (L + Q - 1) // Q
        Lp = nc * Q
        dev = self.inp["x"].device
        dbg = {
            "Acs": torch.zeros((b, H, nc, Q), dtype=torch.float32, device=dev),
            "dq": torch.zeros((b, H, nc), dtype=torch.int32, device=dev),
            "Xq": torch.zeros((b, Lp, H, P), dtype=torch.int8, device=dev),
            "acc_state": torch.zeros((b, nc, H, P, N), dtype=torch.int32, device=dev),
            "S8": torch.zeros((b, nc, H, P, N), dtype=torch.int8, device=dev),
            "H8": torch.zeros((b, nc, H, P, N), dtype=torch.int8, device=dev),
            "cb": torch.zeros((b, nc, G, Q, Q), dtype=torch.int32, device=dev),
            "acc_scan1": torch.zeros((b, Lp, H, P), dtype=torch.int32, device=dev),
        }
        self.quantize(stream)
        i = self.inp
        ssd.ssd_scan_fwd_i8_debug(self.shape, i["x"], i["dt"], i["A"], self.Bq, self.Cq, i["D"], self.params,
                                  self.y, self.final8, self.ws_i8, dbg, stream)
        return dbg
