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
    def run_bf16(self, stream=None, initial_state=None):
        """initial_state: fp32 [B,H,P,N] device tensor to continue from (None: zero state)."""
        i = self.inp
        if initial_state is None:
            ssd.ssd_scan_fwd_bf16(self.shape, i["x"], i["dt"], i["A"], i["B"], i["C"], i["D"], self.y,
                                  self.final32, self.ws_bf16, stream)
        else:
            ssd.ssd_scan_fwd_bf16_from_state(self.shape, i["x"], i["dt"], i["A"], i["B"], i["C"], i["D"],
                                             initial_state, self.y, self.final32, self.ws_bf16, stream)

    # -- W8A8
    def set_scales(self, s_B, s_C, s_x, s_s, shift: int = 7, storage: int = 0):
        """storage: 0, or SSD_STORAGE_* flags (the notes' storage variant)."""
        dev = self.inp["x"].device
        f = lambda a: torch.as_tensor(np.asarray(a, np.float32) if not torch.is_tensor(a) else a,
                                      dtype=torch.float32).to(dev).contiguous()
        self.scales = {"s_B": f(s_B), "s_C": f(s_C), "s_x": f(s_x), "s_s": f(s_s)}
        self.params = ssd.i8_params(self.scales["s_B"], self.scales["s_C"], self.scales["s_x"],
                                    self.scales["s_s"], shift, storage)

    def set_storage(self, storage: int):
        """Switch the W8A8 calls between the library's layout (0) and the storage variant."""
        self.params.storage = int(storage)

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

    def run_i8(self, stream=None, quantize=True, initial_state=None):
        """initial_state: int8 [B,H,P,N] device tensor of state codes (None: zero state)."""
        if quantize:
            self.quantize(stream)
        i = self.inp
        if initial_state is None:
            ssd.ssd_scan_fwd_i8(self.shape, i["x"], i["dt"], i["A"], self.Bq, self.Cq, i["D"], self.params, self.y,
                                self.final8, self.ws_i8, stream)
        else:
            ssd.ssd_scan_fwd_i8_from_state(self.shape, i["x"], i["dt"], i["A"], self.Bq, self.Cq, i["D"],
                                           self.params, initial_state, self.y, self.final8, self.ws_i8, stream)

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
        if self.params.storage & ssd.SSD_STORAGE_CB_INT8:
            dbg["cb8"] = torch.zeros((b, nc, G, Q, Q), dtype=torch.int8, device=dev)
            dbg["s_cb"] = torch.zeros((b, nc, G), dtype=torch.float64, device=dev)
        self.quantize(stream)
        i = self.inp
        ssd.ssd_scan_fwd_i8_debug(self.shape, i["x"], i["dt"], i["A"], self.Bq, self.Cq, i["D"], self.params,
                                  self.y, self.final8, self.ws_i8, dbg, stream)
        return dbg


def plan_groups(batch: int, seqlen: int, chunk: int, rows_per_group: int = 1, seg_len: int | None = None):
    """The copy groups of StreamedScan: (first row, rows, first token, tokens) in enqueue order, and the
    segment length.  Whole rows (seg_len None or >= seqlen) in groups of rows_per_group, or one row's
    segments of seg_len tokens (a multiple of the chunk), the last one possibly shorter."""
    seg = seqlen if seg_len is None or seg_len >= seqlen else int(seg_len)
    if seg < seqlen:
        assert rows_per_group == 1 and seg % chunk == 0, "segments: one row per group, whole chunks"
    groups = [(r, min(rows_per_group, batch - r), t0, min(seg, seqlen - t0))
              for r in range(0, batch, rows_per_group) for t0 in range(0, max(seqlen, 1), max(seg, 1))]
    return groups, seg


class StreamedScan:
    """A batch held in pinned host memory, scanned in groups with the copies overlapped:
    host->device copies, scans and device->host copies run on three streams, groups taking
    turns in `nslots` device buffers.  A group is `rows_per_group` batch rows (independent problems)
    or, with `seg_len`, one batch row's segment of seg_len tokens (a multiple of the chunk):
    the segments of a row are scanned in order, each from the previous one's final state
    (ssd_scan_fwd_*_from_state, which reproduces one call over the whole row bit for bit
    when the splits fall on chunk boundaries), so that many small groups keep the copy
    engines busy from the first group's copy to the last one's.

    host: pinned CPU tensors x [B,L,H,P] (bf16), dt [B,L,H], B and C [B,L,G,N] (bf16), and
    the outputs y [B,L,H,P] (bf16) and final [B,H,P,N] (fp32 for bf16, int8 for W8A8).
    A and D live on the device.  W8A8 takes the static scales (device tensors).
    """

    def __init__(self, host: dict, A, D, chunk: int, path: str, rows_per_group: int = 1, scales=None,
                 shift: int = 7, device="cuda", seg_len: int | None = None, nslots: int = 2):
        assert path in ("bf16", "w8a8")
        self.h, self.path, self.A, self.D = host, path, A, D
        b, L, H, P = host["x"].shape
        G, N = host["B"].shape[2], host["B"].shape[3]
        self.groups, seg = plan_groups(b, L, chunk, rows_per_group, seg_len)    # (row0, rows, token0, tokens)
        self.rows, self.seg, self.L, self.chunk = rows_per_group, seg, L, chunk
        self.shape = ssd.SsdShape.of(rows_per_group, seg, H, P, G, N, chunk)
        dev = torch.device(device)
        i8 = path == "w8a8"
        self.nslots = max(2, int(nslots))
        self.slots = []
        for _ in range(self.nslots):
            sl = {k: torch.empty((rows_per_group, seg) + tuple(host[k].shape[2:]), dtype=host[k].dtype, device=dev)
                  for k in ("x", "dt", "B", "C", "y")}
            sl["final"] = torch.empty((rows_per_group,) + tuple(host["final"].shape[1:]), dtype=host["final"].dtype,
                                      device=dev)
            if i8:
                sl["Bq"] = torch.empty(sl["B"].shape, dtype=torch.int8, device=dev)
                sl["Cq"] = torch.empty(sl["C"].shape, dtype=torch.int8, device=dev)
            self.slots.append(sl)
        # the state carried between the segments of a row (two buffers: read one, write the other)
        self.carry = [torch.empty_like(self.slots[0]["final"]) for _ in range(2)]
        self.ws = torch.empty(max(ssd.ssd_workspace_bytes(self.shape, i8), 256), dtype=torch.uint8, device=dev)
        if i8:
            self.scales = scales
            self.params = ssd.i8_params(scales["s_B"], scales["s_C"], scales["s_x"], scales["s_s"], shift)
        self.streams = [torch.cuda.Stream(device=dev) for _ in range(3)]      # h2d, compute, d2h
        self.ev = {k: [torch.cuda.Event() for _ in range(self.nslots)] for k in ("in", "done", "out")}
        self.seq = 0                                                           # groups enqueued so far
        self.h2d_bytes = sum(host[k].numel() * host[k].element_size() for k in ("x", "dt", "B", "C"))
        self.d2h_bytes = sum(host[k].numel() * host[k].element_size() for k in ("y", "final"))

    def run(self):
        """Enqueue the whole batch; returns at once (synchronise on `self.streams[2]`)."""
        s_in, s_cmp, s_out = self.streams
        sh = self.shape
        for r0, n, t0, ln in self.groups:
            g = self.seq
            self.seq += 1
            k = g % self.nslots
            sl = self.slots[k]
            first, last = t0 == 0, t0 + ln >= self.L
            shape = sh if (n, ln) == (self.rows, self.seg) else ssd.SsdShape.of(
                n, ln, sh.nheads, sh.headdim, sh.ngroups, sh.dstate, sh.chunk)
            seg_i = t0 // self.seg
            init = None if first else self.carry[(seg_i - 1) % 2][:n]
            fin = sl["final"][:n] if last else self.carry[seg_i % 2][:n]
            with torch.cuda.stream(s_in):
                if g >= self.nslots:
                    s_in.wait_event(self.ev["done"][k])             # slot's inputs consumed by its last scan
                for name in ("x", "dt", "B", "C"):
                    sl[name][:n, :ln].copy_(self.h[name][r0:r0 + n, t0:t0 + ln], non_blocking=True)
                self.ev["in"][k].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(self.ev["in"][k])
                if g >= self.nslots:
                    s_cmp.wait_event(self.ev["out"][k])            # slot's outputs read by its last copy
                x, dt, y = sl["x"][:n, :ln], sl["dt"][:n, :ln], sl["y"][:n, :ln]
                if self.path == "w8a8":
                    Bq, Cq = sl["Bq"][:n, :ln], sl["Cq"][:n, :ln]
                    ssd.ssd_quantize_inputs(shape, sl["B"][:n, :ln], sl["C"][:n, :ln], self.scales["s_B"],
                                            self.scales["s_C"], Bq, Cq, s_cmp)
                    ssd.ssd_scan_fwd_i8_from_state(shape, x, dt, self.A, Bq, Cq, self.D, self.params, init, y, fin,
                                                   self.ws, s_cmp)
                else:
                    ssd.ssd_scan_fwd_bf16_from_state(shape, x, dt, self.A, sl["B"][:n, :ln], sl["C"][:n, :ln],
                                                     self.D, init, y, fin, self.ws, s_cmp)
                self.ev["done"][k].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(self.ev["done"][k])
                self.h["y"][r0:r0 + n, t0:t0 + ln].copy_(sl["y"][:n, :ln], non_blocking=True)
                if last:
                    self.h["final"][r0:r0 + n].copy_(sl["final"][:n], non_blocking=True)
                self.ev["out"][k].record(s_out)


class Decoder:
    """One-token steps on a persistent state (serving after a scan).

    state: the scan's final state to continue from — fp32 [B,H,P,N] (bf16 path) or
    int8 codes [B,H,P,N] (W8A8, real value code * s_s) — updated in place by each step.
    A, D: device fp32 [H].  W8A8 takes the static scales (device tensors s_B, s_C, s_x, s_s).
    Each step takes the token's x [B,H,P] (bf16), dt [B,H], B and C [B,G,N] (bf16) and
    returns y [B,H,P] (bf16, a buffer reused by the next step).
    """

    def __init__(self, state, A, D, path: str, scales: dict | None = None, shift: int = 7):
        assert path in ("bf16", "w8a8")
        self.state, self.A, self.D, self.path = state, A, D, path
        b, H, P, N = state.shape
        self.dims = (b, H, P, N)
        self.y = torch.empty((b, H, P), dtype=torch.bfloat16, device=state.device)
        self.params = None
        if path == "w8a8":
            self.scales = scales
            self.params = ssd.i8_params(scales["s_B"], scales["s_C"], scales["s_x"], scales["s_s"], shift)

    def _shape(self, B):
        b, H, P, N = self.dims
        return ssd.SsdShape.of(b, 1, H, P, B.shape[-2], N, 256)

    def step(self, x, dt, B, C, stream=None):
        shape = self._shape(B)
        if self.path == "bf16":
            ssd.ssd_decode_step_bf16(shape, x, dt, self.A, B, C, self.D, self.state, self.y, stream)
            return self.y
        ssd.ssd_decode_step_i8(shape, x, dt, self.A, B, C, self.D, self.params, self.state, self.y, stream)
        return self.y
