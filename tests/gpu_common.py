"""Helpers shared by the GPU parity tests: oracle runs on host copies of the same inputs."""
from __future__ import annotations

import numpy as np

from harness import as_float, make_chain, prefix_inputs, Workload
from oracle import ssd_fp64 as F
from oracle import ssd_w8a8 as W

F32 = np.float32
TOL_BF16 = 5e-3        # relative L2 of y and the final state against fp64
TOL_I8_Y = 5e-2        # relative L2 of the dequantised W8A8 y against fp64


def poison(torch, pb) -> None:
    """Fill an SsdProblem's outputs with values no kernel produces: NaN bit patterns in y and
    the fp32 state, code -128 in the INT8 state."""
    pb.y.view(torch.int16).fill_(-1)
    if getattr(pb, "final32", None) is not None:
        pb.final32.fill_(float("nan"))
    if getattr(pb, "final8", None) is not None:
        pb.final8.fill_(-128)


def bf16_to_np(t) -> np.ndarray:
    """float64 values of a bf16 torch tensor."""
    import torch
    u = t.detach().to("cpu").view(torch.int16).numpy().view(np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def host(t) -> np.ndarray:
    return t.detach().to("cpu").numpy()


def oracle_fp64(inp: dict):
    """fp64 sequential recurrence on the exact values the GPU received."""
    return F.ssd_sequential(as_float(inp["x"]), inp["dt"], inp["A"], as_float(inp["B"]), as_float(inp["C"]),
                            inp["D"])


def oracle_scales(inp: dict, chunk: int, prefix: int = 512) -> dict:
    return F.calibrate(as_float(inp["x"]), inp["dt"], inp["A"], as_float(inp["B"]), as_float(inp["C"]), chunk,
                       prefix)


def oracle_i8(inp: dict, sc: dict, chunk: int, shift: int = 7, **variant) -> dict:
    """The integer W8A8 oracle on the workload's inputs; `variant`: acs_fp16 / cb_int8 switches."""
    Bv, Cv = as_float(inp["B"]).astype(F32), as_float(inp["C"]).astype(F32)
    Bq, Cq = W.quantize_inputs(Bv, Cv, sc["s_B"], sc["s_C"])
    r = W.ssd_w8a8(as_float(inp["x"]).astype(F32), inp["dt"], inp["A"], Bq, Cq, inp["D"], sc["s_B"], sc["s_C"],
                   sc["s_x"], sc["s_s"], chunk, shift, **variant)
    r["Bq"], r["Cq"] = Bq, Cq
    return r


def chain_oracle(w: Workload, b: int, h: int):
    """fp64 sequential result of one (batch, head) chain at full length: (y [L,P], final [P,N], inputs)."""
    ch = make_chain(w, b, h)
    x = as_float(ch["x"])[None, :, None, :]
    dt = ch["dt"][None, :, None].astype(np.float64)
    Bv = as_float(ch["B"])[None, :, None, :]
    Cv = as_float(ch["C"])[None, :, None, :]
    y, fin = F.ssd_sequential(x, dt, np.array([ch["A"]], np.float64), Bv, Cv, np.array([ch["D"]], np.float64))
    return y[0, :, 0, :], fin[0, 0], ch


def chain_oracle_i8(w: Workload, b: int, h: int, sc: dict, shift: int = 7) -> dict:
    """Integer W8A8 pipeline of one chain with the problem's scales."""
    ch = make_chain(w, b, h)
    P = w.headdim
    g = ch["g"]
    x = as_float(ch["x"]).astype(F32)[None, :, None, :]
    dt = ch["dt"][None, :, None]
    Bv = as_float(ch["B"]).astype(F32)[None, :, None, :]
    Cv = as_float(ch["C"]).astype(F32)[None, :, None, :]
    sB, sC = sc["s_B"][g:g + 1], sc["s_C"][g:g + 1]
    sx, ss = sc["s_x"][h * P:(h + 1) * P], sc["s_s"][h * P:(h + 1) * P]
    Bq, Cq = W.quantize_inputs(Bv, Cv, sB, sC)
    r = W.ssd_w8a8(x, dt, np.float32([ch["A"]]), Bq, Cq, np.float32([ch["D"]]), sB, sC, sx, ss, w.chunk, shift)
    r["Bq"], r["Cq"], r["g"] = Bq, Cq, g
    return r


def full_size_scales(w: Workload) -> dict:
    """Oracle calibration over the first min(512, L) tokens of every row, regenerated on the host."""
    pre = prefix_inputs(w)
    return oracle_scales(pre, w.chunk, w.calib_prefix)
