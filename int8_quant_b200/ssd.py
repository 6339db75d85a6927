"""Python binding of libssd.so: argument marshalling only.

Each function has the name of the C entry point it calls and takes torch tensors
that already live on the GPU (torch is used for device memory and streams only);
every step of the scan runs in the library's CUDA kernels.  A missing library is
an ImportError, never a fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libssd.so")

SSD_OK = 0
STATUS_NAMES = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED", 3: "SSD_ERR_WORKSPACE",
                4: "SSD_ERR_CUDA", 5: "SSD_ERR_TIMEOUT"}

# Names declared in include/ssd.h (checked against the header by the tests).
EXPORTS = ("ssd_status_string", "ssd_last_cuda_error", "ssd_workspace_bytes", "ssd_quantize_inputs", "ssd_scan_fwd_bf16",
           "ssd_scan_fwd_i8", "ssd_scan_fwd_i8_debug", "ssd_calibrate_workspace_bytes",
           "ssd_calibrate_i8", "ssd_workspace_status", "ssd_profile_enable", "ssd_profile_read",
           "ssd_profile_reset", "ssd_scan_fwd_bf16_static", "ssd_selftest_bounded_wait",
           "ssd_scan_fwd_bf16_from_state", "ssd_scan_fwd_i8_from_state", "ssd_decode_step_bf16", "ssd_profile_filter",
           "ssd_decode_step_i8", "ssd_out_proj_workspace_bytes", "ssd_out_proj_i8", "ssd_out_proj_status",
           "ssd_static_scratch_status")

# Size of the library's fixed device scratch used by ssd_scan_fwd_bf16_static.
STATIC_SCRATCH_BYTES = 32 << 20


class SsdShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("nheads", ctypes.c_int),
                ("headdim", ctypes.c_int), ("ngroups", ctypes.c_int), ("dstate", ctypes.c_int),
                ("chunk", ctypes.c_int)]

    @classmethod
    def of(cls, batch, seqlen, nheads, headdim, ngroups, dstate, chunk):
        return cls(int(batch), int(seqlen), int(nheads), int(headdim), int(ngroups), int(dstate), int(chunk))

    def __repr__(self):
        return "SsdShape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class SsdI8Params(ctypes.Structure):
    _fields_ = [("s_B", ctypes.c_void_p), ("s_C", ctypes.c_void_p), ("s_x", ctypes.c_void_p),
                ("s_s", ctypes.c_void_p), ("decay_shift", ctypes.c_int), ("storage", ctypes.c_int)]


SSD_STORAGE_ACS_FP16 = 1
SSD_STORAGE_CB_INT8 = 2


class SsdI8Debug(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Acs", "dq", "Xq", "acc_state", "S8", "H8", "cb", "acc_scan1",
                                               "cb8", "s_cb")]


class SsdError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = int(status)
        msg = f"{fn}: {_lib().ssd_status_string(status).decode()}"
        if status == 4:  # SSD_ERR_CUDA
            msg += f" ({_lib().ssd_last_cuda_error().decode()})"
        super().__init__(msg)


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libssd.so is not built ({LIB_PATH}); run int8_quant_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sp = ctypes.POINTER(SsdShape)
        lib.ssd_status_string.restype = ctypes.c_char_p
        lib.ssd_status_string.argtypes = [I]
        lib.ssd_last_cuda_error.restype = ctypes.c_char_p
        lib.ssd_last_cuda_error.argtypes = []
        lib.ssd_workspace_bytes.restype = S
        lib.ssd_workspace_bytes.argtypes = [sp, I]
        lib.ssd_calibrate_workspace_bytes.restype = S
        lib.ssd_calibrate_workspace_bytes.argtypes = [sp, I]
        lib.ssd_quantize_inputs.restype = I
        lib.ssd_quantize_inputs.argtypes = [sp, P, P, P, P, P, P, P]
        lib.ssd_scan_fwd_bf16.restype = I
        lib.ssd_scan_fwd_bf16.argtypes = [sp, P, P, P, P, P, P, P, P, P, S, P]
        lib.ssd_scan_fwd_bf16_from_state.restype = I
        lib.ssd_scan_fwd_bf16_from_state.argtypes = [sp, P, P, P, P, P, P, P, P, P, P, S, P]
        lib.ssd_scan_fwd_i8_from_state.restype = I
        lib.ssd_scan_fwd_i8_from_state.argtypes = [sp, P, P, P, P, P, P, ctypes.POINTER(SsdI8Params), P, P, P, P,
                                                   S, P]
        lib.ssd_decode_step_bf16.restype = I
        lib.ssd_decode_step_bf16.argtypes = [sp, P, P, P, P, P, P, P, P, P]
        lib.ssd_decode_step_i8.restype = I
        lib.ssd_decode_step_i8.argtypes = [sp, P, P, P, P, P, P, ctypes.POINTER(SsdI8Params), P, P, P]
        lib.ssd_out_proj_workspace_bytes.restype = S
        lib.ssd_out_proj_workspace_bytes.argtypes = [I, I]
        lib.ssd_out_proj_i8.restype = I
        lib.ssd_out_proj_i8.argtypes = [I, I, I, P, ctypes.c_float, P, P, P, P, P, P, S, P]
        lib.ssd_out_proj_status.restype = I
        lib.ssd_out_proj_status.argtypes = [P, I, I, P]
        lib.ssd_scan_fwd_bf16_static.restype = I
        lib.ssd_scan_fwd_bf16_static.argtypes = [sp, P, P, P, P, P, P, P, P, P]
        lib.ssd_static_scratch_status.restype = I
        lib.ssd_static_scratch_status.argtypes = [P]
        lib.ssd_scan_fwd_i8.restype = I
        lib.ssd_scan_fwd_i8.argtypes = [sp, P, P, P, P, P, P, ctypes.POINTER(SsdI8Params), P, P, P, S, P]
        lib.ssd_scan_fwd_i8_debug.restype = I
        lib.ssd_scan_fwd_i8_debug.argtypes = [sp, P, P, P, P, P, P, ctypes.POINTER(SsdI8Params), P, P, P, S,
                                              ctypes.POINTER(SsdI8Debug), P]
        lib.ssd_calibrate_i8.restype = I
        lib.ssd_calibrate_i8.argtypes = [sp, I, P, P, P, P, P, P, P, P, P, P, S, P]
        lib.ssd_workspace_status.restype = I
        lib.ssd_workspace_status.argtypes = [P, P]
        lib.ssd_selftest_bounded_wait.restype = I
        lib.ssd_selftest_bounded_wait.argtypes = [ctypes.c_longlong, P, P, P]
        lib.ssd_profile_enable.restype = I
        lib.ssd_profile_enable.argtypes = [I]
        lib.ssd_profile_reset.restype = I
        lib.ssd_profile_reset.argtypes = []
        lib.ssd_profile_filter.restype = I
        lib.ssd_profile_filter.argtypes = [ctypes.c_char_p]
        lib.ssd_profile_read.restype = I
        lib.ssd_profile_read.argtypes = [I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                         ctypes.POINTER(ctypes.c_longlong), ctypes.POINTER(ctypes.c_int)]
        _LIB = lib
    return _LIB


def library():
    """The loaded ctypes library (raises ImportError if it is not built)."""
    return _lib()


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn, st):
    if st != SSD_OK:
        raise SsdError(fn, st)


def shape_of(x, B, chunk) -> SsdShape:
    """Shape from x [B,L,H,P] and B [B,L,G,N]."""
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    return SsdShape.of(b, L, H, P, G, N, chunk)


def ssd_workspace_bytes(shape: SsdShape, is_i8: bool) -> int:
    return int(_lib().ssd_workspace_bytes(ctypes.byref(shape), int(bool(is_i8))))


def ssd_calibrate_workspace_bytes(shape: SsdShape, prefix: int) -> int:
    return int(_lib().ssd_calibrate_workspace_bytes(ctypes.byref(shape), int(prefix)))


def ssd_quantize_inputs(shape, B, C, s_B, s_C, Bq, Cq, stream=None):
    _check("ssd_quantize_inputs", _lib().ssd_quantize_inputs(
        ctypes.byref(shape), _ptr(B), _ptr(C), _ptr(s_B), _ptr(s_C), _ptr(Bq), _ptr(Cq), _stream(stream)))


def ssd_scan_fwd_bf16(shape, x, dt, A, B, C, D, y, final_state, workspace, stream=None):
    _check("ssd_scan_fwd_bf16", _lib().ssd_scan_fwd_bf16(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
        _ptr(final_state), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def ssd_scan_fwd_bf16_from_state(shape, x, dt, A, B, C, D, initial_state, y, final_state, workspace, stream=None):
    _check("ssd_scan_fwd_bf16_from_state", _lib().ssd_scan_fwd_bf16_from_state(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(initial_state), _ptr(y),
        _ptr(final_state), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def ssd_scan_fwd_i8_from_state(shape, x, dt, A, Bq, Cq, D, params: SsdI8Params, initial_state, y, final_state,
                               workspace, stream=None):
    _check("ssd_scan_fwd_i8_from_state", _lib().ssd_scan_fwd_i8_from_state(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bq), _ptr(Cq), _ptr(D), ctypes.byref(params),
        _ptr(initial_state), _ptr(y), _ptr(final_state), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def ssd_decode_step_bf16(shape, x, dt, A, B, C, D, state, y, stream=None):
    _check("ssd_decode_step_bf16", _lib().ssd_decode_step_bf16(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(state), _ptr(y),
        _stream(stream)))


def ssd_decode_step_i8(shape, x, dt, A, B, C, D, params: SsdI8Params, state, y, stream=None):
    _check("ssd_decode_step_i8", _lib().ssd_decode_step_i8(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), ctypes.byref(params),
        _ptr(state), _ptr(y), _stream(stream)))


def ssd_out_proj_workspace_bytes(tokens: int, d_inner: int) -> int:
    return int(_lib().ssd_out_proj_workspace_bytes(int(tokens), int(d_inner)))


def ssd_out_proj_i8(y, s_a: float, Wq, s_w, corr, out, workspace, acc_debug=None, stream=None):
    """y [T, K] bf16; Wq [D, K] int8; s_w, corr [D] fp32 (corr may be None); out [T, D] bf16."""
    T, K = y.shape
    D = Wq.shape[0]
    _check("ssd_out_proj_i8", _lib().ssd_out_proj_i8(
        T, K, D, _ptr(y), float(s_a), _ptr(Wq), _ptr(s_w), _ptr(corr), _ptr(out), _ptr(acc_debug), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def ssd_out_proj_status(workspace, tokens: int, d_inner: int, stream=None) -> int:
    return int(_lib().ssd_out_proj_status(_ptr(workspace), int(tokens), int(d_inner), _stream(stream)))


def ssd_scan_fwd_bf16_static(shape, x, dt, A, B, C, D, y, final_state, stream=None):
    """ssd_scan_fwd_bf16 without a workspace argument: the library's fixed 32 MiB device
    scratch is used instead, for callers that cannot allocate device memory.  Calls
    share that scratch, so calls whose GPU work overlaps must be serialised."""
    _check("ssd_scan_fwd_bf16_static", _lib().ssd_scan_fwd_bf16_static(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y), _ptr(final_state),
        _stream(stream)))


def ssd_static_scratch_status(stream=None) -> int:
    """Status word of the fixed scratch after the last ssd_scan_fwd_bf16_static call
    (synchronises the stream, returns 0 or the recorded error, clears it)."""
    return int(_lib().ssd_static_scratch_status(_stream(stream)))


def i8_params(s_B, s_C, s_x, s_s, decay_shift=7, storage=0) -> SsdI8Params:
    return SsdI8Params(s_B.data_ptr(), s_C.data_ptr(), s_x.data_ptr(), s_s.data_ptr(), int(decay_shift),
                       int(storage))


def ssd_scan_fwd_i8(shape, x, dt, A, Bq, Cq, D, params: SsdI8Params, y, final_state, workspace, stream=None):
    _check("ssd_scan_fwd_i8", _lib().ssd_scan_fwd_i8(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bq), _ptr(Cq), _ptr(D), ctypes.byref(params),
        _ptr(y), _ptr(final_state), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def ssd_scan_fwd_i8_debug(shape, x, dt, A, Bq, Cq, D, params: SsdI8Params, y, final_state, workspace,
                          dbg: dict, stream=None):
    d = SsdI8Debug(*[(dbg[n].data_ptr() if dbg.get(n) is not None else None) for n, _ in SsdI8Debug._fields_])
    _check("ssd_scan_fwd_i8_debug", _lib().ssd_scan_fwd_i8_debug(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(Bq), _ptr(Cq), _ptr(D), ctypes.byref(params),
        _ptr(y), _ptr(final_state), _ptr(workspace), workspace.numel() * workspace.element_size(),
        ctypes.byref(d), _stream(stream)))


def ssd_calibrate_i8(shape, prefix, x, dt, A, B, C, s_B, s_C, s_x, s_s, workspace, stream=None):
    _check("ssd_calibrate_i8", _lib().ssd_calibrate_i8(
        ctypes.byref(shape), int(prefix), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(s_B), _ptr(s_C),
        _ptr(s_x), _ptr(s_s), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def ssd_workspace_status(workspace, stream=None) -> int:
    return int(_lib().ssd_workspace_status(_ptr(workspace), _stream(stream)))


def ssd_selftest_bounded_wait(limit_cycles: int, status, cycles, stream=None) -> None:
    """status: int32 CUDA tensor of 1 element; cycles: int64 CUDA tensor of 2 elements."""
    _check("ssd_selftest_bounded_wait", _lib().ssd_selftest_bounded_wait(
        int(limit_cycles), _ptr(status), _ptr(cycles), _stream(stream)))


def ssd_profile_enable(enable: bool) -> None:
    _check("ssd_profile_enable", _lib().ssd_profile_enable(int(bool(enable))))


def ssd_profile_reset() -> None:
    _check("ssd_profile_reset", _lib().ssd_profile_reset())


def ssd_profile_filter(name: str | None) -> None:
    """Time only the kernel `name` while profiling is enabled (None: every kernel)."""
    _check("ssd_profile_filter", _lib().ssd_profile_filter(name.encode() if name else None))


def ssd_profile_read() -> dict:
    """{kernel name: (total ms, launches)} accumulated since the last reset."""
    lib = _lib()
    cap = 32
    names = (ctypes.c_char_p * cap)()
    ms = (ctypes.c_double * cap)()
    calls = (ctypes.c_longlong * cap)()
    n = ctypes.c_int(0)
    _check("ssd_profile_read", lib.ssd_profile_read(cap, names, ms, calls, ctypes.byref(n)))
    return {names[i].decode(): (ms[i], int(calls[i])) for i in range(min(n.value, cap))}
