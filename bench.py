#!/usr/bin/env python
"""Throughput of the SSD chunked scan forward on B200: tokens/s and roofline fraction.

One step = one pass of the whole path over one batch of synthetic input resident in
HBM: for the W8A8 path ssd_quantize_inputs + ssd_scan_fwd_i8 (ChunkCumsum,
ChunkState, StatePassing, ChunkBMM/ChunkScan), for the bf16 path ssd_scan_fwd_bf16.
The default workload is the Mamba-2 2.7B layer shape (B=8, L=8192, H=80, P=64,
N=128, G=1, chunk 256); its inputs (1.4 GB) are larger than L2, so no flush is
needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own copy of the workload (independent problems:
weak scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import multiprocessing as mp
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from harness import WORKLOADS, make_inputs, make_chain, as_float  # noqa: E402

METRIC = "SSD scan fwd tokens/s (B·L/s) and % of roofline, 2.7B layer shape, bf16 & W8A8"
DATASHEET_HBM_GBS = 8000.0          # the roofline definition's HBM figure (8 TB/s)
FALLBACK_HBM_GBS = 6650.0           # used only when MEASURED_PEAKS.json is absent


# ---------------------------------------------------------------- byte counts
def path_bytes(w, path: str) -> int:
    """Compulsory bytes of one step: every input read once, every output written once.
    Per token x 2HP + y 2HP + dt 4H, and B, C at 4GN (bf16) on the bf16 path, 2GN (their
    INT8 codes) on the W8A8 path; plus the final state, fp32 or INT8."""
    T, H, P, N, G = w.tokens, w.nheads, w.headdim, w.dstate, w.ngroups
    bc = 2 if path == "w8a8" else 4
    per_tok = 2 * H * P + 2 * H * P + bc * G * N + 4 * H
    fin = w.batch * H * P * N * (4 if path == "bf16" else 1)
    return T * per_tok + fin


def config_of(w, path: str, world: int) -> dict:
    """The workload as both arms print it."""
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads,
            "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups, "chunk": w.chunk,
            "path": path, "step": ("ssd_quantize_inputs + ssd_scan_fwd_i8" if path == "w8a8"
                                   else "ssd_scan_fwd_bf16"),
            "l2": f"inputs larger than L2 ({path_bytes(w, path) / 1e9:.2f} GB per step), no flush",
            "parallelism": f"replicas x{world}"}


def kernel_bytes(w, path: str, kernel: str) -> int:
    """Algorithmic bytes of one launch of `kernel` (its own inputs read once, outputs written once)."""
    T, H, P, N, G, Q = w.tokens, w.nheads, w.headdim, w.dstate, w.ngroups, w.chunk
    nc = w.nchunks
    chains = w.batch * H
    states = w.batch * nc * H * P * N
    tc_shape = (P, N) == (64, 128)                              # tensor-core kernels
    bc = 1 if path == "w8a8" else 2                            # bytes per B/C element read by the scan
    st_w = 1 if path == "w8a8" else (2 if tc_shape else 4)     # chunk-state element
    hc_w = 1 if path == "w8a8" else 2                           # passed-state element
    vec = chains * nc * Q * 4                                   # one [B,H,nc,Q] fp32 vector (Acs, LUT_state, dt)
    fin = w.batch * H * P * N * (4 if path == "bf16" else 1)
    if kernel == "quantize_inputs":
        return T * G * N * (2 * 2 + 2 * 1)
    if kernel == "chunk_cumsum":                                # dt in; Acs, LUT_state, dt chunk-major, decay out
        return T * H * 4 + 3 * vec + chains * nc * 4
    if kernel == "chunk_state":                                 # x, B, LUT_state in; chunk states out
        return T * (2 * H * P + bc * G * N) + vec + states * st_w
    if kernel == "state_passing":                               # states, decay in; passed states, final out
        return states * st_w + chains * nc * 4 + states * hc_w + fin
    if kernel == "chunk_scan":                                  # x, B, C, Acs, dt, passed states in; y out
        return T * (2 * H * P + 2 * bc * G * N + 2 * H * P) + 2 * vec + states * hc_w
    if kernel == "ssd_fused_i8":                                # the whole scan: x, Bq, Cq, dt in; y, final out
        return T * (2 * H * P + 2 * G * N + 4 * H + 2 * H * P) + fin + 4 * (2 * G + 2 * H * P) + 8 * H
    return 0


def io_bytes(w, path: str, kernel: str) -> int:
    """Algorithmic bytes of one launch as the roofline counts them: only the path's own inputs
    and outputs that the launch reads or writes, each once (no intermediates: chunk states,
    passed states, per-chunk vectors)."""
    T, H, P, N, G = w.tokens, w.nheads, w.headdim, w.dstate, w.ngroups
    bc = 1 if path == "w8a8" else 2                             # bytes per B/C element the scan reads
    fin = w.batch * H * P * N * (4 if path == "bf16" else 1)
    if kernel == "quantize_inputs":                             # B, C in (bf16); Bq, Cq out
        return T * G * N * (2 * 2 + 2 * 1)
    if kernel == "chunk_cumsum":                                # dt in
        return T * H * 4
    if kernel == "chunk_state":                                 # x, B in
        return T * (2 * H * P + bc * G * N)
    if kernel == "state_passing":                               # final state out
        return fin
    if kernel == "chunk_scan":                                  # x, B, C, dt in; y out
        return T * (4 * H * P + 2 * bc * G * N + 4 * H)
    if kernel == "ssd_fused_i8":                                # the whole scan
        return T * (4 * H * P + 2 * G * N + 4 * H) + fin
    return 0


def path_flops(w, path: str):
    """Algorithmic (triangular where causal) contraction counts of one step, 2 per MAC:
    (bf16 FLOPs, INT8 ops).  Per (b, c, h): ChunkState and ChunkScan1 2 Q P N each,
    ChunkScan2 Q (Q + 1) P; per (b, c, g): ChunkBMM Q (Q + 1) N."""
    Q, P, N = w.chunk, w.headdim, w.dstate
    bch = w.batch * w.nchunks * w.nheads
    bcg = w.batch * w.nchunks * w.ngroups
    state = scan1 = 2.0 * Q * P * N * bch
    scan2 = float(Q) * (Q + 1) * P * bch
    bmm = float(Q) * (Q + 1) * N * bcg
    if path == "w8a8":
        return scan2, state + scan1 + bmm
    return state + scan1 + scan2 + bmm, 0.0


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def measured_bf16_tflops() -> float:
    """Burst bf16 dense GEMM throughput measured on this machine (TFLOP/s), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f).get("bf16_tflops", 1590.0))
    return 1590.0


# Per-launch DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu
# capture, keyed by kernel name, with the sha1 of the kernel source it was taken on.
# A kernel whose source changed since reports null.
NCU_TRAFFIC = {
    # batch-2 captures scaled x4 to the batch-8 launch (traffic grows with the batch); src_sha1 is the
    # code hash (_code_hash) of the kernel's source at the capture
    ("chunk_scan", "w8a8", "mamba2-2.7b"): {"bytes_per_launch": 4 * (224.51e6 + 123.36e6),
                                            "src_sha1": "acb43f60bf2fbd5eb0e9707b62df12477c28a626"},
    ("chunk_scan", "bf16", "mamba2-2.7b"): {"bytes_per_launch": 4 * (270.60e6 + 128.16e6),
                                            "src_sha1": "acb43f60bf2fbd5eb0e9707b62df12477c28a626"},
    ("ssd_fused_i8", "w8a8", "mamba2-2.7b"): {"bytes_per_launch": 4 * (178.17e6 + 176.30e6),
                                              "src_sha1": "1fdea2cb386fcb644dba6640df7309df1be58d3c"},
}


def _code_hash(text: str) -> str:
    """sha1 of a CUDA source with its comments and whitespace removed, so that a capture stays
    attached to a kernel whose code has not changed."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return hashlib.sha1(re.sub(r"\s+", "", text).encode()).hexdigest()


def _src_hash(kernel: str):
    f = {"chunk_scan": "chunk_scan_tc.cu", "chunk_state": "chunk_state_tc.cu", "state_passing": "state_passing.cu",
         "chunk_cumsum": "cumsum.cu", "quantize_inputs": "quantize.cu", "ssd_fused_i8": "fused_i8.cu"}.get(kernel)
    if not f:
        return None
    with open(os.path.join(ROOT, "int8_quant_b200", "csrc", f)) as fh:
        return _code_hash(fh.read())


def traffic_for(kernel: str, path: str, workload: str):
    e = NCU_TRAFFIC.get((kernel, path, workload))
    if not e or e["src_sha1"] != _src_hash(kernel):
        return None
    return e["bytes_per_launch"]


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons of the GPU, read through NVML every
    millisecond on a background thread while the context is open (read-only queries;
    the timed steps last milliseconds, below nvidia-smi's sampling interval).  Falls
    back to an nvidia-smi subprocess when NVML is not importable."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))
    SMI_Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.device = device
        self.samples = []            # (sm MHz, max sm MHz, set of reasons)
        self.source = None
        self.err = None

    def _uuid(self):
        try:
            u = str(torch.cuda.get_device_properties(self.device).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return None

    def _nvml_loop(self, nv, h):
        names = [(n, getattr(nv, c)) for n, c in self.REASONS if hasattr(nv, c)]
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop.is_set():
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.samples.append((float(sm), float(mx), {n for n, b in names if bits & b}))
            self._stop.wait(0.001)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._thread = self.proc = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = self._uuid()
            h = nv.nvmlDeviceGetHandleByUUID(uuid) if uuid else nv.nvmlDeviceGetHandleByIndex(self.device.index)
            self._thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self._thread.start()
            self.source = "nvml, 1 ms"
        except Exception as e:                 # no NVML: nvidia-smi at its fastest interval
            self.err = f"nvml: {e}"
            try:
                self.path = os.path.join("/tmp", f"ssd_bench_clocks_{os.getpid()}.csv")
                self.fh = open(self.path, "w")
                gpu = self._uuid() or str(self.device.index)
                self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.SMI_Q}", "--format=csv,noheader,nounits",
                                              "-i", gpu, "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
                self.source = "nvidia-smi, 100 ms"
            except (OSError, FileNotFoundError):
                self.proc = None
                if getattr(self, "fh", None):
                    self.fh.close()
                    try:
                        os.remove(self.path)
                    except OSError:
                        pass
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    try:
                        self.samples.append((float(parts[1]), float(parts[2]),
                                             {n for n, v in zip(names, parts[5:9]) if v.lower() == "active"}))
                    except (ValueError, IndexError):
                        continue
            try:
                os.remove(self.path)
            except OSError:
                pass

    def summary(self):
        if not self.source:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": f"unavailable ({self.err})"}
        sm = [x[0] for x in self.samples]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(x[1] for x in self.samples) if sm else None,
                "reasons": sorted(set().union(*[x[2] for x in self.samples])) if sm else [],
                "samples": len(sm), "source": self.source}


# ---------------------------------------------------------------- CPU oracle baseline
def _oracle_chain(args):
    """Time the oracle on one (batch, head) chain of the workload (inputs generated untimed)."""
    name, b, h, path, budget_s = args
    sys.path.insert(0, ROOT)
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    from harness import WORKLOADS as WL, make_chain as mk, as_float as af
    from oracle import ssd_fp64 as F, ssd_w8a8 as W
    w = WL[name]
    ch = mk(w, b, h)
    x = af(ch["x"])[None, :, None, :]
    dt = ch["dt"][None, :, None]
    Bv = af(ch["B"])[None, :, None, :]
    Cv = af(ch["C"])[None, :, None, :]
    A = np.array([ch["A"]], np.float32)
    D = np.array([ch["D"]], np.float32)
    if path != "bf16":
        # static scales, calibrated once on the chain's prefix outside the timed loop (the GPU step
        # also runs with scales set beforehand); the loop times quantisation + the integer scan
        sc = F.calibrate(x, dt, A, Bv, Cv, w.chunk, w.calib_prefix)
    done, t0 = 0, time.perf_counter()
    while True:
        if path == "bf16":
            F.ssd_sequential(x, dt, A, Bv, Cv, D)
        else:
            Bq, Cq = W.quantize_inputs(Bv.astype(np.float32), Cv.astype(np.float32), sc["s_B"], sc["s_C"])
            W.ssd_w8a8(x.astype(np.float32), dt, A, Bq, Cq, D, sc["s_B"], sc["s_C"], sc["s_x"], sc["s_s"],
                       w.chunk)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            return done, el


def cpu_oracle_sample(w, path: str, budget_s: float, pool=None):
    """Oracle throughput on host cores: each worker repeats one full-length chain for ~budget_s.

    tokens/s = (chains finished × L / H) / slowest worker's time, i.e. the rate at which
    the oracle would process whole tokens (all H heads)."""
    cores = os.cpu_count() or 1
    rs = np.random.default_rng(0)
    jobs = [(w.name, int(rs.integers(w.batch)), int(rs.integers(w.nheads)), path, budget_s) for _ in range(cores)]
    own = pool is None
    if own:
        pool = mp.get_context("spawn").Pool(cores)
    try:
        res = pool.map(_oracle_chain, jobs)
    finally:
        if own:
            pool.close()
            pool.join()
    chains = sum(r[0] for r in res)
    t = max(r[1] for r in res)
    value = chains * w.seqlen / w.nheads / t
    sample = (f"{chains} full-length (L={w.seqlen}) (batch, head) chains of {w.name}, "
              f"{'fp64 sequential recurrence' if path == 'bf16' else 'quantisation + integer W8A8 pipeline, scales calibrated once per chain, untimed'}, "
              f"{cores} spawn workers, {t:.1f} s")
    return {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}


# ---------------------------------------------------------------- GPU arm
# ---------------------------------------------------------------- replicas
def max_over_ranks(v: float, dist=None, device="cpu") -> float:
    """The largest of every rank's `v` (the slowest replica's time); `dist` None: one process."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank: int, ms_per_step: float, world: int) -> float:
    """Whole-job tokens/s of `world` replicas that each process `tokens_per_rank` tokens per step,
    with the step time taken as the max over ranks (weak scaling)."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# kernels each profiled stage launches (the single-launch scan's stage also runs the
# small kernel that forms its per-(h,p) factors)
KERNELS_PER_STAGE = {"ssd_fused_i8": 2}


def kernel_launches(kern) -> int:
    """This library's kernel launches behind the per-stage counts of ssd_profile_read."""
    return sum(c * KERNELS_PER_STAGE.get(k, 1) for k, (_, c) in kern.items())


def tc_shape(w) -> bool:
    """(P, N) = (64, 128): the shape the tensor-core kernels (and the single-launch scan) take."""
    return (w.headdim, w.dstate) == (64, 128)


def run_ours(args, rank, world, dist):
    import torch
    import int8_quant_b200 as iq
    from int8_quant_b200.runner import SsdProblem, to_device

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    host = make_inputs(w)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        dinp = to_device(host, dev)
        pb = SsdProblem(dinp, w.chunk, with_i8=True, with_bf16=True)
        pb.calibrate(w.calib_prefix)            # static W8A8 scales on the prefix (GPU)
    torch.cuda.synchronize()
    peak, peak_src = measured_peaks()
    bf16_peak = measured_bf16_tflops()

    def step_fn(path, pb):
        if path == "w8a8":
            return lambda: pb.run_i8(stream)
        return lambda: pb.run_bf16(stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    def timed(path, pb=pb):
        """Step time over the timed loop, CUDA events around all its steps.  Inside that loop only
        the dominant kernel (the largest share of the warm-up steps' device time) is bracketed by
        an event pair, so its launch time is measured live in the timed region at two events per
        step; the other kernels' split comes from a profiled pass of the same number of steps
        right after (an event pair around every kernel adds about 14 us to a W8A8 step)."""
        step = step_fn(path, pb)
        iq.ssd_profile_filter(None)
        iq.ssd_profile_reset()
        iq.ssd_profile_enable(True)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        iq.ssd_profile_enable(False)
        warm = {k: v for k, v in iq.ssd_profile_read().items() if v[1]}
        dom = max(warm, key=lambda k: warm[k][0])
        iq.ssd_profile_reset()
        iq.ssd_profile_filter(dom)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev) as clk:
            barrier()
            torch.cuda.synchronize()
            iq.ssd_profile_enable(True)
            ev0.record(stream)
            for _ in range(args.steps):
                step()
            ev1.record(stream)
            torch.cuda.synchronize()
            iq.ssd_profile_enable(False)
            barrier()
        ms = max_over_ranks(ev0.elapsed_time(ev1), dist, dev) / args.steps
        dom_t = iq.ssd_profile_read()[dom]
        iq.ssd_profile_filter(None)
        iq.ssd_profile_reset()
        iq.ssd_profile_enable(True)
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
        iq.ssd_profile_enable(False)
        kern = iq.ssd_profile_read()
        kern[dom] = dom_t                                   # the dominant kernel as timed in the timed loop
        return ms, kern, clk.summary()

    def roofline(path, kern, w=w):
        # dominant kernel = largest share of the step's device time; its algorithmic bytes are
        # the path inputs and outputs it touches (no intermediates)
        name = max(kern, key=lambda k: kern[k][0])
        tot_ms, calls = kern[name]
        per_launch_s = tot_ms / calls / 1e3
        alg = io_bytes(w, path, name)
        achieved = alg / per_launch_s / 1e9
        kb = kernel_bytes(w, path, name)
        return {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "frac_of_8TBs": round(achieved / DATASHEET_HBM_GBS, 4),
                "traffic": traffic_for(name, path, w.name), "alg_bytes_per_launch": alg,
                "alg_bytes_def": "path inputs and outputs the launch touches, each once",
                "launch_ms": round(per_launch_s * 1e3, 4), "peak_source": peak_src,
                "with_intermediates": {"bytes_per_launch": kb, "frac": round(kb / per_launch_s / 1e9 / peak, 4)},
                "kernel_shares": {k: round(v[0] / sum(x[0] for x in kern.values()), 4) for k, v in kern.items()}}

    def path_roofline(path, ms, w=w):
        """The step against the SSD scan's roofline: the slower of the compulsory HBM bytes over
        8 TB/s and the contractions at the datasheet tensor peaks (bf16 2.25 PFLOP/s, int8
        4.5 POP/s), and the same with this machine's measured peaks (copy bandwidth; bf16 GEMM,
        int8 taken as twice it)."""
        alg = path_bytes(w, path)
        fb, oi = path_flops(w, path)
        t = ms / 1e3
        t_hbm, t_mma = alg / (DATASHEET_HBM_GBS * 1e9), fb / 2.25e15 + oi / 4.5e15
        t_hbm_m, t_mma_m = alg / (peak * 1e9), fb / (bf16_peak * 1e12) + oi / (2 * bf16_peak * 1e12)
        return {"alg_bytes": alg, "bf16_flops": fb, "int8_ops": oi, "achieved_GBs": round(alg / t / 1e9, 1),
                "t_roof_us": round(max(t_hbm, t_mma) * 1e6, 2), "bound": "hbm" if t_hbm >= t_mma else "tensor",
                "frac": round(max(t_hbm, t_mma) / t, 4),
                "frac_of_measured": round(max(t_hbm_m, t_mma_m) / t, 4),
                "frac_of_measured_hbm": round(alg / t / 1e9 / peak, 4),
                "frac_of_8TBs": round(alg / t / 1e9 / DATASHEET_HBM_GBS, 4)}

    def decode_time(path, state, toks, steps, warm):
        """Average decode-kernel time (µs) over `steps` one-token steps, L2 refilled before each."""
        from int8_quant_b200.runner import Decoder
        dec = Decoder(state, dinp["A"], dinp["D"], path, pb.scales if path == "w8a8" else None)
        flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        for i in range(warm):
            dec.step(**toks[i % len(toks)], stream=stream)
        torch.cuda.synchronize()
        iq.ssd_profile_reset()
        for i in range(steps):
            with torch.cuda.stream(stream):
                flush.amax()
            iq.ssd_profile_enable(True)
            dec.step(**toks[i % len(toks)], stream=stream)
            iq.ssd_profile_enable(False)
        torch.cuda.synchronize()
        kern = iq.ssd_profile_read()
        return {k: v[0] / max(v[1], 1) * 1e3 for k, v in kern.items()}

    def decode_bytes(path, b):
        H, P, N, G = w.nheads, w.headdim, w.dstate, w.ngroups
        eb = 1 if path == "w8a8" else 4
        return b * H * P * N * eb * 2 + b * H * P * 4 + b * H * 4 + b * G * N * 4

    def decode(path, steps=50, warm=5):
        """One-token steps continuing the scan's final state (ssd_decode_step_*, one launch
        per token; W8A8 quantises the token's B and C inside).  L2 is refilled with other
        data before every step (a read of 256 MB, which leaves no dirty lines to write
        back), so each step reads and writes the whole state from HBM, as it would between
        the other layers of a model; the time is the decode kernel's own (CUDA events
        around each launch), not the refill.  `batch_sweep` repeats the step at larger
        batches (synthetic tokens of the same recipe, a random state) to separate the
        per-launch floor from the per-byte cost."""
        state = (pb.final8 if path == "w8a8" else pb.final32).clone()
        toks = [{k: dinp[k][:, t].contiguous() for k in ("x", "dt", "B", "C")} for t in range(8)]
        us = decode_time(path, state, toks, steps, warm)
        step_us = sum(us.values())
        b = w.batch
        alg = decode_bytes(path, b)
        k_us = us.get("decode_step", 0.0)
        sweep = {}
        g = torch.Generator(device=dev).manual_seed(11)
        for bb in (32, 128):
            ti = to_device(make_inputs(w.with_(batch=bb, seqlen=8)), dev)
            tk = [{k: ti[k][:, t].contiguous() for k in ("x", "dt", "B", "C")} for t in range(8)]
            shp = (bb, w.nheads, w.headdim, w.dstate)
            st = (torch.randint(-90, 91, shp, generator=g, device=dev, dtype=torch.int8) if path == "w8a8"
                  else torch.randn(shp, generator=g, device=dev))
            t_us = decode_time(path, st, tk, 20, 3).get("decode_step", 0.0)
            ab = decode_bytes(path, bb)
            sweep[str(bb)] = {"us": round(t_us, 3), "alg_bytes": ab,
                              "achieved": round(ab / (t_us * 1e-6) / 1e9, 1) if t_us else None,
                              "frac": round(ab / (t_us * 1e-6) / 1e9 / peak, 4) if t_us else None}
            del ti, tk, st
        return {"tokens_per_s": round(b / (step_us * 1e-6), 1), "us_per_step": round(step_us, 3),
                "kernels_us": {k: round(v, 3) for k, v in us.items() if v},
                "roofline": {"kernel": "decode_step", "bound": "hbm", "alg_bytes": alg,
                             "achieved": round(alg / (k_us * 1e-6) / 1e9, 1) if k_us else None, "peak": peak,
                             "unit": "GB/s", "frac": round(alg / (k_us * 1e-6) / 1e9 / peak, 4) if k_us else None},
                "batch_sweep": sweep,
                "state": f"{'int8' if path == 'w8a8' else 'fp32'} [{b},{w.nheads},{w.headdim},{w.dstate}], "
                         "continuing the scan's final state",
                "l2": "refilled with 256 MB of other reads before every step"}

    def out_proj(steps=10, warm=3):
        """The SSD epilogue on the scan's y seen as [B*L, H*P]: RMSNorm codes + the INT8 output
        projection to d_model = H*P/2 (the 2.7B layer's 2560) on synthetic weights (seeded; the
        weight codes and the static scales are set up with torch outside the timed region).
        y (671 MB) is larger than L2, so every launch reads it from HBM."""
        T, K = w.tokens, w.nheads * w.headdim
        Dm = K // 2
        g = torch.Generator(device=dev).manual_seed(0)
        Wf = torch.randn((Dm, K), generator=g, device=dev) / K ** 0.5
        s_w = (Wf.abs().amax(dim=1) / 127).contiguous()
        Wq = torch.clamp(torch.round(Wf / s_w[:, None]), -127, 127).to(torch.int8).contiguous()
        corr = (1e-3 * torch.randn(Dm, generator=g, device=dev)).contiguous()
        y2 = pb.y.view(T, K)
        u = y2[: 4096].float()
        s_a = float((u * torch.rsqrt(u.pow(2).mean(dim=1, keepdim=True) + 1e-5)).abs().amax() / 127)
        out = torch.empty((T, Dm), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(iq.ssd_out_proj_workspace_bytes(T, K), dtype=torch.uint8, device=dev)
        for _ in range(warm):
            iq.ssd_out_proj_i8(y2, s_a, Wq, s_w, corr, out, ws, stream=stream)
        torch.cuda.synchronize()
        iq.ssd_profile_reset()
        iq.ssd_profile_enable(True)
        for _ in range(steps):
            iq.ssd_out_proj_i8(y2, s_a, Wq, s_w, corr, out, ws, stream=stream)
        iq.ssd_profile_enable(False)
        torch.cuda.synchronize()
        assert iq.ssd_out_proj_status(ws, T, K) == 0
        kern = {k: v[0] / max(v[1], 1) for k, v in iq.ssd_profile_read().items() if v[1]}
        gemm_ms, norm_ms = kern.get("out_proj_gemm", 0.0), kern.get("out_proj_norm", 0.0)
        ops = 2.0 * T * K * Dm
        i8_peak = 2.0 * bf16_peak
        norm_bytes = T * K * 2 + T * K                     # y read (its second pass per token hits L2), codes written
        return {"tokens": T, "d_inner": K, "d_model": Dm, "ms_per_call": round(gemm_ms + norm_ms, 5),
                "tokens_per_s": round(T / ((gemm_ms + norm_ms) * 1e-3), 1),
                "gemm": {"ms": round(gemm_ms, 5), "bound": "tensor", "achieved": round(ops / (gemm_ms * 1e-3) / 1e12, 1),
                         "peak": round(i8_peak, 1), "unit": "TOP/s", "frac": round(ops / (gemm_ms * 1e-3) / 1e12 / i8_peak, 4),
                         "peak_source": "2 x measured bf16 burst (MEASURED_PEAKS.json), the nominal int8/bf16 ratio"},
                "norm": {"ms": round(norm_ms, 5), "bound": "hbm", "alg_bytes": norm_bytes,
                         "achieved": round(norm_bytes / (norm_ms * 1e-3) / 1e9, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(norm_bytes / (norm_ms * 1e-3) / 1e9 / peak, 4)},
                "weights": "synthetic, seeded; corr = synthetic mean-correction vector"}

    def e2e(path):
        """Same metric with the batch in pinned host memory: every step copies the inputs in and y and
        the final state out, group by group (StreamedScan: one batch row per group, or with
        `--e2e-seg` one row's segment of that many tokens, each continuing from the previous
        one's state), overlapping the copies in both directions with the scans."""
        from int8_quant_b200.runner import StreamedScan
        names = ["x", "dt", "B", "C"]
        host_io = {k: dinp[k].to("cpu").pin_memory() for k in names}
        fin = pb.final8 if path == "w8a8" else pb.final32
        host_io["y"] = torch.empty_like(pb.y, device="cpu").pin_memory()
        host_io["final"] = torch.empty_like(fin, device="cpu").pin_memory()
        seg = args.e2e_seg if args.e2e_seg and args.e2e_seg % w.chunk == 0 else None
        runner = StreamedScan(host_io, dinp["A"], dinp["D"], w.chunk, path, rows_per_group=1,
                              scales=pb.scales if path == "w8a8" else None, device=dev, seg_len=seg)
        n = max(1, args.steps)
        runner.run()                                             # warm-up
        torch.cuda.synchronize()
        barrier()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(runner.streams[0])
        for _ in range(n):
            runner.run()
        ev1.record(runner.streams[2])
        torch.cuda.synchronize()
        barrier()
        ms = max_over_ranks(ev0.elapsed_time(ev1), dist, dev) / n
        return {"value": replica_throughput(w.tokens, ms, world), "unit": "tokens/s",
                "h2d_bytes_per_step": runner.h2d_bytes, "d2h_bytes_per_step": runner.d2h_bytes,
                "ms_per_step": round(ms, 4), "steps": n, "rows_per_group": 1, "segment_tokens": runner.seg,
                "groups_per_step": len(runner.groups),
                "api": "ssd_quantize_inputs + ssd_scan_fwd_i8" if path == "w8a8" else "ssd_scan_fwd_bf16"}

    def fused_i8(w=w, pb=pb):
        """The W8A8 step with the scan as one persistent launch (SSD_I8_FUSED=1): same integers,
        timed the same way."""
        old = os.environ.get("SSD_I8_FUSED")
        os.environ["SSD_I8_FUSED"] = "1"
        try:
            ms, kern, clocks = timed("w8a8", pb)
        finally:
            if old is None:
                del os.environ["SSD_I8_FUSED"]
            else:
                os.environ["SSD_I8_FUSED"] = old
        return {"value": replica_throughput(w.tokens, ms, world), "ms_per_step": round(ms, 5),
                "roofline": roofline("w8a8", kern, w), "path_roofline": path_roofline("w8a8", ms, w),
                "gpu_launches": kernel_launches(kern), "clocks": clocks,
                "kernels_ms_per_step": {k: round(v[0] / args.steps, 5) for k, v in kern.items()}}

    def storage_variant(w=w, pb=pb):
        """The W8A8 step with the notes' storage variant (Acs as FP16, CB requantised to INT8
        tiles in HBM by a ChunkBMM kernel and read back by ChunkScan2), timed the same way;
        its DRAM traffic is measured with ncu (the bytes it adds are intermediates, so the
        path roofline's compulsory bytes are the same)."""
        pb.set_storage(iq.SSD_STORAGE_ACS_FP16 | iq.SSD_STORAGE_CB_INT8)
        try:
            ms, kern, clocks = timed("w8a8", pb)
        finally:
            pb.set_storage(0)
        return {"value": replica_throughput(w.tokens, ms, world), "ms_per_step": round(ms, 5),
                "path_roofline": path_roofline("w8a8", ms, w), "gpu_launches": kernel_launches(kern),
                "clocks": clocks, "kernels_ms_per_step": {k: round(v[0] / args.steps, 5) for k, v in kern.items()},
                "storage": "Acs FP16 + CB INT8 in HBM (SSD_STORAGE_ACS_FP16 | SSD_STORAGE_CB_INT8)"}

    def other_config(name):
        """Device-timed step of another workload on both paths (its own inputs, calibrated the
        same way); no e2e, decode or epilogue."""
        wo = WORKLOADS[name]
        with torch.cuda.stream(stream):
            di = to_device(make_inputs(wo), dev)
            po = SsdProblem(di, wo.chunk, with_i8=True, with_bf16=True)
            po.calibrate(wo.calib_prefix)
        torch.cuda.synchronize()
        cfg = config_of(wo, "bf16", world)
        cfg.update(path="bf16 and w8a8", step="as in the main line, per path",
                   l2=f"inputs larger than L2 ({path_bytes(wo, 'w8a8') / 1e9:.2f} GB or more per step), no flush")
        out = {"config": cfg}
        for path in ("bf16", "w8a8"):
            ms, kern, clocks = timed(path, po)
            rf = roofline(path, kern, wo)
            out[path] = {"value": replica_throughput(wo.tokens, ms, world), "ms_per_step": round(ms, 5),
                         "path_roofline": path_roofline(path, ms, wo),
                         "roofline": {k: rf[k] for k in ("kernel", "achieved", "frac", "frac_of_8TBs", "launch_ms")},
                         "gpu_launches": kernel_launches(kern), "clocks": clocks,
                         "kernels_ms_per_step": {k: round(v[0] / args.steps, 5) for k, v in kern.items()}}
        if tc_shape(wo):
            out["w8a8_fused"] = {k: v for k, v in fused_i8(wo, po).items() if k != "kernels_ms_per_step"}
        del po, di
        torch.cuda.empty_cache()
        return out

    results = {}
    paths = (args.path,) if args.only_path else (args.path, "bf16" if args.path == "w8a8" else "w8a8")
    for path in paths:
        ms, kern, clocks = timed(path)
        launches = kernel_launches(kern)
        results[path] = {
            "ms_per_step": ms, "value": replica_throughput(w.tokens, ms, world), "kern": kern, "clocks": clocks,
            "roofline": roofline(path, kern), "gpu_launches": launches,
            "path_roofline": path_roofline(path, ms),
        }
        if not args.no_e2e:
            results[path]["e2e"] = e2e(path)
    if "w8a8" in paths and tc_shape(w) and not args.no_fused:
        results["w8a8_fused"] = fused_i8()
    if "w8a8" in paths and tc_shape(w) and w.chunk == 256 and not args.no_storage_variant:
        results["w8a8_notes_storage"] = storage_variant()
    if not args.no_decode:
        results["decode"] = {p: decode(p) for p in paths}
    if not args.no_out_proj:
        results["out_proj"] = out_proj()
    if args.all_configs:                          # "tiny" is a parity case (launch-bound), not timed
        results["configs"] = {n: other_config(n) for n in sorted(WORKLOADS) if n not in (w.name, "tiny")}
    return w, results


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba2-2.7b", choices=sorted(WORKLOADS))
    ap.add_argument("--path", choices=["w8a8", "bf16"], default="w8a8")
    ap.add_argument("--no-decode", action="store_true", help="skip the one-token decode-step measurement")
    ap.add_argument("--no-out-proj", action="store_true", help="skip the SSD-epilogue (INT8 out projection) measurement")
    ap.add_argument("--only-path", action="store_true", help="time only --path (profiling runs)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling runs)")
    ap.add_argument("--seqlen", type=int, default=None, help="override the workload's length (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-seg", type=int, default=0,
                    help="tokens per copy group in the e2e leg (a multiple of the chunk; 0: whole batch rows, "
                         "the fastest measured: 15.7 ms per 2.7B W8A8 step against 20.3 ms with 1024-token groups)")
    ap.add_argument("--no-fused", action="store_true", help="skip the single-launch W8A8 scan measurement")
    ap.add_argument("--no-storage-variant", action="store_true",
                    help="skip the W8A8 step with the notes' storage variant (FP16 Acs, INT8 CB in HBM)")
    ap.add_argument("--all-configs", action="store_true",
                    help="also time every other workload on both paths (device time only); the default on one GPU")
    ap.add_argument("--no-all-configs", action="store_true", help="time only --workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work per CPU worker")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    # every workload on one GPU by default (input generation dominates its added time); opt-in under torchrun
    if int(os.environ.get("WORLD_SIZE", "1")) == 1 and args.batch is None and args.seqlen is None:
        args.all_configs = True
    if args.no_all_configs:
        args.all_configs = False

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.batch is not None or args.seqlen is not None:
        base = WORKLOADS[args.workload]
        name = f"{base.name}-b{args.batch or base.batch}-l{args.seqlen or base.seqlen}"
        WORKLOADS[name] = base.with_(name=name, batch=args.batch or base.batch, seqlen=args.seqlen or base.seqlen)
        args.workload = name
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        # The reference arm is the CPU oracle, timed on the host cores; rank 0 only.
        if rank != 0:
            return
        vals = []
        pool = mp.get_context("spawn").Pool(os.cpu_count() or 1)
        try:
            for i in range(args.warmup + args.steps):
                r = cpu_oracle_sample(w, args.path, args.cpu_budget / 4, pool)
                if i >= args.warmup:
                    vals.append(r)
        finally:
            pool.close()
            pool.join()
        value = statistics.median(v["value"] for v in vals)
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * w.tokens / value,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64" if args.path == "bf16" else "int64", "data": "synthetic",
                "config": config_of(w, args.path, args.gpus),
                "ms_per_step_note": ("extrapolated: the workload's B*L tokens over the oracle's throughput "
                                     "on sampled chains, not a timed whole step"),
                "cpu_baseline": {"kind": "oracle", "cores": vals[0]["cores"], "sample": vals[0]["sample"],
                                 "value": value, "unit": "tokens/s"},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    # CPU pool for the oracle baseline: spawned before the first GPU call.
    pool = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pool = mp.get_context("spawn").Pool(os.cpu_count() or 1)

    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as td
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = td
    try:
        w, res = run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    cpu = None
    if pool is not None:
        try:
            cpu = cpu_oracle_sample(w, args.path, args.cpu_budget, pool)
        finally:
            pool.close()
            pool.join()
    if rank != 0:
        return
    main_r = res[args.path]
    other = "bf16" if args.path == "w8a8" else "w8a8"
    o = res.get(other)
    line = {
        "metric": METRIC, "value": main_r["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(main_r["ms_per_step"], 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8" if args.path == "w8a8" else "bf16",
        "data": "synthetic",
        "config": config_of(w, args.path, world),
        "roofline": main_r["roofline"], "path_roofline": main_r["path_roofline"],
        "cpu_baseline": cpu, "e2e": main_r.get("e2e"), "gpu_launches": main_r["gpu_launches"],
        "clocks": main_r["clocks"],
        "kernels_ms_per_step": {k: round(v[0] / args.steps, 5) for k, v in main_r["kern"].items()},
    }
    if "w8a8_fused" in res:
        line["w8a8_fused"] = res["w8a8_fused"]
    if "w8a8_notes_storage" in res:
        line["w8a8_notes_storage"] = res["w8a8_notes_storage"]
    if "configs" in res:
        line["configs"] = res["configs"]
    if "decode" in res:
        line["decode"] = res["decode"]
    if "out_proj" in res:
        line["out_proj"] = res["out_proj"]
    if o is not None:
        line[other] = {"value": o["value"], "ms_per_step": round(o["ms_per_step"], 5), "roofline": o["roofline"],
                       "path_roofline": o["path_roofline"], "e2e": o.get("e2e"), "gpu_launches": o["gpu_launches"],
                       "clocks": o["clocks"],
                       "kernels_ms_per_step": {k: round(v[0] / args.steps, 5) for k, v in o["kern"].items()}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
