"""bench.py's roofline arithmetic on CPU: compulsory bytes, contraction counts and t_roof.

The expected figures are worked by hand from the definitions (each input read once, each
output written once; causal contraction counts, 2 per multiply-add), not by calling the
functions under test.  For the Mamba-2 2.7B layer shape (B=8, L=8192, H=80, P=64, N=128,
G=1, Q=256): per token x and y are 2*80*64 bytes each and dt 4*80; B and C are 4*128
bytes as bf16 and 2*128 as INT8 codes; the final state is 8*80*64*128 elements.  Chunks:
32 per sequence, so 8*32*80 = 20480 (b, c, h) triples and 256 (b, c, g) pairs.
"""
import pytest

import bench
from harness import WORKLOADS


def test_path_bytes_27b():
    w = WORKLOADS["mamba2-2.7b"]
    tok = 8 * 8192
    fin = 8 * 80 * 64 * 128
    assert bench.path_bytes(w, "bf16") == tok * (2 * 2 * 80 * 64 + 4 * 128 + 4 * 80) + 4 * fin
    assert bench.path_bytes(w, "w8a8") == tok * (2 * 2 * 80 * 64 + 2 * 128 + 4 * 80) + fin
    assert round(bench.path_bytes(w, "bf16") / 1e6, 1) == 1417.7
    assert round(bench.path_bytes(w, "w8a8") / 1e6, 1) == 1385.2


def test_path_flops_27b():
    w = WORKLOADS["mamba2-2.7b"]
    bch, bcg = 20480, 256
    state = 2 * 256 * 64 * 128 * bch            # ChunkState; ChunkScan1 is the same
    scan2 = 256 * 257 * 64 * bch                # causal Q x Q against x, lower triangle incl. diagonal
    bmm = 256 * 257 * 128 * bcg                 # causal C B^T per group
    fb, oi = bench.path_flops(w, "bf16")
    assert (fb, oi) == (2 * state + scan2 + bmm, 0.0)
    fb, oi = bench.path_flops(w, "w8a8")
    assert (fb, oi) == (scan2, 2 * state + bmm)
    assert round((2 * state + scan2 + bmm) / 1e9, 1) == 260.2


@pytest.mark.parametrize("name,path,us", [("mamba2-2.7b", "bf16", 177.2), ("mamba2-8b", "w8a8", 72.9),
                                          ("long-256k", "bf16", 698.7)])
def test_t_roof_is_hbm_bound(name, path, us):
    """t_roof = max(bytes / 8 TB/s, bf16 FLOPs / 2.25 PFLOP/s + INT8 ops / 4.5 POP/s)."""
    w = WORKLOADS[name]
    b = bench.path_bytes(w, path)
    fb, oi = bench.path_flops(w, path)
    t_hbm, t_mma = b / 8e12, fb / 2.25e15 + oi / 4.5e15
    assert t_hbm > t_mma
    assert round(t_hbm * 1e6, 1) == us


def test_io_bytes_are_path_bytes_for_one_launch():
    """The single-launch scan touches every path input and output: with quantisation counted
    in a launch of its own, the two add up to the path's bytes plus quantisation's B/C traffic."""
    w = WORKLOADS["mamba2-2.7b"]
    tok, G, N = w.tokens, w.ngroups, w.dstate
    assert bench.io_bytes(w, "w8a8", "ssd_fused_i8") == bench.path_bytes(w, "w8a8")
    assert bench.io_bytes(w, "w8a8", "quantize_inputs") == tok * G * N * 6
    # the scan's own I/O never exceeds the path's
    for k in ("chunk_cumsum", "chunk_state", "state_passing", "chunk_scan"):
        for p in ("bf16", "w8a8"):
            assert 0 < bench.io_bytes(w, p, k) <= bench.path_bytes(w, p)


def test_reference_arm_config_matches_ours():
    w = WORKLOADS["mamba2-2.7b"]
    c = bench.config_of(w, "w8a8", 1)
    assert c["workload"] == "mamba2-2.7b" and c["step"] == "ssd_quantize_inputs + ssd_scan_fwd_i8"
    assert set(c) == {"workload", "batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "chunk",
                      "path", "step", "l2", "parallelism"}
