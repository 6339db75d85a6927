"""Synthetic Mamba-2 SSD workloads: shapes, value distributions and the seeded inputs.

The inputs stand in for the activations of Mamba-2 layers (no trained weights or
datasets are used).  Recipe, per tensor (all draws from `harness.rng`):

* x[b,t,h,p]  ~ N(0,1), optionally scaled per head by U[1,5] and, on
  round(0.005*H*P) distinct (h,p) channels picked by a seeded permutation, by 20;
  stored as bfloat16 (round to nearest even).
* B, C[b,t,g,n] ~ N(0, 1/N) (variance 1/N), stored as bfloat16.
* dt[b,t,h] = softplus(0.5*z + dt_bias[h]), z ~ N(0,1), with
  dt_bias[h] = softplus^-1(exp(U[ln 1e-3, ln 1e-1])) so that dt is roughly
  log-uniform over [1e-3, 1e-1]; stored as float32 (already positive: the scan
  applies no softplus of its own).
* A[h] = -exp(U[0, ln 16]) (float32), D[h] ~ N(0,1) (float32).

Layouts are the library's: x [B,L,H,P], dt [B,L,H], A [H], B/C [B,L,G,N], D [H],
all row-major.  bfloat16 tensors are carried as uint16 bit patterns.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np

from . import rng


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int          # P
    dstate: int           # N
    ngroups: int          # G
    chunk: int            # Q
    head_scale: bool = False
    outliers: bool = False
    paths: tuple = ("bf16",)
    calib_prefix: int = 512
    seed: int = 0
    note: str = ""

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    @property
    def nchunks(self) -> int:
        return (self.seqlen + self.chunk - 1) // self.chunk

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The measured workloads.  "tiny" is generated in float32 and handed to both
# paths after the bf16 cast, like every other workload.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 256, 4, 16, 16, 1, 64, paths=("bf16", "w8a8"),
                     note="tiny SSD (fp32 recipe, bf16 storage)"),
    "mamba2-1.3b": Workload("mamba2-1.3b", 4, 2048, 64, 64, 128, 1, 256, paths=("bf16",),
                            note="Mamba-2 1.3B layer SSD"),
    "mamba2-2.7b": Workload("mamba2-2.7b", 8, 8192, 80, 64, 128, 1, 256, head_scale=True,
                            outliers=True, paths=("bf16", "w8a8"),
                            note="Mamba-2 2.7B layer SSD, per-head x scale and 0.5% outlier channels"),
    "mamba2-8b": Workload("mamba2-8b", 4, 4096, 128, 64, 128, 8, 256, paths=("w8a8",),
                          note="Mamba-2 8B layer SSD, 8 groups broadcast to 128 heads"),
    "long-16k": Workload("long-16k", 1, 16384, 80, 64, 128, 1, 256, paths=("bf16", "w8a8"),
                         note="long context, 2.7B shape"),
    "long-64k": Workload("long-64k", 1, 65536, 80, 64, 128, 1, 256, paths=("bf16", "w8a8"),
                         note="long context, 2.7B shape"),
    "long-256k": Workload("long-256k", 1, 262144, 80, 64, 128, 1, 256, paths=("bf16", "w8a8"),
                          note="long context, 2.7B shape (1024 chunks)"),
}


def group_of_head(h, nheads: int, ngroups: int):
    """Group g(h) that head h reads B and C from: contiguous blocks of H/G heads."""
    return np.asarray(h) // (nheads // ngroups)


# ---------------------------------------------------------------- per-head parameters

def head_params(w: Workload) -> dict:
    """Per-head quantities: A, D, dt_bias and the x multiplier [H,P] (head scale x outliers)."""
    H, P = w.nheads, w.headdim
    hidx = np.arange(H, dtype=np.uint64)
    ua = rng.uniform(rng.stream_key(w.seed, rng.STREAM_A), hidx)
    A = (-np.exp(ua * math.log(16.0))).astype(np.float32)
    D = rng.normal(rng.stream_key(w.seed, rng.STREAM_D), hidx).astype(np.float32)
    ub = rng.uniform(rng.stream_key(w.seed, rng.STREAM_DT_BIAS), hidx)
    e = np.exp(math.log(1e-3) + ub * (math.log(1e-1) - math.log(1e-3)))
    dt_bias = e + np.log(-np.expm1(-e))                      # softplus^-1(e)
    mult = np.ones((H, P), dtype=np.float64)
    if w.head_scale:
        hs = 1.0 + 4.0 * rng.uniform(rng.stream_key(w.seed, rng.STREAM_HEAD_SCALE), hidx)
        mult *= hs[:, None]
    if w.outliers:
        n_out = int(round(0.005 * H * P))
        keys = rng.uniform(rng.stream_key(w.seed, rng.STREAM_OUTLIER), np.arange(H * P, dtype=np.uint64))
        chosen = np.argsort(keys, kind="stable")[:n_out]
        mult.reshape(-1)[chosen] *= 20.0
    return {"A": A, "D": D, "dt_bias": dt_bias, "x_mult": mult}


def _softplus(v: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, v)


# ---------------------------------------------------------------- whole tensors

def _fill_bf16(key, shape, mult_last2=None, scale=1.0) -> np.ndarray:
    """bf16 bits of scale * N(0,1) [* mult over the two trailing axes], whole tensor."""
    count = int(np.prod(shape))
    out = np.empty(count, dtype=np.uint16)
    tail = None if mult_last2 is None else np.asarray(mult_last2, dtype=np.float64).reshape(-1)

    def work(lo, hi):
        e = hi + (hi & 1)
        v = rng.normal_block(key, lo, e)[: hi - lo] * scale
        if tail is not None:
            v *= tail[np.arange(lo, hi) % tail.size]
        out[lo:hi] = rng.f32_to_bf16_bits(v.astype(np.float32))

    rng.parallel_blocks(count, work)
    return out.reshape(shape)


def make_inputs(w: Workload) -> dict:
    """All inputs of one workload as host arrays (bf16 tensors as uint16 bits)."""
    Bt, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    hp = head_params(w)
    x = _fill_bf16(rng.stream_key(w.seed, rng.STREAM_X), (Bt, L, H, P), mult_last2=hp["x_mult"])
    sd = 1.0 / math.sqrt(N)
    Bm = _fill_bf16(rng.stream_key(w.seed, rng.STREAM_B), (Bt, L, G, N), scale=sd)
    Cm = _fill_bf16(rng.stream_key(w.seed, rng.STREAM_C), (Bt, L, G, N), scale=sd)
    z = rng.normal_range(rng.stream_key(w.seed, rng.STREAM_DT_NOISE), Bt * L * H).reshape(Bt, L, H)
    dt = _softplus(0.5 * z.astype(np.float64) + hp["dt_bias"][None, None, :]).astype(np.float32)
    return {"x": x, "dt": dt, "A": hp["A"], "B": Bm, "C": Cm, "D": hp["D"]}


# ---------------------------------------------------------------- one (batch, head) chain

def make_chain(w: Workload, b: int, h: int, t_end: int | None = None) -> dict:
    """Inputs that the outputs of chain (b, h) depend on, regenerated on their own.

    Returns x [T,P] and B, C [T,N] as bf16 bits, dt [T] float32 and the scalars
    A, D of head h, for tokens [0, T) with T = t_end or the full length.
    """
    L, H, P, N, G = w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    T = L if t_end is None else int(t_end)
    g = int(group_of_head(h, H, G))
    hp = head_params(w)
    t = np.arange(T, dtype=np.uint64)[:, None]
    xi = ((np.uint64(b) * np.uint64(L) + t) * np.uint64(H) + np.uint64(h)) * np.uint64(P) \
        + np.arange(P, dtype=np.uint64)[None, :]
    xv = rng.normal(rng.stream_key(w.seed, rng.STREAM_X), xi) * hp["x_mult"][h][None, :]
    bi = ((np.uint64(b) * np.uint64(L) + t) * np.uint64(G) + np.uint64(g)) * np.uint64(N) \
        + np.arange(N, dtype=np.uint64)[None, :]
    sd = 1.0 / math.sqrt(N)
    Bv = rng.normal(rng.stream_key(w.seed, rng.STREAM_B), bi) * sd
    Cv = rng.normal(rng.stream_key(w.seed, rng.STREAM_C), bi) * sd
    di = (np.uint64(b) * np.uint64(L) + t[:, 0]) * np.uint64(H) + np.uint64(h)
    z = rng.normal(rng.stream_key(w.seed, rng.STREAM_DT_NOISE), di).astype(np.float32)
    dt = _softplus(0.5 * z.astype(np.float64) + hp["dt_bias"][h]).astype(np.float32)
    return {
        "x": rng.f32_to_bf16_bits(xv.astype(np.float32)),
        "B": rng.f32_to_bf16_bits(Bv.astype(np.float32)),
        "C": rng.f32_to_bf16_bits(Cv.astype(np.float32)),
        "dt": dt, "A": hp["A"][h], "D": hp["D"][h], "g": g,
    }


def make_group_prefix(w: Workload, b: int, g: int, t_end: int) -> dict:
    """B and C of group g, batch row b, tokens [0, t_end), as bf16 bits [T,N]."""
    L, N, G = w.seqlen, w.dstate, w.ngroups
    t = np.arange(t_end, dtype=np.uint64)[:, None]
    bi = ((np.uint64(b) * np.uint64(L) + t) * np.uint64(G) + np.uint64(g)) * np.uint64(N) \
        + np.arange(N, dtype=np.uint64)[None, :]
    sd = 1.0 / math.sqrt(N)
    Bv = rng.normal(rng.stream_key(w.seed, rng.STREAM_B), bi) * sd
    Cv = rng.normal(rng.stream_key(w.seed, rng.STREAM_C), bi) * sd
    return {"B": rng.f32_to_bf16_bits(Bv.astype(np.float32)),
            "C": rng.f32_to_bf16_bits(Cv.astype(np.float32))}


def prefix_inputs(w: Workload) -> dict:
    """The calibration prefix: the first min(calib_prefix, L) tokens of every batch row."""
    T = min(w.calib_prefix, w.seqlen)
    # Flat indices depend on the full length L, so each row's prefix is
    # regenerated through the chain and group helpers.
    Bt, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    x = np.empty((Bt, T, H, P), dtype=np.uint16)
    dt = np.empty((Bt, T, H), dtype=np.float32)
    Bm = np.empty((Bt, T, G, N), dtype=np.uint16)
    Cm = np.empty((Bt, T, G, N), dtype=np.uint16)
    for b in range(Bt):
        for h in range(H):
            ch = make_chain(w, b, h, T)
            x[b, :, h, :] = ch["x"]
            dt[b, :, h] = ch["dt"]
        for g in range(G):
            gp = make_group_prefix(w, b, g, T)
            Bm[b, :, g, :] = gp["B"]
            Cm[b, :, g, :] = gp["C"]
    hp = head_params(w)
    return {"x": x, "dt": dt, "A": hp["A"], "B": Bm, "C": Cm, "D": hp["D"]}


def as_float(bits: np.ndarray) -> np.ndarray:
    """float64 values of bf16 bit patterns."""
    return rng.bf16_bits_to_f32(bits).astype(np.float64)
