"""Seeded synthetic workloads for the selective mixed-precision attention forward.

This module is shared by the CUDA path's tests and bench and by the CPU
oracle's tests.  It holds no arithmetic of the method itself: only the
problem shapes and a counter-based random generator that turns a seed into
FP16 Q, K, V tensors.

Shapes and value distributions stand in for the workloads the ThriftAttention
pages evaluate on (long-context LLM prefill at 8k-131k context, "Resultaten"
section; diffusion-style attention on the Attn-QAT page, "Ergebnisse").  No
dataset is read: every tensor is drawn from the generator below.

Generator (stated so that any implementation can reproduce it bit for bit):

* splitmix64: state_i = key + (i + 1) * 0x9E3779B97F4A7C15 (mod 2^64),
  mix(z) = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
  z *= 0x94D049BB133111EB; z ^= z >> 31.
* key(seed, stream) = mix(seed * 2^20 + stream).
* uniform(i) = (mix(state_i) >> 11) * 2^-53 in [0, 1).
* normal(i) = sqrt(-2 ln(1 - uniform(2i))) * cos(2 pi uniform(2i + 1)),
  evaluated in float64 (libm) and rounded once to FP16 (round to nearest
  even) after the per-distribution transform.

The loops run in the small C helper ``_gen.c`` (compiled with gcc on first
use); numpy does the FP16 rounding.
"""

from __future__ import annotations

import dataclasses
import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_CHUNK = 1 << 22
_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "_gen.c")
_LIB = os.path.join(_HERE, "libwlgen.so")
_lock = threading.Lock()
_lib = None

# Stream ids: one independent sequence per tensor and per random ingredient.
STREAM_Q, STREAM_K, STREAM_V = 1, 2, 3
STREAM_KBIAS = 4
STREAM_QOUT, STREAM_KOUT, STREAM_VOUT = 5, 6, 7
STREAM_QROW, STREAM_KROW, STREAM_VROW = 8, 9, 10
STREAM_QDEC = 11  # the query rows of a decode step

_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_u64 = ctypes.c_uint64
_i64 = ctypes.c_int64


def _gen():
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
                tmp = _LIB + f".tmp{os.getpid()}"
                subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", _SRC,
                                       "-o", tmp, "-lm"])
                os.replace(tmp, _LIB)
            L = ctypes.CDLL(_LIB)
            L.wl_key.restype = _u64
            L.wl_key.argtypes = [_u64, _u64]
            L.wl_uniform.argtypes = [_u64, _i64, _i64, _f64p]
            L.wl_normal.argtypes = [_u64, _i64, _i64, _f64p]
            L.wl_fill.argtypes = [ctypes.c_int, _u64, _u64, _i64, _i64, ctypes.c_void_p, _i64, _i64,
                                  _f64p]
            _lib = L
    return _lib


def build() -> None:
    _gen()


def stream_key(seed: int, stream: int) -> int:
    return int(_gen().wl_key(seed, stream))


def uniform(key: int, start: int, count: int) -> np.ndarray:
    """uniform(i) for i in [start, start + count), float64 in [0, 1)."""
    out = np.empty(count, np.float64)
    _gen().wl_uniform(key, start, count, out)
    return out


def normal(key: int, start: int, count: int) -> np.ndarray:
    """normal(i) for i in [start, start + count), float64."""
    out = np.empty(count, np.float64)
    _gen().wl_normal(key, start, count, out)
    return out


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, selection granularity and budget."""

    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    block_q: int
    block_k: int
    topk_abs: int  # >= 0: absolute k per head; -1: use topk_bp
    topk_bp: int   # budget in basis points of the valid pairs
    dist: str      # "normal" | "heavy_bias" | "student_t" | "row_lognormal"
    n_query: int = 0  # > 0: a decode step, n_query query rows against a cache of N keys

    @property
    def seed(self) -> int:
        return 20260000 + self.index

    @property
    def n_qb(self) -> int:
        return self.N // self.block_q

    @property
    def n_kb(self) -> int:
        return self.N // self.block_k

    @property
    def is_decode(self) -> bool:
        return self.n_query > 0

    def with_budget(self, topk_bp: int, topk_abs: int = -1) -> "Workload":
        return dataclasses.replace(self, topk_bp=topk_bp, topk_abs=topk_abs)

    def with_shape(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 2, 2, 512, 64, False, 64, 64, 4, 0, "normal"),
    "n4k": Workload("n4k", 1, 1, 8, 8, 4096, 128, False, 128, 64, -1, 500, "heavy_bias"),
    "prefill32k": Workload("prefill32k", 2, 1, 32, 8, 32768, 128, True, 128, 64, -1, 500,
                           "heavy_bias"),
    # same distribution and blocking as the 32K prefill at half the length: a profiling size
    "prefill16k": Workload("prefill16k", 5, 1, 32, 8, 16384, 128, True, 128, 64, -1, 500,
                           "heavy_bias"),
    # the 32K prefill with "inputs as in config 1" read 1-based (the 4K workload's plain N(0,1)
    # inputs, no heavy tail or key bias) instead of 0-based: an extra, labelled row
    "prefill32k_plain": Workload("prefill32k_plain", 9, 1, 32, 8, 32768, 128, True, 128, 64, -1, 500,
                                 "normal"),
    "long131k": Workload("long131k", 3, 1, 32, 8, 131072, 128, True, 128, 128, -1, 200,
                         "student_t"),
    "diffusion": Workload("diffusion", 4, 2, 24, 24, 16384, 64, False, 128, 64, -1, 500,
                          "row_lognormal"),
    # decode steps: n_query new query rows (the newest positions) against a cache of N keys;
    # block_q is unused (the query rows form one block)
    "decode_tiny": Workload("decode_tiny", 6, 1, 4, 2, 1024, 64, True, 128, 64, -1, 1000, "normal",
                            n_query=2),
    "decode32k": Workload("decode32k", 7, 1, 32, 8, 32768, 128, True, 128, 64, -1, 500, "heavy_bias",
                          n_query=1),
    "decode131k": Workload("decode131k", 8, 1, 32, 8, 131072, 128, True, 128, 128, -1, 200,
                           "student_t", n_query=1),
}
DIFFUSION_BUDGETS_BP = (0, 100, 500, 2000, 10000)


def _fill(out: np.ndarray, dist: int, key: int, key2: int, vec, N: int, d: int) -> None:
    flat = out.reshape(-1)
    n = flat.size
    vec = None if vec is None else np.ascontiguousarray(vec, np.float64)
    L = _gen()

    def work(s):
        c = min(_CHUNK, n - s)
        buf = np.empty(c, np.float64)
        L.wl_fill(dist, key, key2, s, c, None if vec is None else vec.ctypes.data, N, d, buf)
        flat[s:s + c] = buf.astype(np.float16)

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(work, range(0, n, _CHUNK)))


def _tensor(w: Workload, stream: int, shape, which: str) -> np.ndarray:
    """One FP16 tensor of the workload's distribution, shape [B, H, N, d]."""
    key = stream_key(w.seed, stream)
    out = np.empty(shape, dtype=np.float16)
    B, H, N, d = shape
    if w.dist == "normal":
        _fill(out, 0, key, 0, None, N, d)
    elif w.dist == "heavy_bias":
        # N(0,1); each entry independently x20 with probability 0.01; K also gets one
        # fixed per-channel bias b ~ N(0, sigma=2) per (batch, kv head), added to every token.
        okey = stream_key(w.seed, {"q": STREAM_QOUT, "k": STREAM_KOUT, "v": STREAM_VOUT}[which])
        bias = None
        if which == "k":
            bias = 2.0 * normal(stream_key(w.seed, STREAM_KBIAS), 0, B * H * d)
        _fill(out, 1, key, okey, bias, N, d)
    elif w.dist == "student_t":
        # Student-t with nu = 3: z0 / sqrt((z1^2 + z2^2 + z3^2) / 3), clipped at |x| <= 60.
        _fill(out, 2, key, 0, None, N, d)
    elif w.dist == "row_lognormal":
        # N(0,1) times one LogNormal(0, sigma=0.5) factor per token row.
        rkey = stream_key(w.seed, {"q": STREAM_QROW, "k": STREAM_KROW, "v": STREAM_VROW}[which])
        rowscale = np.exp(0.5 * normal(rkey, 0, B * H * N))
        _fill(out, 3, key, 0, rowscale, N, d)
    else:
        raise ValueError(w.dist)
    return out


def make_qkv(w: Workload):
    """Seeded FP16 Q [B,Hq,N,d] (decode: [B,Hq,n_query,d]), K [B,Hkv,N,d], V [B,Hkv,N,d] as
    numpy arrays."""
    if w.is_decode:
        q = _tensor(w, STREAM_QDEC, (w.B, w.Hq, w.n_query, w.d), "q")
    else:
        q = _tensor(w, STREAM_Q, (w.B, w.Hq, w.N, w.d), "q")
    k = _tensor(w, STREAM_K, (w.B, w.Hkv, w.N, w.d), "k")
    v = _tensor(w, STREAM_V, (w.B, w.Hkv, w.N, w.d), "v")
    return q, k, v


def sample_units(w: Workload, count: int, seed_offset: int = 0):
    """A seeded, stratified sample of (b, q-head, query-block) units.

    The query blocks are spread evenly over [0, n_qb) (so causal rows of every
    length appear) and always include the first and the last block; heads and
    batches are drawn from the generator.
    """
    key = stream_key(w.seed + 7919 * (seed_offset + 1), 99)
    u = uniform(key, 0, 2 * count)
    nqb = w.n_qb
    units = set()
    for t in range(count):
        if t == 0:
            i = 0
        elif t == 1:
            i = nqb - 1
        else:
            i = min(nqb - 1, int((t - 2 + u[2 * t]) * nqb / max(1, count - 2)))
        bh = int(u[2 * t + 1] * w.B * w.Hq)
        units.add((bh // w.Hq, bh % w.Hq, i))
    return sorted(units)
