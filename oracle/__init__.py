"""CPU oracle for the selective mixed-precision attention forward (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may
import this package.  The product path (``precision_attention_block_b200``)
never does, and it shares no code with the C file here.

The arithmetic lives in ``thrift_oracle.c`` (plain C, float64, IEEE FP32 where
the NVFP4 codec is defined on FP32 values); this module only compiles it with
gcc and marshals numpy arrays through ctypes.  Each function cites the passage
of the ThriftAttention technical summary ("Methodologie") that it follows.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "thrift_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
P_LEVEL1 = 2688.0  # 6 * 448: largest E2M1 value times largest E4M3 value

_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_int = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fused multiply-add, no fast-math)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call([
                "gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                "-pthread", _SRC, "-o", tmp, "-lm"])
            os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.orc_half_to_double.restype = ctypes.c_double
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_encode_array.argtypes = [_f32p, _i64, _u8p]
        L.orc_e4m3_encode_array.argtypes = [_f32p, _i64, _u8p]
        L.orc_double_to_half_array.argtypes = [_f64p, _i64, _u16p]
        L.orc_quantize_nvfp4.restype = ctypes.c_float
        L.orc_quantize_nvfp4.argtypes = [_u16p, _i64, _i32, _i32, _i32, _u8p, _u8p]
        L.orc_quantize_nvfp4_scaled.argtypes = [_u16p, _i64, _i32, _i32, _i32, ctypes.c_float, _u8p, _u8p]
        L.orc_block_scores.argtypes = [_u16p, _u16p] + [_int] * 8 + [_f64p]
        L.orc_block_scores_qk.argtypes = [_u16p, _u16p] + [_int] * 10 + [_f64p]
        L.orc_topk_count.restype = _i64
        L.orc_topk_count.argtypes = [_i64, _int, _int]
        L.orc_select.argtypes = [_f64p, _i64, _i64, _int, _int, _u8p, _f64p, _i64p]
        L.orc_pair_valid.restype = _int
        L.orc_pair_valid.argtypes = [_int] * 5
        L.orc_tile_pq.restype = _int
        L.orc_tile_pq.argtypes = [_f64p, _int, _int, ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(ctypes.c_double), _f64p]
        L.orc_attn.argtypes = (
            [_u16p, _u16p, _u16p, _u8p, _u8p, ctypes.c_float, _u8p, _u8p, ctypes.c_float,
             _u8p, _u8p, ctypes.c_float, _u8p] + [_int] * 8 + [ctypes.c_float, _i32p, _int, _int,
             ctypes.c_void_p, _u16p, _f32p, ctypes.c_void_p, _int])
        L.orc_attn_qk.argtypes = (
            [_u16p, _u16p, _u16p, _u8p, _u8p, ctypes.c_float, _u8p, _u8p, ctypes.c_float,
             _u8p, _u8p, ctypes.c_float, _u8p] + [_int] * 9 + [ctypes.c_float, _int, _int, _i32p, _int, _int,
             ctypes.c_void_p, _u16p, _f32p, ctypes.c_void_p, _int])
        L.orc_tile_scores.argtypes = (
            [_u16p, _u16p, _u8p, _u8p, ctypes.c_float, _u8p, _u8p, ctypes.c_float] + [_int] * 8
            + [ctypes.c_float] + [_int] * 5 + [_f64p])
        _lib = L
    return _lib


def _u16(x: np.ndarray) -> np.ndarray:
    assert x.dtype == np.float16
    return np.ascontiguousarray(x).view(np.uint16)


# --------------------------------------------------------------- codecs

def e2m1_encode(x) -> np.ndarray:
    """FP4 E2M1 code of each FP32 value: nearest of {0,.5,1,1.5,2,3,4,6}, ties to the
    even code, saturating, sign kept (NVFP4 element format on the ThriftAttention pages,
    "FP4-pad")."""
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    out = np.empty(x.size, np.uint8)
    lib().orc_e2m1_encode_array(x, x.size, out)
    return out


def e2m1_decode(codes) -> np.ndarray:
    grid = np.array(E2M1_GRID + tuple(-g for g in E2M1_GRID), np.float64)
    return grid[np.asarray(codes, np.uint8) & 15]


def e4m3_encode(x) -> np.ndarray:
    """FP8 E4M3 (fn) code of each non-negative FP32 value, round to nearest even, saturating at 448."""
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    out = np.empty(x.size, np.uint8)
    lib().orc_e4m3_encode_array(x, x.size, out)
    return out


def e4m3_decode(codes) -> np.ndarray:
    L = lib()
    table = np.array([L.orc_e4m3_decode(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, np.uint8)]


def half_to_double(h) -> np.ndarray:
    L = lib()
    table = np.array([L.orc_half_to_double(c) for c in range(65536)], np.float64)
    return table[np.asarray(h, np.uint16)]


def double_to_half(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64).reshape(-1)
    out = np.empty(x.size, np.uint16)
    lib().orc_double_to_half_array(x, x.size, out)
    return out


# --------------------------------------------------------------- NVFP4

class NVFP4:
    """Oracle NVFP4 tensor: codes (E2M1 nibbles), scales (E4M3 bytes), tensor scale (FP32)."""

    def __init__(self, codes, scales, tensor_scale, group_axis):
        self.codes, self.scales = codes, scales
        self.tensor_scale = np.float32(tensor_scale)
        self.group_axis = group_axis


def quantize_nvfp4(x: np.ndarray, group_axis: int, tensor_scale=None) -> NVFP4:
    """NVFP4 quantisation of x [.., N, d] (ThriftAttention "FP4-pad": NVFP4 microscaling,
    E2M1 values, one E4M3 scale per 16 elements, one FP32 tensor scale).
    group_axis 0: groups along d, codes [.., N, d/2]; 1: groups along N, codes [.., d, N/2].
    tensor_scale: a given FP32 tensor scale (reading R-append: a cache encodes with the scale it
    was built with); None: the tensor's own amax / 2688."""
    *lead, N, d = x.shape
    outer = int(np.prod(lead)) if lead else 1
    if group_axis == 0:
        codes = np.empty((*lead, N, d // 2), np.uint8)
        scales = np.empty((*lead, N, d // 16), np.uint8)
    else:
        codes = np.empty((*lead, d, N // 2), np.uint8)
        scales = np.empty((*lead, d, N // 16), np.uint8)
    if tensor_scale is None:
        st = lib().orc_quantize_nvfp4(_u16(x).reshape(-1), outer, N, d, group_axis,
                                      codes.reshape(-1), scales.reshape(-1))
    else:
        st = np.float32(tensor_scale)
        lib().orc_quantize_nvfp4_scaled(_u16(x).reshape(-1), outer, N, d, group_axis, st,
                                        codes.reshape(-1), scales.reshape(-1))
    return NVFP4(codes, scales, st, group_axis)


def dequantize_nvfp4(t: NVFP4) -> np.ndarray:
    """Element values code * s_b * s_t in float64, in the codes' own layout (nibbles unpacked)."""
    lo = t.codes & 15
    hi = t.codes >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(*t.codes.shape[:-1], t.codes.shape[-1] * 2)
    sb = np.repeat(e4m3_decode(t.scales), 16, axis=-1)
    return e2m1_decode(codes) * sb * np.float64(t.tensor_scale)


# --------------------------------------------------------------- selection

def block_scores(q: np.ndarray, k: np.ndarray, w) -> np.ndarray:
    """S^_ij = qbar_i . kbar_j (ThriftAttention "Heuristische Blokkenselectie"), float64
    [B, Hq, nQb, nKb], -inf for causal-invalid pairs."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    out = np.empty((B, Hq, N // w.block_q, N // w.block_k), np.float64)
    lib().orc_block_scores(_u16(q).reshape(-1), _u16(k).reshape(-1), B, Hq, Hkv, N, d, w.block_q,
                           w.block_k, int(w.causal), out.reshape(-1))
    return out


def topk_count(n_valid: int, topk_abs: int, topk_bp: int) -> int:
    return int(lib().orc_topk_count(n_valid, topk_abs, topk_bp))


def select(scores: np.ndarray, w):
    """Top-k pairs per (batch, query head) over the valid pairs, ties to the smaller flat
    index.  Returns (sel uint8 [B,Hq,nQb,nKb], kth score per head, k per head)."""
    B, Hq, nqb, nkb = scores.shape
    heads = B * Hq
    sel = np.empty(scores.shape, np.uint8)
    kth = np.empty(heads, np.float64)
    kc = np.empty(heads, np.int64)
    lib().orc_select(np.ascontiguousarray(scores).reshape(-1), heads, nqb * nkb, w.topk_abs, w.topk_bp,
                     sel.reshape(-1), kth, kc)
    return sel, kth.reshape(B, Hq), kc.reshape(B, Hq)


# --------------------------------------------------------------- attention

def softmax_scale(d: int) -> np.float32:
    """Default tau = 1/sqrt(d), rounded to FP32 (the value the kernels receive)."""
    return np.float32(1.0) / np.sqrt(np.float32(d))


def tile_pq(S: np.ndarray, fp16: bool):
    """Quantised probabilities of one row of one key block (two-level scheme, reading R1).
    Returns (M, sumP, Pq) or None when every entry is masked (-inf)."""
    S = np.ascontiguousarray(S, np.float64)
    Pq = np.empty(S.size, np.float64)
    M = ctypes.c_double()
    sp = ctypes.c_double()
    ok = lib().orc_tile_pq(S, S.size, int(fp16), ctypes.byref(M), ctypes.byref(sp), Pq)
    return (M.value, sp.value, Pq) if ok else None


def tile_scores(q, k, q4: NVFP4, k4: NVFP4, w, tau, b, h, i, j, fp16: bool) -> np.ndarray:
    B, Hq, N, d = q.shape
    S = np.empty((w.block_q, w.block_k), np.float64)
    lib().orc_tile_scores(_u16(q).reshape(-1), _u16(k).reshape(-1), q4.codes.reshape(-1),
                          q4.scales.reshape(-1), q4.tensor_scale, k4.codes.reshape(-1),
                          k4.scales.reshape(-1), k4.tensor_scale, B, Hq, k.shape[1], N, d,
                          w.block_q, w.block_k, int(w.causal), np.float32(tau), b, h, i, j,
                          int(fp16), S.reshape(-1))
    return S


def attn(q, k, v, q4: NVFP4, k4: NVFP4, v4: NVFP4, sel, w, tau=None, units=None, online=False,
         order=None, want_f64=False, threads=None):
    """Attention forward (ThriftAttention "Gemengd-Precisie Berekening & Samenvoeging"):
    FP16 for the selected pairs, NVFP4 for the other valid pairs, one softmax over both.

    units: list of (b, h, i) query-block units to compute (default: all).  Returns
    (out fp16 [B,Hq,N,d], lse f32 [B,Hq,N], out64 or None); rows outside the units are 0."""
    B, Hq, N, d = q.shape
    if tau is None:
        tau = softmax_scale(d)
    if units is None:
        units = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(N // w.block_q)]
    u = np.ascontiguousarray(np.array(units, np.int32).reshape(-1))
    out = np.zeros((B, Hq, N, d), np.uint16)
    lse = np.zeros((B, Hq, N), np.float32)
    out64 = np.zeros((B, Hq, N, d), np.float64) if want_f64 else None
    order_arr = None if order is None else np.ascontiguousarray(np.array(order, np.int32))
    if threads is None:
        threads = os.cpu_count() or 1
    lib().orc_attn(_u16(q).reshape(-1), _u16(k).reshape(-1), _u16(v).reshape(-1),
                   q4.codes.reshape(-1), q4.scales.reshape(-1), q4.tensor_scale,
                   k4.codes.reshape(-1), k4.scales.reshape(-1), k4.tensor_scale,
                   v4.codes.reshape(-1), v4.scales.reshape(-1), v4.tensor_scale,
                   np.ascontiguousarray(sel, np.uint8).reshape(-1),
                   B, Hq, k.shape[1], N, d, w.block_q, w.block_k, int(w.causal), np.float32(tau),
                   u, len(units), int(online),
                   None if order_arr is None else order_arr.ctypes.data,
                   out.reshape(-1), lse.reshape(-1),
                   None if out64 is None else out64.ctypes.data, int(threads))
    return out.view(np.float16), lse, out64


def attn_r2(q, k, v, q4: NVFP4, k4: NVFP4, v4: NVFP4, sel, w, tau=None, units=None, want_f64=False,
            threads=None):
    """Attention forward under reading R2 of the two-level P quantisation (the running maximum,
    in the fused kernel's visiting order -- NVFP4 key blocks ascending, then FP16 ones -- as the
    first level).  Same arguments and return values as `attn`."""
    B, Hq, N, d = q.shape
    if tau is None:
        tau = softmax_scale(d)
    if units is None:
        units = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(N // w.block_q)]
    u = np.ascontiguousarray(np.array(units, np.int32).reshape(-1))
    out = np.zeros((B, Hq, N, d), np.uint16)
    lse = np.zeros((B, Hq, N), np.float32)
    out64 = np.zeros((B, Hq, N, d), np.float64) if want_f64 else None
    if threads is None:
        threads = os.cpu_count() or 1
    lib().orc_attn(_u16(q).reshape(-1), _u16(k).reshape(-1), _u16(v).reshape(-1),
                   q4.codes.reshape(-1), q4.scales.reshape(-1), q4.tensor_scale,
                   k4.codes.reshape(-1), k4.scales.reshape(-1), k4.tensor_scale,
                   v4.codes.reshape(-1), v4.scales.reshape(-1), v4.tensor_scale,
                   np.ascontiguousarray(sel, np.uint8).reshape(-1),
                   B, Hq, k.shape[1], N, d, w.block_q, w.block_k, int(w.causal), np.float32(tau),
                   u, len(units), 2, None, out.reshape(-1), lse.reshape(-1),
                   None if out64 is None else out64.ctypes.data, int(threads))
    return out.view(np.float16), lse, out64


def attn_sparse(q, k, v, sel, w, tau=None, units=None, want_f64=False, threads=None):
    """Compute-matched sparse variant (reading R-sparse): only the selected pairs, in FP16; every
    other pair dropped.  A row left with no key gets output 0 and lse -inf.  Same return values as
    `attn`; no NVFP4 tensor is used."""
    B, Hq, N, d = q.shape
    if tau is None:
        tau = softmax_scale(d)
    if units is None:
        units = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(N // w.block_q)]
    u = np.ascontiguousarray(np.array(units, np.int32).reshape(-1))
    out = np.zeros((B, Hq, N, d), np.uint16)
    lse = np.zeros((B, Hq, N), np.float32)
    out64 = np.zeros((B, Hq, N, d), np.float64) if want_f64 else None
    if threads is None:
        threads = os.cpu_count() or 1
    z8 = np.zeros(1, np.uint8)
    lib().orc_attn_qk(_u16(q).reshape(-1), _u16(k).reshape(-1), _u16(v).reshape(-1),
                      z8, z8, np.float32(1), z8, z8, np.float32(1), z8, z8, np.float32(1),
                      np.ascontiguousarray(sel, np.uint8).reshape(-1),
                      B, Hq, k.shape[1], N, N, d, w.block_q, w.block_k, int(w.causal), np.float32(tau), 1, N,
                      u, len(units), 0, None, out.reshape(-1), lse.reshape(-1),
                      None if out64 is None else out64.ctypes.data, int(threads))
    return out.view(np.float16), lse, out64


def quantize_all(q, k, v):
    """The three NVFP4 tensors of one problem: Q, K grouped along d; V grouped along tokens."""
    return quantize_nvfp4(q, 0), quantize_nvfp4(k, 0), quantize_nvfp4(v, 1)


def forward(w, q, k, v, units=None, want_f64=False, threads=None):
    """The whole path for one workload: quantise, score, select, attend.  Returns a dict."""
    q4, k4, v4 = quantize_all(q, k, v)
    scores = block_scores(q, k, w)
    sel, kth, kc = select(scores, w)
    out, lse, out64 = attn(q, k, v, q4, k4, v4, sel, w, units=units, want_f64=want_f64,
                           threads=threads)
    return dict(q4=q4, k4=k4, v4=v4, scores=scores, sel=sel, kth=kth, k=kc, out=out, lse=lse,
                out64=out64)


# ------------------------------------------------------------------ decode

def decode_block_scores(q: np.ndarray, k: np.ndarray, block_k: int, causal: bool, n_valid=None) -> np.ndarray:
    """Decode selection scores (reading R-decode): the Nq query rows of each (batch, query head)
    form one query block; S^_j = qbar . kbar_j over the key blocks of the cache, float64
    [B, Hq, 1, Nk/block_k].  n_valid: the cache's valid length (reading R-append; default Nk):
    blocks at or past it are -inf and a partly filled block averages the keys it holds."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    nv = Nk if n_valid is None else int(n_valid)
    out = np.empty((B, Hq, 1, Nk // block_k), np.float64)
    lib().orc_block_scores_qk(_u16(q).reshape(-1), _u16(k).reshape(-1), B, Hq, Hkv, Nq, Nk, d, Nq,
                              block_k, int(causal), nv, out.reshape(-1))
    return out


def decode_attn(q, k, v, q4: NVFP4, k4: NVFP4, v4: NVFP4, sel, block_k: int, causal: bool, tau=None,
                want_f64=False, threads=None, sparse=False, n_valid=None):
    """Decode attention (reading R-decode): the Nq rows of q [B,Hq,Nq,d] are the newest
    positions of the cache k, v [B,Hkv,Nk,d]; sel [B,Hq,1,Nk/block_k] marks the FP16 key blocks.
    The same mixed-precision computation as `attn` (sparse: only the selected blocks, reading
    R-sparse).  n_valid: the cache's valid length (default Nk): keys at or past it are masked.
    Returns (out fp16 [B,Hq,Nq,d], lse f32 [B,Hq,Nq], out64 or None)."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    nv = Nk if n_valid is None else int(n_valid)
    if tau is None:
        tau = softmax_scale(d)
    units = [(b, h, 0) for b in range(B) for h in range(Hq)]
    u = np.ascontiguousarray(np.array(units, np.int32).reshape(-1))
    out = np.zeros((B, Hq, Nq, d), np.uint16)
    lse = np.zeros((B, Hq, Nq), np.float32)
    out64 = np.zeros((B, Hq, Nq, d), np.float64) if want_f64 else None
    if threads is None:
        threads = os.cpu_count() or 1
    lib().orc_attn_qk(_u16(q).reshape(-1), _u16(k).reshape(-1), _u16(v).reshape(-1),
                      q4.codes.reshape(-1), q4.scales.reshape(-1), q4.tensor_scale,
                      k4.codes.reshape(-1), k4.scales.reshape(-1), k4.tensor_scale,
                      v4.codes.reshape(-1), v4.scales.reshape(-1), v4.tensor_scale,
                      np.ascontiguousarray(sel, np.uint8).reshape(-1),
                      B, Hq, Hkv, Nq, Nk, d, Nq, block_k, int(causal), np.float32(tau), int(sparse), nv,
                      u, len(units), 0, None, out.reshape(-1), lse.reshape(-1),
                      None if out64 is None else out64.ctypes.data, int(threads))
    return out.view(np.float16), lse, out64


def decode_forward(w, q, k, v, k4=None, v4=None, want_f64=False, threads=None, n_valid=None):
    """One decode step: quantise the query rows, score and select key blocks, attend.
    k4, v4: the cache's NVFP4 copies (computed here when None).  n_valid: the cache's valid
    length (default: all of k).  Returns a dict."""
    q4 = quantize_nvfp4(q, 0)
    if k4 is None:
        k4 = quantize_nvfp4(k, 0)
    if v4 is None:
        v4 = quantize_nvfp4(v, 1)
    scores = decode_block_scores(q, k, w.block_k, w.causal, n_valid)
    sel, kth, kc = select(scores, w)
    out, lse, out64 = decode_attn(q, k, v, q4, k4, v4, sel, w.block_k, w.causal, want_f64=want_f64,
                                  threads=threads, n_valid=n_valid)
    return dict(q4=q4, k4=k4, v4=v4, scores=scores, sel=sel, kth=kth, k=kc, out=out, lse=lse,
                out64=out64)
