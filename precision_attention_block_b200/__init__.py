"""B200-native selective mixed-precision attention forward (NVFP4 + FP16).

The method is the one the ThriftAttention technical summary describes ("Methodologie"):
block-mean importance scores S^_ij = qbar_i . kbar_j, the top-k block pairs per head in FP16,
every other pair in NVFP4, one online softmax over both.  All arithmetic runs in libthrift's
sm_100a kernels; this module only allocates device memory with PyTorch, picks the current
CUDA stream and passes pointers through the C ABI.

    cfg = Config(B=1, Hq=32, Hkv=8, N=32768, d=128, causal=True, block_q=128, block_k=64,
                 topk_bp=500)
    out, lse = attn_fwd_auto(q, k, v, cfg)          # quantise + select + attend
"""

from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from . import _lib
from ._lib import ThriftError, check, load

__all__ = ["Config", "NVFP4Tensor", "Selection", "Workspace", "quantize_nvfp4", "quantize_qkv",
           "block_select", "attn_fwd", "attn_fwd_auto", "DecodeConfig", "KVCache", "kv_block_means",
           "decode_select", "decode_attn", "decode_fwd", "attn_fwd_sparse", "decode_attn_sparse",
           "device_status", "reset_device_status",
           "ThriftError", "load"]


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@dataclasses.dataclass
class Config:
    """Problem description (thrift_cfg)."""

    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    block_q: int = 128
    block_k: int = 64
    topk_abs: int = -1
    topk_bp: int = 500
    softmax_scale: float = 0.0

    @classmethod
    def from_workload(cls, w) -> "Config":
        return cls(w.B, w.Hq, w.Hkv, w.N, w.d, bool(w.causal), w.block_q, w.block_k, w.topk_abs,
                   w.topk_bp)

    def c(self) -> _lib.CCfg:
        return _lib.CCfg(self.B, self.Hq, self.Hkv, self.N, self.d, int(self.causal), self.block_q,
                         self.block_k, self.topk_abs, self.topk_bp, self.softmax_scale)

    @property
    def n_qb(self) -> int:
        return self.N // self.block_q

    @property
    def n_kb(self) -> int:
        return self.N // self.block_k

    @property
    def mask_words(self) -> int:
        return (self.n_kb + 31) // 32


@dataclasses.dataclass
class NVFP4Tensor:
    """Device NVFP4 tensor (thrift_nvfp4): E2M1 codes, E4M3 scales (canonical and MMA layout),
    FP32 tensor scale."""

    codes: torch.Tensor
    scales: torch.Tensor
    scales_mma: torch.Tensor
    tensor_scale: torch.Tensor
    group_axis: int

    @classmethod
    def empty(cls, outer: int, N: int, d: int, group_axis: int, device) -> "NVFP4Tensor":
        L = load()
        if group_axis == 0:
            cshape, sshape = (outer, N, d // 2), (outer, N, d // 16)
        else:
            cshape, sshape = (outer, d, N // 2), (outer, d, N // 16)
        mma = int(L.thrift_nvfp4_scales_mma_bytes(outer, N, d, group_axis))
        u8 = dict(dtype=torch.uint8, device=device)
        return cls(torch.empty(cshape, **u8), torch.empty(sshape, **u8), torch.empty(mma, **u8),
                   torch.empty(1, dtype=torch.float32, device=device), group_axis)

    def c(self) -> _lib.CNVFP4:
        return _lib.CNVFP4(self.codes.data_ptr(), self.scales.data_ptr(), self.scales_mma.data_ptr(),
                           self.tensor_scale.data_ptr(), self.group_axis)


@dataclasses.dataclass
class Selection:
    """Output of block_select: FP16-pair bitmask, per-row counts and sorted lists, scores."""

    mask: torch.Tensor
    counts: torch.Tensor
    lists: torch.Tensor
    scores: Optional[torch.Tensor]


class Workspace:
    """Caller-owned device scratch (256-byte aligned).  The first 256 bytes hold the device
    status word, zeroed on creation."""

    def __init__(self, nbytes: int, device):
        self.buf = torch.zeros(max(int(nbytes), 256) + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + max(int(nbytes), 256)]
        self.nbytes = self.view.numel()

    @property
    def ptr(self):
        return ctypes.c_void_p(self.view.data_ptr())

    @classmethod
    def for_config(cls, cfg: Config, device, auto: bool = False) -> "Workspace":
        L = load()
        c = cfg.c()
        n = L.thrift_auto_workspace_bytes(ctypes.byref(c)) if auto else L.thrift_workspace_bytes(ctypes.byref(c))
        if n == 0:
            raise ThriftError(_lib.THRIFT_ERR_UNSUPPORTED, "workspace size")
        return cls(n, device)


def _strides(t: Optional[torch.Tensor]):
    """thrift_strides of a [B, H, N, d] view (None when dense): a token-major [B, N, H, d] tensor
    passed as t.transpose(1, 2) reaches the kernels without a copy."""
    if t is None or t.is_contiguous():
        return None
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("strided tensors must be [B, H, N, d] views with contiguous d")
    # the stride of a dimension of size 1 is never used, and torch may report any value for it:
    # pass the dense layout's stride there (a valid multiple of 16 bytes for the tensor maps)
    B, H, N, d = t.shape
    dense = (H * N * d, N * d, d)
    sb, sh, sn = (dense[i] if t.shape[i] == 1 else t.stride(i) for i in range(3))
    return _lib.CStrides(sb, sh, sn)


def _sref(st):
    return None if st is None else ctypes.byref(st)


def quantize_nvfp4(x: torch.Tensor, group_axis: int, out: Optional[NVFP4Tensor] = None,
                   ws: Optional[Workspace] = None) -> NVFP4Tensor:
    """NVFP4 quantisation of an FP16 [.., N, d] CUDA tensor (thrift_quantize_nvfp4), or of a
    strided [B, H, N, d] view (thrift_quantize_nvfp4_strided)."""
    assert x.is_cuda and x.dtype == torch.float16
    *lead, N, d = x.shape
    outer = 1
    for s in lead:
        outer *= s
    if out is None:
        out = NVFP4Tensor.empty(outer, N, d, group_axis, x.device)
    if ws is None:
        ws = Workspace(256, x.device)
    c = out.c()
    st = _strides(x)
    if st is not None:
        check(load().thrift_quantize_nvfp4_strided(_ptr(x), ctypes.byref(st), x.shape[0], x.shape[1], N, d,
                                                   ctypes.byref(c), ws.ptr, ws.nbytes, _stream()),
              "thrift_quantize_nvfp4_strided")
        return out
    check(load().thrift_quantize_nvfp4(_ptr(x), outer, N, d, ctypes.byref(c), ws.ptr, ws.nbytes, _stream()),
          "thrift_quantize_nvfp4")
    return out


def quantize_qkv(q, k, v, ws: Optional[Workspace] = None):
    """Q, K grouped along d; V grouped along tokens."""
    return quantize_nvfp4(q, 0, ws=ws), quantize_nvfp4(k, 0, ws=ws), quantize_nvfp4(v, 1, ws=ws)


def block_select(q: torch.Tensor, k: torch.Tensor, cfg: Config, ws: Optional[Workspace] = None,
                 want_scores: bool = False, out: Optional[Selection] = None) -> Selection:
    """Block-mean scores and per-head top-k FP16 pairs (thrift_block_select)."""
    dev = q.device
    rows = cfg.B * cfg.Hq * cfg.n_qb
    if out is None:
        out = Selection(
            torch.empty((cfg.B, cfg.Hq, cfg.n_qb, cfg.mask_words), dtype=torch.int32, device=dev),
            torch.empty((cfg.B, cfg.Hq, cfg.n_qb), dtype=torch.int32, device=dev),
            torch.empty((cfg.B, cfg.Hq, cfg.n_qb, cfg.n_kb), dtype=torch.int16, device=dev),
            torch.empty((cfg.B, cfg.Hq, cfg.n_qb, cfg.n_kb), dtype=torch.float64, device=dev)
            if want_scores else None)
    assert out.counts.numel() == rows
    if ws is None:
        ws = Workspace.for_config(cfg, dev)
    c = cfg.c()
    qs, ks = _strides(q), _strides(k)
    if qs is not None or ks is not None:
        check(load().thrift_block_select_strided(_ptr(q), _sref(qs), _ptr(k), _sref(ks), ctypes.byref(c),
                                                 _ptr(out.mask), _ptr(out.counts), _ptr(out.lists),
                                                 _ptr(out.scores), ws.ptr, ws.nbytes, _stream()),
              "thrift_block_select_strided")
        return out
    check(load().thrift_block_select(_ptr(q), _ptr(k), ctypes.byref(c), _ptr(out.mask), _ptr(out.counts),
                                     _ptr(out.lists), _ptr(out.scores), ws.ptr, ws.nbytes, _stream()),
          "thrift_block_select")
    return out


def attn_fwd(q, k, v, q4: Optional[NVFP4Tensor], k4: Optional[NVFP4Tensor], v4: Optional[NVFP4Tensor],
             sel: Optional[Selection], cfg: Config, out: Optional[torch.Tensor] = None,
             lse: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None, want_lse: bool = True,
             running_max: bool = False):
    """Selective mixed-precision attention forward (thrift_attn_fwd).  Returns (out, lse).
    running_max: requantise P against the row's running maximum instead of each key block's own
    maximum (thrift_attn_fwd_running_max)."""
    ref = q if q is not None else q4.codes
    dev = ref.device
    if out is None:
        out = torch.empty((cfg.B, cfg.Hq, cfg.N, cfg.d), dtype=torch.float16, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)
    if ws is None:
        ws = Workspace(256, dev)
    c = cfg.c()
    n4 = [None if t is None else t.c() for t in (q4, k4, v4)]
    refs = [None if t is None else ctypes.byref(t) for t in n4]
    strided = [_strides(t) for t in (q, k, v, out)]
    if any(st is not None for st in strided):
        if running_max:
            raise ValueError("the running-maximum variant takes dense tensors")
        qs, ks, vs, os_ = strided
        check(load().thrift_attn_fwd_strided(_ptr(q), _sref(qs), _ptr(k), _sref(ks), _ptr(v), _sref(vs),
                                             refs[0], refs[1], refs[2], None if sel is None else _ptr(sel.mask),
                                             _ptr(out), _sref(os_), _ptr(lse), ctypes.byref(c), ws.ptr, ws.nbytes,
                                             _stream()), "thrift_attn_fwd_strided")
        return out, lse
    if running_max:
        check(load().thrift_attn_fwd_running_max(_ptr(q), _ptr(k), _ptr(v), refs[0], refs[1], refs[2],
                                                 None if sel is None else _ptr(sel.mask), _ptr(out), _ptr(lse),
                                                 ctypes.byref(c), ws.ptr, ws.nbytes, _stream()),
              "thrift_attn_fwd_running_max")
        return out, lse
    check(load().thrift_attn_fwd(_ptr(q), _ptr(k), _ptr(v), refs[0], refs[1], refs[2],
                                 None if sel is None else _ptr(sel.mask),
                                 None if sel is None else _ptr(sel.counts),
                                 None if sel is None else _ptr(sel.lists),
                                 _ptr(out), _ptr(lse), ctypes.byref(c), ws.ptr, ws.nbytes, _stream()),
          "thrift_attn_fwd")
    return out, lse


def attn_fwd_qat(q, k, v, q4: Optional[NVFP4Tensor], k4: Optional[NVFP4Tensor], v4: Optional[NVFP4Tensor],
                 sel: Optional[Selection], cfg: Config, out: Optional[torch.Tensor] = None,
                 out_hp: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 ws: Optional[Workspace] = None):
    """Attn-QAT forward variant (thrift_attn_fwd_qat): the FP16 output plus its FP32 copy O' before
    the FP16 rounding.  Returns (out, out_hp, lse)."""
    ref = q if q is not None else q4.codes
    dev = ref.device
    shape = (cfg.B, cfg.Hq, cfg.N, cfg.d)
    if out is None:
        out = torch.empty(shape, dtype=torch.float16, device=dev)
    if out_hp is None:
        out_hp = torch.empty(shape, dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)
    if ws is None:
        ws = Workspace(256, dev)
    c = cfg.c()
    n4 = [None if t is None else t.c() for t in (q4, k4, v4)]
    refs = [None if t is None else ctypes.byref(t) for t in n4]
    check(load().thrift_attn_fwd_qat(_ptr(q), _ptr(k), _ptr(v), refs[0], refs[1], refs[2],
                                     None if sel is None else _ptr(sel.mask), _ptr(out), _ptr(out_hp),
                                     _ptr(lse), ctypes.byref(c), ws.ptr, ws.nbytes, _stream()),
          "thrift_attn_fwd_qat")
    return out, out_hp, lse


def attn_fwd_sparse(q, k, v, sel: Selection, cfg: Config, out=None, lse=None, ws: Optional[Workspace] = None,
                    want_lse: bool = True):
    """Compute-matched sparse variant (thrift_attn_fwd_sparse): only the selected pairs, in FP16;
    rows left with no key get 0 and lse -inf.  Returns (out, lse)."""
    dev = q.device
    if out is None:
        out = torch.empty((cfg.B, cfg.Hq, cfg.N, cfg.d), dtype=torch.float16, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)
    if ws is None:
        ws = Workspace(256, dev)
    c = cfg.c()
    check(load().thrift_attn_fwd_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(sel.mask), _ptr(sel.counts),
                                        _ptr(sel.lists), _ptr(out), _ptr(lse), ctypes.byref(c), ws.ptr, ws.nbytes,
                                        _stream()), "thrift_attn_fwd_sparse")
    return out, lse


def attn_fwd_auto(q, k, v, cfg: Config, out=None, lse=None, ws: Optional[Workspace] = None,
                  want_lse: bool = True):
    """Quantise, select and attend in one call (thrift_attn_fwd_auto).  Returns (out, lse)."""
    dev = q.device
    if out is None:
        out = torch.empty((cfg.B, cfg.Hq, cfg.N, cfg.d), dtype=torch.float16, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)
    if ws is None:
        ws = Workspace.for_config(cfg, dev, auto=True)
    c = cfg.c()
    strided = [_strides(t) for t in (q, k, v, out)]
    if any(st is not None for st in strided):
        qs, ks, vs, os_ = strided
        check(load().thrift_attn_fwd_auto_strided(_ptr(q), _sref(qs), _ptr(k), _sref(ks), _ptr(v), _sref(vs),
                                                  _ptr(out), _sref(os_), _ptr(lse), ctypes.byref(c), ws.ptr,
                                                  ws.nbytes, _stream()), "thrift_attn_fwd_auto_strided")
        return out, lse
    check(load().thrift_attn_fwd_auto(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), ctypes.byref(c),
                                      ws.ptr, ws.nbytes, _stream()), "thrift_attn_fwd_auto")
    return out, lse


def attn_debug_dump(q, k, v, q4, k4, v4, sel, cfg: Config, entry: int, ws: Optional[Workspace] = None):
    """thrift_debug_attn_dump: (out, lse, dbg) with the raw S, PV operand row bytes and PV of one
    entry of the first unit of CTA 0."""
    ref = q if q is not None else q4.codes
    dev = ref.device
    out = torch.empty((cfg.B, cfg.Hq, cfg.N, cfg.d), dtype=torch.float16, device=dev)
    lse = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)
    dbg = torch.full((128 * cfg.block_k + 64 * cfg.block_k + 128 * cfg.d,), float("nan"),
                     dtype=torch.float32, device=dev)
    if ws is None:
        ws = Workspace(256, dev)
    c = cfg.c()
    n4 = [None if t is None else t.c() for t in (q4, k4, v4)]
    refs = [None if t is None else ctypes.byref(t) for t in n4]
    check(load().thrift_debug_attn_dump(_ptr(q), _ptr(k), _ptr(v), refs[0], refs[1], refs[2],
                                        None if sel is None else _ptr(sel.mask), _ptr(out), _ptr(lse),
                                        ctypes.byref(c), ws.ptr, ws.nbytes, _ptr(dbg), entry, _stream()),
          "thrift_debug_attn_dump")
    return out, lse, dbg


def pipe_rates(device=None):
    """Measured MUFU ex2 and FMA lanes per SM clock (thrift_debug_pipe_rates); synchronises."""
    dev = torch.device("cuda") if device is None else device
    L = load()
    ws = Workspace(L.thrift_debug_pipe_rates_ws_bytes(), dev)
    out = torch.zeros(2, dtype=torch.float64, device=dev)
    check(L.thrift_debug_pipe_rates(ws.ptr, ws.nbytes, _ptr(out), _stream()), "thrift_debug_pipe_rates")
    r = out.cpu().tolist()
    return {"mufu_ex2": r[0], "fma": r[1]}


def reset_device_status(ws: Workspace) -> None:
    check(load().thrift_reset_device_status(ws.ptr, _stream()), "thrift_reset_device_status")


def device_status(ws: Workspace) -> int:
    """The device status word (0 = no device-side error).  Synchronises the current stream."""
    v = ctypes.c_int32(0)
    check(load().thrift_get_device_status(ws.ptr, _stream(), ctypes.byref(v)), "thrift_get_device_status")
    return int(v.value)


# ------------------------------------------------------------------ decode

@dataclasses.dataclass
class DecodeConfig:
    """Decode step description (thrift_decode_cfg): Nq new query rows per head, the newest
    positions of a cache of Nk keys."""

    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool = True
    block_k: int = 64
    topk_abs: int = -1
    topk_bp: int = 500
    softmax_scale: float = 0.0
    n_valid: int = 0  # keys the cache holds (0: all Nk)

    @classmethod
    def from_workload(cls, w) -> "DecodeConfig":
        return cls(w.B, w.Hq, w.Hkv, w.n_query, w.N, w.d, bool(w.causal), w.block_k, w.topk_abs,
                   w.topk_bp)

    def c(self) -> _lib.CDecodeCfg:
        return _lib.CDecodeCfg(self.B, self.Hq, self.Hkv, self.Nq, self.Nk, self.d, int(self.causal),
                               self.block_k, self.topk_abs, self.topk_bp, self.softmax_scale, self.n_valid)

    def for_cache(self, cache: "KVCache") -> "DecodeConfig":
        """This step against `cache`: its capacity as Nk and the keys it holds as n_valid."""
        return dataclasses.replace(self, Nk=cache.capacity, n_valid=cache.length)

    @property
    def n_kb(self) -> int:
        return self.Nk // self.block_k

    @property
    def mask_words(self) -> int:
        return (self.n_kb + 31) // 32

    def workspace(self, device) -> Workspace:
        c = self.c()
        n = load().thrift_decode_workspace_bytes(ctypes.byref(c))
        if n == 0:
            raise ThriftError(_lib.THRIFT_ERR_UNSUPPORTED, "decode workspace size")
        return Workspace(n, device)


def kv_block_means(k: torch.Tensor, block_k: int) -> torch.Tensor:
    """Block means of the cache's keys, float64 [.., Nk/block_k, d] (thrift_kv_block_means)."""
    assert k.is_cuda and k.dtype == torch.float16 and k.is_contiguous()
    *lead, Nk, d = k.shape
    outer = 1
    for s in lead:
        outer *= s
    kbar = torch.empty((*lead, Nk // block_k, d), dtype=torch.float64, device=k.device)
    check(load().thrift_kv_block_means(_ptr(k), outer, Nk, d, block_k, _ptr(kbar), _stream()),
          "thrift_kv_block_means")
    return kbar


@dataclasses.dataclass
class KVCache:
    """A KV cache held twice, FP16 and NVFP4, with the key block means the selection reads.
    `capacity` keys of storage, of which the first `length` are held (the rest zero)."""

    k: torch.Tensor
    v: torch.Tensor
    k4: NVFP4Tensor
    v4: NVFP4Tensor
    kbar: torch.Tensor
    block_k: int
    length: int = -1
    capacity: int = -1

    def __post_init__(self):
        if self.capacity < 0:
            self.capacity = self.k.shape[-2]
        if self.length < 0:
            self.length = self.capacity

    @classmethod
    def build(cls, k: torch.Tensor, v: torch.Tensor, block_k: int, ws: Optional[Workspace] = None,
              capacity: Optional[int] = None) -> "KVCache":
        """The cache of the keys and values k, v [B, Hkv, N, d].  Without `capacity` (and N a
        multiple of 128 and of block_k) the cache is exactly k, v; with it, zero-filled storage of
        `capacity` keys holds them and appends can follow (thrift_kv_append): the NVFP4 tensor
        scales are fixed here, from these first N keys."""
        if capacity is None:
            return cls(k, v, quantize_nvfp4(k, 0, ws=ws), quantize_nvfp4(v, 1, ws=ws), kv_block_means(k, block_k),
                       block_k)
        B, H, N, d = k.shape
        dev = k.device
        kc = torch.zeros((B, H, capacity, d), dtype=torch.float16, device=dev)
        vc = torch.zeros_like(kc)
        k4 = NVFP4Tensor.empty(B * H, capacity, d, 0, dev)
        v4 = NVFP4Tensor.empty(B * H, capacity, d, 1, dev)
        for t in (k4, v4):
            t.codes.zero_(); t.scales.zero_(); t.scales_mma.zero_()
        kbar = torch.zeros((B, H, capacity // block_k, d), dtype=torch.float64, device=dev)
        cache = cls(kc, vc, k4, v4, kbar, block_k, 0, capacity)
        kc[:, :, :N].copy_(k)
        vc[:, :, :N].copy_(v)
        if ws is None:
            ws = Workspace(256, dev)
        L = load()
        for x, t in ((kc, k4), (vc, v4)):
            check(L.thrift_nvfp4_tensor_scale(_ptr(x), x.numel(), _ptr(t.tensor_scale), ws.ptr, ws.nbytes,
                                              _stream()), "thrift_nvfp4_tensor_scale")
        cache.append(None, None, N)
        return cache

    def append(self, k_new: Optional[torch.Tensor], v_new: Optional[torch.Tensor], T: Optional[int] = None):
        """Append T keys and values [B, Hkv, T, d] (thrift_kv_append); None: they are already in
        the FP16 storage at [length, length + T)."""
        if T is None:
            T = k_new.shape[-2]
        B, H, cap, d = self.k.shape
        check(load().thrift_kv_append(_ptr(k_new), _ptr(v_new), B * H, cap, d, self.block_k, self.length, T,
                                      _ptr(self.k), _ptr(self.v), ctypes.byref(self.k4.c()),
                                      ctypes.byref(self.v4.c()), _ptr(self.kbar), _stream()),
              "thrift_kv_append")
        self.length += T
        return self


def decode_select(q: torch.Tensor, cache: KVCache, cfg: DecodeConfig, ws: Optional[Workspace] = None,
                  want_scores: bool = False) -> Selection:
    """Per-head top-k key blocks of one decode step (thrift_decode_select); the Selection's
    tensors have a query-block axis of length 1."""
    cfg = cfg.for_cache(cache)
    dev = q.device
    sel = Selection(
        torch.empty((cfg.B, cfg.Hq, 1, cfg.mask_words), dtype=torch.int32, device=dev),
        torch.empty((cfg.B, cfg.Hq, 1), dtype=torch.int32, device=dev),
        torch.empty((cfg.B, cfg.Hq, 1, cfg.n_kb), dtype=torch.int16, device=dev),
        torch.empty((cfg.B, cfg.Hq, 1, cfg.n_kb), dtype=torch.float64, device=dev) if want_scores else None)
    if ws is None:
        ws = cfg.workspace(dev)
    c = cfg.c()
    check(load().thrift_decode_select(_ptr(q), _ptr(cache.kbar), ctypes.byref(c), _ptr(sel.mask),
                                      _ptr(sel.counts), _ptr(sel.lists), _ptr(sel.scores), ws.ptr, ws.nbytes,
                                      _stream()), "thrift_decode_select")
    return sel


def _decode_out(q, cfg, out, lse, want_lse):
    if out is None:
        out = torch.empty((cfg.B, cfg.Hq, cfg.Nq, cfg.d), dtype=torch.float16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((cfg.B, cfg.Hq, cfg.Nq), dtype=torch.float32, device=q.device)
    return out, lse


def decode_attn(q: torch.Tensor, cache: KVCache, sel: Optional[Selection], cfg: DecodeConfig,
                out=None, lse=None, ws: Optional[Workspace] = None, want_lse: bool = True):
    """Decode attention with a given selection (thrift_decode_attn).  Returns (out, lse)."""
    cfg = cfg.for_cache(cache)
    out, lse = _decode_out(q, cfg, out, lse, want_lse)
    if ws is None:
        ws = cfg.workspace(q.device)
    c = cfg.c()
    k4, v4 = cache.k4.c(), cache.v4.c()
    check(load().thrift_decode_attn(_ptr(q), _ptr(cache.k), _ptr(cache.v), ctypes.byref(k4), ctypes.byref(v4),
                                    None if sel is None else _ptr(sel.mask), _ptr(out), _ptr(lse),
                                    ctypes.byref(c), ws.ptr, ws.nbytes, _stream()), "thrift_decode_attn")
    return out, lse


def decode_fwd(q: torch.Tensor, cache: KVCache, cfg: DecodeConfig, out=None, lse=None,
               ws: Optional[Workspace] = None, want_lse: bool = True):
    """One decode step, selection and attention (thrift_decode_fwd).  Returns (out, lse)."""
    cfg = cfg.for_cache(cache)
    out, lse = _decode_out(q, cfg, out, lse, want_lse)
    if ws is None:
        ws = cfg.workspace(q.device)
    c = cfg.c()
    k4, v4 = cache.k4.c(), cache.v4.c()
    check(load().thrift_decode_fwd(_ptr(q), _ptr(cache.k), _ptr(cache.v), ctypes.byref(k4), ctypes.byref(v4),
                                   _ptr(cache.kbar), _ptr(out), _ptr(lse), ctypes.byref(c), ws.ptr, ws.nbytes,
                                   _stream()), "thrift_decode_fwd")
    return out, lse


def decode_attn_sparse(q: torch.Tensor, cache: KVCache, sel: Selection, cfg: DecodeConfig, out=None, lse=None,
                       ws: Optional[Workspace] = None, want_lse: bool = True):
    """Compute-matched sparse decode (thrift_decode_attn_sparse): only the selected key blocks, in
    FP16.  Returns (out, lse)."""
    cfg = cfg.for_cache(cache)
    out, lse = _decode_out(q, cfg, out, lse, want_lse)
    if ws is None:
        ws = cfg.workspace(q.device)
    c = cfg.c()
    check(load().thrift_decode_attn_sparse(_ptr(q), _ptr(cache.k), _ptr(cache.v), _ptr(sel.mask), _ptr(out),
                                           _ptr(lse), ctypes.byref(c), ws.ptr, ws.nbytes, _stream()),
          "thrift_decode_attn_sparse")
    return out, lse
