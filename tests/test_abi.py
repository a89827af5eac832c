"""The C ABI without a GPU: the library loads, exports every function the headers declare, sizes
its buffers, and rejects bad arguments on the host with a status code before touching CUDA."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from precision_attention_block_b200 import build
    build.build()
    from precision_attention_block_b200 import _lib
    return _lib.load()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^\s*(?:const\s+char\s*\*|size_t|int32_t|thrift_status)\s+(thrift_\w+)\s*\(",
                                    src, re.M))
    return names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert {"thrift_quantize_nvfp4", "thrift_block_select", "thrift_attn_fwd"} <= names
    for n in names:
        assert hasattr(L, n), n


def test_checked_build_exports_the_same_abi(L):
    """libthrift_checked.so (in-kernel bounds checks) is a drop-in build of the same ABI; only it
    reports the checks as enabled."""
    from precision_attention_block_b200 import build
    path = build.build(checked=True)
    C = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(C, n), n
    C.thrift_debug_checks_enabled.restype = ctypes.c_int32
    assert C.thrift_debug_checks_enabled() == 1
    assert L.thrift_debug_checks_enabled() == 0
    assert L.thrift_status_str(8) == b"in-kernel bounds check failed"


def test_binding_covers_every_declared_symbol():
    from precision_attention_block_b200 import _lib
    assert declared_functions() <= set(_lib.SIGNATURES)


def cfg(**kw):
    from precision_attention_block_b200 import Config
    base = dict(B=1, Hq=32, Hkv=8, N=32768, d=128, causal=True, block_q=128, block_k=64, topk_bp=500)
    base.update(kw)
    return Config(**base).c()


def test_workspace_sizes(L):
    c = cfg()
    n = L.thrift_workspace_bytes(ctypes.byref(c))
    # block means (float64) + dense score matrix (float64) + header
    assert n >= 256 + 32 * 256 * 128 * 8 + 8 * 512 * 128 * 8 + 32 * 256 * 512 * 8
    auto = L.thrift_auto_workspace_bytes(ctypes.byref(c))
    assert auto > n + (32 + 16) * 32768 * 128 // 2
    assert L.thrift_nvfp4_scales_mma_bytes(32, 32768, 128, 0) == 32 * 32768 * 128 // 16
    assert L.thrift_nvfp4_scales_mma_bytes(8, 32768, 128, 1) == 8 * 128 * 32768 // 16
    assert L.thrift_nvfp4_scales_mma_bytes(3, 256, 64, 1) == 2 * (256 // 64) * 512  # rows padded to 128


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 2), (dict(Hkv=5), 1), (dict(block_k=32), 2), (dict(N=1000), 2), (dict(topk_bp=20000), 1),
    (dict(causal=2), 1), (dict(topk_abs=-2), 1), (dict(block_q=256), 2)])
def test_bad_config_rejected_on_host(L, kw, status):
    c = cfg(**kw)
    assert L.thrift_workspace_bytes(ctypes.byref(c)) == 0
    from precision_attention_block_b200 import _lib
    out = ctypes.c_void_p(0x1000)
    rc = L.thrift_attn_fwd(out, out, out, None, None, None, out, out, out, out, None, ctypes.byref(c),
                           ctypes.c_void_p(0x100000), 1 << 20, None)
    assert rc == status
    rc = L.thrift_block_select(out, out, ctypes.byref(c), out, out, out, None, ctypes.c_void_p(0x100000),
                               1 << 30, None)
    assert rc == status


def test_null_and_workspace_errors(L):
    from precision_attention_block_b200 import _lib
    c = cfg()
    p = ctypes.c_void_p(0x1000)
    assert L.thrift_attn_fwd_auto(None, p, p, p, None, ctypes.byref(c), p, 1 << 40, None) == 1
    assert L.thrift_attn_fwd_auto(p, p, p, p, None, ctypes.byref(c), ctypes.c_void_p(0x1001), 1 << 40, None) == 5
    assert L.thrift_attn_fwd_auto(p, p, p, p, None, ctypes.byref(c), ctypes.c_void_p(0x1000), 16, None) == 5
    assert L.thrift_quantize_nvfp4(None, 1, 128, 128, None, p, 256, None) == 1
    nv = _lib.CNVFP4(0x1000, 0x1000, 0x1000, 0x1000, 0)
    assert L.thrift_quantize_nvfp4(p, 1, 128, 96, ctypes.byref(nv), p, 256, None) == 2
    assert L.thrift_quantize_nvfp4(p, 1, 100, 128, ctypes.byref(nv), p, 256, None) == 2
    assert L.thrift_quantize_nvfp4(p, 1, 128, 128, ctypes.byref(nv), None, 256, None) == 5
    assert L.thrift_reset_device_status(None, None) == 5
    assert L.thrift_get_device_status(p, None, None) == 1
    assert L.thrift_debug_wait_timeout(p, 0, None) == 1
    # uniform NVFP4 needs the NVFP4 tensors; all-FP16 needs the FP16 ones; mixed needs the mask
    assert L.thrift_attn_fwd(p, p, p, None, None, None, p, p, p, p, None, ctypes.byref(cfg(topk_bp=0)),
                             p, 256, None) == 1
    assert L.thrift_attn_fwd(None, None, None, ctypes.byref(nv), ctypes.byref(nv), ctypes.byref(nv), p, p, p, p,
                             None, ctypes.byref(cfg(topk_bp=10000)), p, 256, None) == 1
    assert L.thrift_status_str(4) == b"device wait timed out"
    # the Attn-QAT variant needs its FP32 output
    assert L.thrift_attn_fwd_qat(p, p, p, ctypes.byref(nv), ctypes.byref(nv), ctypes.byref(nv), p, p, None, None,
                                 ctypes.byref(c), p, 256, None) == 1
    # the running-maximum variant checks its arguments as thrift_attn_fwd does
    assert L.thrift_attn_fwd_running_max(p, p, p, None, None, None, p, p, None, ctypes.byref(cfg(topk_bp=0)),
                                         p, 256, None) == 1
    assert L.thrift_attn_fwd_running_max(p, p, p, ctypes.byref(nv), ctypes.byref(nv), ctypes.byref(nv), None, p,
                                         None, ctypes.byref(c), p, 256, None) == 1
    nv1 = _lib.CNVFP4(0x1000, 0x1000, 0x1000, 0x1000, 1)
    assert L.thrift_attn_fwd_running_max(p, p, p, ctypes.byref(nv), ctypes.byref(nv), ctypes.byref(nv1), p, p,
                                         None, ctypes.byref(c), None, 0, None) == 5
    # strides: multiples of 8 elements, token rows at least d apart; NULL is dense
    bad = [_lib.CStrides(8 * 512 * 128, 512 * 128, 100), _lib.CStrides(8 * 512 * 128, 512 * 128, 64),
           _lib.CStrides(-8, 512 * 128, 128), _lib.CStrides(4, 512 * 128, 128)]
    for st in bad:
        assert L.thrift_attn_fwd_auto_strided(p, ctypes.byref(st), p, None, p, None, p, None, None,
                                              ctypes.byref(c), p, 1 << 40, None) == 1
        assert L.thrift_block_select_strided(p, None, p, ctypes.byref(st), ctypes.byref(c), p, p, p, None, p,
                                             1 << 40, None) == 1
        assert L.thrift_quantize_nvfp4_strided(p, ctypes.byref(st), 1, 8, 512, 128, ctypes.byref(nv), p, 256,
                                               None) == 1
        assert L.thrift_attn_fwd_strided(p, None, p, None, p, None, ctypes.byref(nv), ctypes.byref(nv),
                                         ctypes.byref(nv1), p, p, ctypes.byref(st), None, ctypes.byref(c), p, 256,
                                         None) == 1
    good = _lib.CStrides(512 * 8 * 128, 128, 8 * 128)  # token-major [B, N, H, d]
    assert L.thrift_quantize_nvfp4_strided(p, ctypes.byref(good), 1, 8, 512, 128, ctypes.byref(nv), None, 0,
                                           None) == 5
    assert L.thrift_quantize_nvfp4_strided(p, ctypes.byref(good), 0, 8, 512, 128, ctypes.byref(nv), p, 256,
                                           None) == 1


def dcfg(**kw):
    from precision_attention_block_b200 import DecodeConfig
    base = dict(B=1, Hq=32, Hkv=8, Nq=1, Nk=131072, d=128, causal=True, block_k=128, topk_bp=200)
    base.update(kw)
    return DecodeConfig(**base).c()


def test_decode_workspace_sizes(L):
    c = dcfg()
    n = L.thrift_decode_workspace_bytes(ctypes.byref(c))
    # at least the selection scratch (qbar + scores in float64) and the lists
    assert n >= 256 + 32 * 128 * 8 + 32 * 1024 * 8 + 32 * 1024 * 2
    assert n < 64 << 20
    assert L.thrift_decode_workspace_bytes(ctypes.byref(dcfg(Nq=4))) > 0          # 4 heads x 4 rows = 16
    assert L.thrift_decode_workspace_bytes(ctypes.byref(dcfg(Nq=1, Hkv=2))) > 0   # 16 heads x 1 row


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 2), (dict(Hkv=5), 1), (dict(block_k=32), 2), (dict(Nk=1000), 2), (dict(topk_bp=20000), 1),
    (dict(causal=2), 1), (dict(Nq=0), 1), (dict(Nq=5), 2), (dict(Hkv=1), 2), (dict(Nq=200, Nk=128), 1)])
def test_bad_decode_config_rejected_on_host(L, kw, status):
    c = dcfg(**kw)
    assert L.thrift_decode_workspace_bytes(ctypes.byref(c)) == 0
    p = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x100000)
    assert L.thrift_decode_attn(p, p, p, None, None, p, p, None, ctypes.byref(c), ws, 1 << 30, None) == status
    assert L.thrift_decode_select(p, p, ctypes.byref(c), p, p, p, None, ws, 1 << 30, None) == status
    assert L.thrift_decode_fwd(p, p, p, None, None, p, p, None, ctypes.byref(c), ws, 1 << 30, None) == status


def test_decode_null_and_workspace_errors(L):
    from precision_attention_block_b200 import _lib
    c = dcfg()
    p = ctypes.c_void_p(0x1000)
    nv0 = _lib.CNVFP4(0x1000, 0x1000, 0x1000, 0x1000, 0)
    nv1 = _lib.CNVFP4(0x1000, 0x1000, 0x1000, 0x1000, 1)
    big = 1 << 40
    # missing query rows, missing NVFP4 cache, wrong group axis, missing mask, misaligned pointers
    assert L.thrift_decode_attn(None, p, p, ctypes.byref(nv0), ctypes.byref(nv1), p, p, None, ctypes.byref(c), p,
                                big, None) == 1
    assert L.thrift_decode_attn(p, p, p, None, None, p, p, None, ctypes.byref(c), p, big, None) == 1
    assert L.thrift_decode_attn(p, p, p, ctypes.byref(nv1), ctypes.byref(nv1), p, p, None, ctypes.byref(c), p,
                                big, None) == 1
    assert L.thrift_decode_attn(p, p, p, ctypes.byref(nv0), ctypes.byref(nv1), None, p, None, ctypes.byref(c), p,
                                big, None) == 1
    odd = ctypes.c_void_p(0x1008)
    assert L.thrift_decode_attn(odd, p, p, ctypes.byref(nv0), ctypes.byref(nv1), p, p, None, ctypes.byref(c), p,
                                big, None) == 1
    # all-FP16 needs no NVFP4 cache but the FP16 one; uniform NVFP4 needs no mask
    assert L.thrift_decode_attn(p, None, None, None, None, None, p, None, ctypes.byref(dcfg(topk_bp=10000)), p,
                                big, None) == 1
    # workspace too small or misaligned
    assert L.thrift_decode_attn(p, p, p, ctypes.byref(nv0), ctypes.byref(nv1), p, p, None, ctypes.byref(c), p,
                                1024, None) == 5
    assert L.thrift_decode_fwd(p, p, p, ctypes.byref(nv0), ctypes.byref(nv1), p, p, None, ctypes.byref(c),
                               ctypes.c_void_p(0x1001), big, None) == 5
    assert L.thrift_kv_block_means(None, 1, 128, 128, 64, p, None) == 1
    assert L.thrift_kv_block_means(p, 1, 100, 128, 64, p, None) == 2
    assert L.thrift_kv_block_means(p, 1, 128, 96, 64, p, None) == 2
    # appending: the new keys must fit the capacity; unsupported sizes; misaligned buffers
    n0 = _lib.CNVFP4(0x1000, 0x1000, 0x1000, 0x1000, 0)
    n1 = _lib.CNVFP4(0x1000, 0x1000, 0x1000, 0x1000, 1)
    assert L.thrift_kv_append(p, p, 2, 1024, 64, 64, 1000, 25, p, p, ctypes.byref(n0), ctypes.byref(n1), p,
                              None) == 1
    assert L.thrift_kv_append(p, p, 2, 1024, 96, 64, 0, 1, p, p, ctypes.byref(n0), ctypes.byref(n1), p, None) == 2
    assert L.thrift_kv_append(p, p, 2, 1000, 64, 64, 0, 1, p, p, ctypes.byref(n0), ctypes.byref(n1), p, None) == 2
    assert L.thrift_kv_append(p, p, 2, 1024, 64, 64, 0, 1, p, p, ctypes.byref(n1), ctypes.byref(n1), p, None) == 1
    assert L.thrift_kv_append(ctypes.c_void_p(0x1008), p, 2, 1024, 64, 64, 0, 1, p, p, ctypes.byref(n0),
                              ctypes.byref(n1), p, None) == 1
    assert L.thrift_nvfp4_tensor_scale(p, 12, p, p, 256, None) == 1
    assert L.thrift_nvfp4_tensor_scale(p, 16, p, None, 256, None) == 5
    # the decode step's valid length lies between Nq and the capacity
    assert L.thrift_decode_workspace_bytes(ctypes.byref(dcfg(n_valid=131072 + 1))) == 0
    assert L.thrift_decode_workspace_bytes(ctypes.byref(dcfg(n_valid=1000))) > 0
