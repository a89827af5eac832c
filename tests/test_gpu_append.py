"""Appending to the double-cached KV cache (thrift_kv_append, reading R-append) against the
oracle: after every append the cache's NVFP4 copies (codes, both scale layouts) and key-block
means are bit for bit those of the oracle's one-shot quantisation of the zero-padded grown cache
with the scales fixed at build time; a decode step at the ragged final length then matches the
oracle's decode of the same cache (selection exact, output within the parity bar)."""

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pab(cuda_device):
    from precision_attention_block_b200 import build
    build.build()
    import precision_attention_block_b200 as pab
    pab.load()
    return pab


def sf_mma_index(rows, len_):
    r = np.arange(rows)[:, None]
    g = np.arange(len_ // 16)[None, :]
    nkb = len_ // 64
    return ((r >> 7) * nkb + (g >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (g & 3)


def check_cache(cache, k, v, length, k_ts, v_ts, bk):
    cap = k.shape[2]
    kp, vp = k.copy(), v.copy()
    kp[:, :, length:] = 0
    vp[:, :, length:] = 0
    k4 = oracle.quantize_nvfp4(kp, 0, tensor_scale=k_ts)
    v4 = oracle.quantize_nvfp4(vp, 1, tensor_scale=v_ts)
    for g, o in ((cache.k4, k4), (cache.v4, v4)):
        assert np.array_equal(g.codes.cpu().numpy().reshape(o.codes.shape), o.codes)
        sc = g.scales.cpu().numpy().reshape(o.scales.shape)
        assert np.array_equal(sc, o.scales)
        rows, len_ = int(np.prod(o.scales.shape[:-1])), o.scales.shape[-1] * 16
        assert np.array_equal(g.scales_mma.cpu().numpy()[sf_mma_index(rows, len_)], o.scales.reshape(rows, -1))
    kb = cache.kbar.cpu().numpy()
    for j in range((length + bk - 1) // bk):
        rows = kp[:, :, j * bk:min((j + 1) * bk, length)].astype(np.float64)
        assert np.array_equal(kb[:, :, j], rows.sum(2) / rows.shape[2])
    assert np.array_equal(cache.k[:, :, :length].cpu().numpy(), k[:, :, :length])
    assert not cache.k[:, :, length:].any() and not cache.v[:, :, length:].any()
    return kp, vp, k4, v4


@pytest.mark.parametrize("d,bk", [(64, 64), (128, 128)])
def test_append_then_decode(pab, d, bk):
    w = workloads.WORKLOADS["decode_tiny"].with_shape(N=1280, d=d, block_k=bk, topk_bp=2000)
    q, k, v = workloads.make_qkv(w)
    dev = torch.device("cuda")
    gk, gv = torch.from_numpy(k).to(dev), torch.from_numpy(v).to(dev)
    L0 = 1000
    cache = pab.KVCache.build(gk[:, :, :L0].contiguous(), gv[:, :, :L0].contiguous(), bk, capacity=1280)
    torch.cuda.synchronize()
    # the build fixes the tensor scales at those of the first L0 keys
    k_ts = oracle.quantize_nvfp4(np.where(np.arange(1280)[None, None, :, None] < L0, k, 0).astype(np.float16),
                                 0).tensor_scale
    v_ts = oracle.quantize_nvfp4(np.where(np.arange(1280)[None, None, :, None] < L0, v, 0).astype(np.float16),
                                 1).tensor_scale
    assert cache.k4.tensor_scale.item() == float(k_ts) and cache.v4.tensor_scale.item() == float(v_ts)
    check_cache(cache, k, v, L0, k_ts, v_ts, bk)
    length = L0
    for T in (1, 7, 64, 33, 1, 50):
        cache.append(gk[:, :, length:length + T].contiguous(), gv[:, :, length:length + T].contiguous())
        length += T
        torch.cuda.synchronize()
        assert cache.length == length
        kp, vp, k4, v4 = check_cache(cache, k, v, length, k_ts, v_ts, bk)
    gq = torch.from_numpy(q).to(dev)
    for bp in (0, 2000, 10000):
        wb = w.with_budget(bp)
        cfg = pab.DecodeConfig.from_workload(wb)
        out, lse = pab.decode_fwd(gq, cache, cfg)
        sel = pab.decode_select(gq, cache, cfg, want_scores=True)
        torch.cuda.synchronize()
        ref = oracle.decode_forward(wb, q, kp, vp, k4=k4, v4=v4, n_valid=length)
        sc_o = ref["scores"]
        sc_g = sel.scores.cpu().numpy()
        assert np.array_equal(np.isfinite(sc_g), np.isfinite(sc_o))
        fin = np.isfinite(sc_o)
        assert np.array_equal(sc_g[fin], sc_o[fin])
        mask = sel.mask.cpu().numpy().view(np.uint32)
        bits = ((mask[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(*mask.shape[:-1], -1)
        assert np.array_equal(bits[..., :sc_o.shape[-1]].astype(bool), ref["sel"].astype(bool))
        a = out.cpu().numpy().astype(np.float64)
        e = ref["out"].astype(np.float64)
        rel = np.linalg.norm(a - e) / np.linalg.norm(e)
        assert rel <= 1e-3 and np.abs(a - e).max() <= 1e-2, (bp, rel)
        assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= 1e-3
