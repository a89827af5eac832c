"""Parity of the compute-matched sparse variant (thrift_attn_fwd_sparse, thrift_decode_attn_sparse)
with the oracle's sparse form on the same seeded inputs and selections.  Bar as for the mixed path:
rel-L2 <= 1e-3, element-wise within max(1e-2, one FP16 step), lse within 1e-3; rows left with no
key are 0 with lse -inf on both sides."""

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


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def fp16_ulp(x):
    a = np.maximum(np.abs(x), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(a)) - 10)


def compare(out_g, lse_g, out_o, lse_o, rows=None):
    og = out_g.cpu().numpy().astype(np.float64)
    lg = lse_g.cpu().numpy().astype(np.float64)
    oo = out_o.astype(np.float64)
    lo = lse_o.astype(np.float64)
    if rows is not None:
        og, lg, oo, lo = og[rows], lg[rows], oo[rows], lo[rows]
    empty = np.isneginf(lo)
    assert np.array_equal(np.isneginf(lg), empty)
    assert np.all(og[empty] == 0)
    fin = ~empty
    a, e = og[fin], oo[fin]
    rel = np.linalg.norm(a - e) / max(np.linalg.norm(e), 1e-30)
    err = np.abs(a - e)
    assert np.isfinite(a).all()
    lmx = np.abs(lg[fin] - lo[fin]).max() if fin.any() else 0.0
    print(f"sparse parity: rel-L2 {rel:.3e} max-abs {err.max() if err.size else 0:.3e} lse {lmx:.3e} "
          f"empty rows {int(empty.sum())}")
    assert rel <= 1e-3 and lmx <= 1e-3 and np.all(err <= np.maximum(1e-2, fp16_ulp(e)))


@pytest.mark.parametrize("name,bp,shape", [
    ("tiny", None, {}), ("n4k", None, {}), ("n4k", 10000, {}),
    ("n4k", 700, dict(N=1024, causal=True, Hq=4, Hkv=2, block_q=64, block_k=64)),
    ("n4k", 300, dict(N=2048, causal=True, Hq=4, Hkv=1, block_q=128, block_k=128, d=64)),
])
def test_prefill_sparse(pab, name, bp, shape):
    w = workloads.WORKLOADS[name].with_shape(**shape)
    if bp is not None:
        w = w.with_budget(bp)
    q, k, v = workloads.make_qkv(w)
    sel_o, _, _ = oracle.select(oracle.block_scores(q, k, w), w)
    out_o, lse_o, _ = oracle.attn_sparse(q, k, v, sel_o, w)
    gq, gk, gv = dev(q), dev(k), dev(v)
    cfg = pab.Config.from_workload(w)
    sel = pab.block_select(gq, gk, cfg)
    ws = pab.Workspace(256, gq.device)
    out, lse = pab.attn_fwd_sparse(gq, gk, gv, sel, cfg, ws=ws)
    torch.cuda.synchronize()
    assert pab.device_status(ws) == 0
    compare(out, lse, out_o, lse_o)


def test_prefill32k_sparse_sampled(pab):
    w = workloads.WORKLOADS["prefill32k"]
    q, k, v = workloads.make_qkv(w)
    sel_o, _, _ = oracle.select(oracle.block_scores(q, k, w), w)
    units = workloads.sample_units(w, 16)
    out_o, lse_o, _ = oracle.attn_sparse(q, k, v, sel_o, w, units=units)
    gq, gk, gv = dev(q), dev(k), dev(v)
    cfg = pab.Config.from_workload(w)
    sel = pab.block_select(gq, gk, cfg)
    out, lse = pab.attn_fwd_sparse(gq, gk, gv, sel, cfg)
    torch.cuda.synchronize()
    idx = np.concatenate([(((b * w.Hq + h) * w.N) + np.arange(i * w.block_q, (i + 1) * w.block_q))
                          for (b, h, i) in units])
    compare(out.reshape(-1, w.d), lse.reshape(-1), out_o.reshape(-1, w.d), lse_o.reshape(-1), rows=idx)


@pytest.mark.parametrize("name,shape", [("decode_tiny", {}), ("decode_tiny", dict(Hq=8, Hkv=2, n_query=4, d=128)),
                                        ("decode32k", {})])
def test_decode_sparse(pab, name, shape):
    w = workloads.WORKLOADS[name].with_shape(**shape)
    q, k, v = workloads.make_qkv(w)
    q4, k4, v4 = oracle.quantize_all(q, k, v)
    sel_o, _, _ = oracle.select(oracle.decode_block_scores(q, k, w.block_k, w.causal), w)
    out_o, lse_o, _ = oracle.decode_attn(q, k, v, q4, k4, v4, sel_o, w.block_k, w.causal, sparse=True)
    gq, gk, gv = dev(q), dev(k), dev(v)
    cfg = pab.DecodeConfig.from_workload(w)
    cache = pab.KVCache.build(gk, gv, w.block_k)
    ws = cfg.workspace(gq.device)
    sel = pab.decode_select(gq, cache, cfg, ws=ws)
    out, lse = pab.decode_attn_sparse(gq, cache, sel, cfg, ws=ws)
    torch.cuda.synchronize()
    assert pab.device_status(ws) == 0
    compare(out, lse, out_o, lse_o)


@pytest.mark.parametrize("sparse", [False, True])
def test_short_entry_lists(pab, sparse):
    """Many one-tile heads whose lists hold a single key block (d = 64, 128-key blocks, N = 128,
    causal): more units than SMs, so a CTA runs several such tiles in a row."""
    w = workloads.WORKLOADS["n4k"].with_shape(B=1, Hq=300, Hkv=300, N=128, d=64, causal=True, block_q=128,
                                              block_k=128).with_budget(5000)
    q, k, v = workloads.make_qkv(w)
    gq, gk, gv = dev(q), dev(k), dev(v)
    cfg = pab.Config.from_workload(w)
    sel = pab.block_select(gq, gk, cfg)
    ws = pab.Workspace(256, gq.device)
    sel_o, _, _ = oracle.select(oracle.block_scores(q, k, w), w)
    if sparse:
        out, lse = pab.attn_fwd_sparse(gq, gk, gv, sel, cfg, ws=ws)
        out_o, lse_o, _ = oracle.attn_sparse(q, k, v, sel_o, w)
    else:
        q4, k4, v4 = pab.quantize_qkv(gq, gk, gv)
        out, lse = pab.attn_fwd(gq, gk, gv, q4, k4, v4, sel, cfg, ws=ws)
        out_o, lse_o, _ = oracle.attn(q, k, v, *oracle.quantize_all(q, k, v), sel_o, w)
    torch.cuda.synchronize()
    assert pab.device_status(ws) == 0
    compare(out, lse, out_o, lse_o)
