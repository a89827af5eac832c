"""Pins for the oracle's compute-matched sparse variant (only the selected block pairs, in FP16;
every other pair dropped), checked against float64 SDPA with the corresponding block mask and
against the mixed-precision oracle where the two coincide."""

import numpy as np
import pytest
import torch

import oracle
import workloads


def small(**kw):
    base = dict(name="s", index=92, B=1, Hq=4, Hkv=2, N=256, d=64, causal=True, block_q=64,
                block_k=32, topk_abs=-1, topk_bp=2500, dist="normal")
    base.update(kw)
    return workloads.Workload(**base)


def sdpa_masked(q, k, v, tau, vis):
    """float64 softmax attention with a boolean visibility mask [B, Hq, Nq, Nk]; rows that see no
    key get 0 and lse -inf."""
    qq, kk, vv = (torch.from_numpy(np.asarray(a, np.float64)) for a in (q, k, v))
    g = qq.shape[1] // kk.shape[1]
    kk = kk.repeat_interleave(g, dim=1)
    vv = vv.repeat_interleave(g, dim=1)
    s = (float(tau) * qq @ kk.transpose(-1, -2)).masked_fill(~torch.from_numpy(vis), float("-inf"))
    lse = torch.logsumexp(s, -1)
    p = torch.exp(s - lse[..., None]).nan_to_num(0.0)
    return (p @ vv).numpy(), lse.numpy()


def block_mask(sel, w, nq, nk, qoff=0):
    """Key visibility of the selected pairs (and the causal mask) per query row."""
    rows = np.arange(nq)[:, None] + qoff
    keys = np.arange(nk)[None, :]
    m = np.repeat(np.repeat(sel.astype(bool), w.block_q if sel.shape[2] > 1 else nq, axis=2),
                  w.block_k, axis=3)[:, :, :nq, :nk]
    if w.causal:
        m = m & (keys <= rows)[None, None]
    return m


@pytest.mark.parametrize("causal,bp", [(True, 2500), (False, 1000), (True, 600)])
def test_sparse_equals_masked_softmax(causal, bp):
    w = small(causal=causal, topk_bp=bp)
    q, k, v = workloads.make_qkv(w)
    sel, _, _ = oracle.select(oracle.block_scores(q, k, w), w)
    out, lse, o64 = oracle.attn_sparse(q, k, v, sel, w, want_f64=True)
    vis = block_mask(sel, w, w.N, w.N)
    ref, lse_ref = sdpa_masked(q, k, v, oracle.softmax_scale(w.d), vis)
    empty = ~vis.any(-1)
    assert np.all(o64[empty] == 0) and np.all(np.isneginf(lse[empty]))
    full = ~empty
    err = np.abs(o64[full] - ref[full]).max()
    assert err <= 2e-3 * max(1.0, np.abs(ref).max())
    assert np.abs(lse[full] - lse_ref[full]).max() < 1e-5
    # a plausible mistake -- computing the dropped pairs -- changes the result
    mixed, _, m64 = oracle.attn(q, k, v, *oracle.quantize_all(q, k, v), sel, w, want_f64=True)
    assert np.abs(m64 - o64).max() > 1e-2


def test_sparse_with_every_pair_equals_all_fp16():
    w = small(topk_bp=10000)
    q, k, v = workloads.make_qkv(w)
    r = oracle.forward(w, q, k, v, want_f64=True)
    _, lse, o64 = oracle.attn_sparse(q, k, v, r["sel"], w, want_f64=True)
    assert np.array_equal(o64, r["out64"]) and np.array_equal(lse, r["lse"])


def test_decode_sparse_equals_masked_softmax():
    w = workloads.Workload(name="ds", index=93, B=1, Hq=4, Hkv=2, N=512, d=64, causal=True, block_q=64,
                           block_k=32, topk_abs=-1, topk_bp=2000, dist="normal", n_query=3)
    q, k, v = workloads.make_qkv(w)
    q4, k4, v4 = oracle.quantize_all(q, k, v)
    sel, _, _ = oracle.select(oracle.decode_block_scores(q, k, w.block_k, True), w)
    out, lse, o64 = oracle.decode_attn(q, k, v, q4, k4, v4, sel, w.block_k, True, want_f64=True, sparse=True)
    vis = block_mask(sel, w, 3, w.N, qoff=w.N - 3)
    ref, lse_ref = sdpa_masked(q, k, v, oracle.softmax_scale(w.d), vis)
    assert np.abs(o64 - ref).max() <= 2e-3 * max(1.0, np.abs(ref).max())
    assert np.abs(lse - lse_ref).max() < 1e-5
