"""Pins for the oracle's decode form (Nq newest query rows against a cache of Nk keys).

Each test checks the decode oracle against something other than itself: torch SDPA in float64
with an explicit bottom-right causal mask, and the prefill oracle (pinned in test_oracle.py) on
a sequence whose last rows are the decode rows.  A wrong causal offset, a wrong row or key
index, or a selection taken over the wrong query block fails one of them."""

import numpy as np
import pytest
import torch

import oracle
import workloads


def dec(**kw):
    base = dict(name="d", index=91, B=1, Hq=4, Hkv=2, N=256, d=64, causal=True, block_q=64,
                block_k=32, topk_abs=-1, topk_bp=1000, dist="normal", n_query=3)
    base.update(kw)
    return workloads.Workload(**base)


def _sdpa_bottom_right(q, k, v, tau, causal):
    qq, kk, vv = (torch.from_numpy(np.asarray(a, np.float64)) for a in (q, k, v))
    g = qq.shape[1] // kk.shape[1]
    kk = kk.repeat_interleave(g, dim=1)
    vv = vv.repeat_interleave(g, dim=1)
    nq, nk = qq.shape[2], kk.shape[2]
    vis = torch.ones(nq, nk, dtype=torch.bool)
    if causal:
        vis = torch.arange(nk)[None, :] <= (nk - nq + torch.arange(nq))[:, None]
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=vis, scale=float(tau))
    s = (float(tau) * qq @ kk.transpose(-1, -2)).masked_fill(~vis, float("-inf"))
    return o.numpy(), torch.logsumexp(s, -1).numpy()


@pytest.mark.parametrize("causal,nq", [(True, 1), (True, 5), (False, 3)])
def test_decode_all_fp16_equals_softmax_attention(causal, nq):
    """k = every key block: only the FP16 rounding of P remains; the mask is bottom-right."""
    w = dec(causal=causal, n_query=nq, topk_bp=10000)
    q, k, v = workloads.make_qkv(w)
    assert q.shape == (1, 4, nq, 64) and k.shape == (1, 2, 256, 64)
    r = oracle.decode_forward(w, q, k, v, want_f64=True)
    assert r["sel"].all()
    ref, lse_ref = _sdpa_bottom_right(q, k, v, oracle.softmax_scale(w.d), causal)
    rel = np.linalg.norm(r["out64"] - ref) / np.linalg.norm(ref)
    assert rel < 3e-4
    assert np.abs(r["lse"] - lse_ref).max() < 1e-5


def test_decode_mask_is_bottom_right():
    """With Nq > 1 the first decode row must not see the last keys: dropping them from the
    cache (and the rows that see them) leaves that row unchanged in the softmax reference,
    and the oracle agrees with the reference row by row."""
    w = dec(n_query=4, topk_bp=10000, N=128, block_k=32)
    q, k, v = workloads.make_qkv(w)
    r = oracle.decode_forward(w, q, k, v, want_f64=True)
    tau = oracle.softmax_scale(w.d)
    for row in range(4):
        n_vis = 128 - 4 + row + 1
        ref, _ = _sdpa_bottom_right(q[:, :, row:row + 1], k[:, :, :n_vis], v[:, :, :n_vis], tau, False)
        err = np.abs(r["out64"][:, :, row] - ref[:, :, 0]).max()
        assert err < 2e-3 * np.abs(ref).max()


def _prefill_with_decode_tail(w, nq, seed):
    """A full-length query tensor whose last nq rows are the decode rows and whose amax lies in
    those rows (so that both quantise the decode rows with the same tensor scale)."""
    qd, k, v = workloads.make_qkv(w)
    wp = w.with_shape(n_query=0)
    qp, _, _ = workloads.make_qkv(wp)
    qp = (qp.astype(np.float32) * 0.25).astype(np.float16)
    qp[:, :, -nq:] = qd
    return qp, qd, k, v


@pytest.mark.parametrize("bp", [0, 2500, 10000])
def test_decode_equals_prefill_last_block(bp):
    """Decode of the last query block with that block's selection row equals the prefill
    oracle's output for those rows, bit for bit (same scores, same codes, same merge)."""
    nq = 64
    w = dec(n_query=nq, N=256, block_q=64, block_k=32, topk_bp=bp)
    qp, qd, k, v = _prefill_with_decode_tail(w, nq, 0)
    wp = w.with_shape(n_query=0)
    rp = oracle.forward(wp, qp, k, v, want_f64=True)
    q4d = oracle.quantize_nvfp4(qd, 0)
    assert q4d.tensor_scale == rp["q4"].tensor_scale
    assert np.array_equal(q4d.codes, rp["q4"].codes[:, :, -nq:])
    sel_last = np.ascontiguousarray(rp["sel"][:, :, -1:, :])
    out, lse, o64 = oracle.decode_attn(qd, k, v, q4d, rp["k4"], rp["v4"], sel_last, w.block_k, True,
                                       want_f64=True)
    assert np.array_equal(o64, rp["out64"][:, :, -nq:])
    assert np.array_equal(lse, rp["lse"][:, :, -nq:])
    # the decode selection over the same rows is the prefill selection's last row
    sd = oracle.decode_block_scores(qd, k, w.block_k, True)
    sp = oracle.block_scores(qp, k, wp)
    assert np.array_equal(sd, sp[:, :, -1:, :])


def test_decode_selection_topk_count_and_order():
    """Selection over one query block: k = ceil(bp * nKb / 10000) blocks per head, the largest
    qbar . kbar, with qbar the mean of the decode rows (checked by brute force in numpy)."""
    w = dec(n_query=3, N=512, block_k=32, topk_bp=1500)
    q, k, v = workloads.make_qkv(w)
    s = oracle.decode_block_scores(q, k, w.block_k, True)
    sel, kth, kc = oracle.select(s, w)
    nkb = 512 // 32
    assert (kc == -(-1500 * nkb // 10000)).all()
    qbar = q.astype(np.float64).mean(axis=2)                     # [B, Hq, d]
    kbar = k.astype(np.float64).reshape(1, 2, nkb, 32, 64).mean(axis=3)
    kbar = np.repeat(kbar, 2, axis=1)                            # [B, Hq, nKb, d]
    brute = np.einsum("bhd,bhjd->bhj", qbar, kbar)
    assert np.allclose(s[:, :, 0], brute, rtol=1e-12, atol=1e-12)
    for h in range(4):
        top = np.argsort(-brute[0, h], kind="stable")[:kc[0, h]]
        assert set(np.nonzero(sel[0, h, 0])[0]) == set(top)


def test_decode_single_row_causal_equals_noncausal():
    """The newest row sees every key, so the causal and full forms agree exactly."""
    w = dec(n_query=1, topk_bp=2000)
    q, k, v = workloads.make_qkv(w)
    a = oracle.decode_forward(w, q, k, v, want_f64=True)
    b = oracle.decode_forward(w.with_shape(causal=False), q, k, v, want_f64=True)
    assert np.array_equal(a["out64"], b["out64"]) and np.array_equal(a["lse"], b["lse"])


def test_decode_workloads_shapes():
    w = workloads.WORKLOADS["decode_tiny"]
    q, k, v = workloads.make_qkv(w)
    assert q.shape == (1, 4, 2, 64) and k.shape == (1, 2, 1024, 64) and v.shape == k.shape
    for name in ("decode32k", "decode131k"):
        w = workloads.WORKLOADS[name]
        assert w.is_decode and w.n_query == 1 and w.N % 128 == 0
