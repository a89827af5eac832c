"""Pins for the oracle's reading of appending to the double cache (reading R-append): the cache
keeps the tensor scales it was built with and encodes appended tokens with them, and a decode
step sees only the first n_valid keys of a cache of capacity Nk (a partly filled last key block
averages the keys it holds for the selection, and its other keys are masked)."""

import numpy as np
import pytest
import torch

import oracle
import workloads


def small_decode(**kw):
    base = dict(name="t", index=91, B=1, Hq=4, Hkv=2, N=512, d=64, causal=True, block_q=128, block_k=64,
                topk_abs=-1, topk_bp=2500, dist="normal", n_query=2)
    base.update(kw)
    return workloads.Workload(**base)


def padded(x, n_valid):
    y = x.copy()
    y[:, :, n_valid:, :] = 0
    return y


def test_scaled_quantiser_equals_own_scale_and_saturates():
    w = small_decode()
    _, k, v = workloads.make_qkv(w)
    for axis, x in ((0, k), (1, v)):
        own = oracle.quantize_nvfp4(x, axis)
        fixed = oracle.quantize_nvfp4(x, axis, tensor_scale=own.tensor_scale)
        assert np.array_equal(own.codes, fixed.codes) and np.array_equal(own.scales, fixed.scales)
    # a cache built from values of at most 1 (scale 1/2688) meets a value of 4: its group scale
    # saturates at the E4M3 maximum 448 and the value at the E2M1 maximum 6 (it reads back as 1)
    x = np.zeros((1, 1, 16, 16), np.float16)
    x[0, 0, 0, :] = 1.0
    x[0, 0, 1, 0] = 4.0
    t = oracle.quantize_nvfp4(x, 0, tensor_scale=np.float32(1.0) / np.float32(2688.0))
    assert oracle.e4m3_decode(t.scales[0, 0, 1, :1])[0] == 448.0
    assert (t.codes[0, 0, 1, 0] & 15) == 7  # E2M1 code of +6
    assert oracle.dequantize_nvfp4(t)[0, 0, 1, 0] == pytest.approx(1.0, rel=1e-6)


def test_full_valid_length_is_the_plain_decode():
    w = small_decode()
    q, k, v = workloads.make_qkv(w)
    a = oracle.decode_forward(w, q, k, v, want_f64=True)
    b = oracle.decode_forward(w, q, k, v, want_f64=True, n_valid=w.N)
    assert np.array_equal(a["sel"], b["sel"]) and np.array_equal(a["out64"], b["out64"])


@pytest.mark.parametrize("bp", [0, 2500, 10000])
def test_block_aligned_valid_length_equals_truncated_cache(bp):
    """With n_valid a multiple of the key block, the capacity-padded cache decodes exactly as the
    cache cut at n_valid (same NVFP4 codes below n_valid, same scales)."""
    w = small_decode(topk_bp=bp)
    q, k, v = workloads.make_qkv(w)
    nv = 320
    kp, vp = padded(k, nv), padded(v, nv)
    k4, v4 = oracle.quantize_nvfp4(kp, 0), oracle.quantize_nvfp4(vp, 1)
    full = oracle.decode_forward(w, q, kp, vp, k4=k4, v4=v4, want_f64=True, n_valid=nv)
    k4t = oracle.NVFP4(k4.codes[:, :, :nv].copy(), k4.scales[:, :, :nv].copy(), k4.tensor_scale, 0)
    v4t = oracle.NVFP4(v4.codes[..., :nv // 2].copy(), v4.scales[..., :nv // 16].copy(), v4.tensor_scale, 1)
    wt = w.with_shape(N=nv)
    cut = oracle.decode_forward(wt, q, kp[:, :, :nv].copy(), vp[:, :, :nv].copy(), k4=k4t, v4=v4t,
                                want_f64=True)
    assert np.array_equal(full["sel"][..., :nv // 64], cut["sel"])
    assert not full["sel"][..., nv // 64:].any()
    assert np.array_equal(full["out64"], cut["out64"])
    assert np.array_equal(full["lse"], cut["lse"])


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("nv", [257, 300, 447])
def test_ragged_all_fp16_equals_sdpa_over_valid_keys(causal, nv):
    w = small_decode(topk_bp=10000, causal=causal)
    q, k, v = workloads.make_qkv(w)
    r = oracle.decode_forward(w, q, padded(k, nv), padded(v, nv), want_f64=True, n_valid=nv)
    tau = float(oracle.softmax_scale(w.d))
    qq = torch.from_numpy(q.astype(np.float64))
    kk = torch.from_numpy(k[:, :, :nv].astype(np.float64)).repeat_interleave(2, 1)
    vv = torch.from_numpy(v[:, :, :nv].astype(np.float64)).repeat_interleave(2, 1)
    s = tau * qq @ kk.transpose(-1, -2)
    if causal:  # query row r at position nv - Nq + r
        pos = nv - w.n_query + torch.arange(w.n_query)[:, None]
        s = s.masked_fill(torch.arange(nv)[None, :] > pos, float("-inf"))
    ref = torch.softmax(s, -1) @ vv
    rel = np.linalg.norm(r["out64"] - ref.numpy()) / np.linalg.norm(ref.numpy())
    assert rel < 3e-4
    assert np.abs(r["lse"] - torch.logsumexp(s, -1).numpy()).max() < 1e-5


def test_partial_block_mean_and_budget():
    w = small_decode(topk_bp=5000)
    q, k, v = workloads.make_qkv(w)
    nv = 300  # blocks 0..3 full, block 4 holds 44 keys, blocks 5..7 empty
    kp = padded(k, nv)
    sc = oracle.decode_block_scores(q, kp, w.block_k, True, nv)
    qbar = q.astype(np.float64).mean(2)
    for h in range(w.Hq):
        kb = kp[0, h // 2].astype(np.float64)
        for j in range(8):
            if j * 64 >= nv:
                assert sc[0, h, 0, j] == -np.inf
                continue
            kbar = kb[j * 64:min((j + 1) * 64, nv)].mean(0)
            assert sc[0, h, 0, j] == pytest.approx(float(qbar[0, h] @ kbar), rel=1e-13)
    sel, _, kc = oracle.select(sc, w)
    assert np.all(kc == 3)  # ceil(5000 * 5 / 10000) of the 5 valid blocks
    assert not sel[..., 5:].any()
