"""Pins for the oracle's reading R2 of the two-level P quantisation: the first level is the row's
running maximum in the fused kernel's visiting order (NVFP4 key blocks in ascending order, then
the FP16 ones), so a block whose maximum lies below the running maximum re-quantises exp(S - m)
with a group scale below 448 (ThriftAttention summary, "Methodologie", "Online Samenvoeging": a
two-level quantisation of the probability blocks adapted from SageAttention3, inside an online
softmax; the running maximum of that online softmax is taken as the first level).

Each test checks the oracle against a closed form built from library casts (ml_dtypes E4M3/E2M1,
numpy float16), torch SDPA in float64, or the R1 oracle where the two readings coincide."""

import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads


def small(**kw):
    base = dict(name="t", index=91, B=1, Hq=2, Hkv=2, N=256, d=64, causal=False, block_q=64,
                block_k=32, topk_abs=-1, topk_bp=1000, dist="normal")
    base.update(kw)
    return workloads.Workload(**base)


def _quantised(w, q, k, v):
    return oracle.quantize_nvfp4(q, 0), oracle.quantize_nvfp4(k, 0), oracle.quantize_nvfp4(v, 1)


def _nvfp4_requant(ph):
    """One 16-key group of equal probabilities ph (FP32): E4M3 group scale of 2688 ph / 6, E2M1
    code of 2688 ph / scale, dequantised back to probability units (library casts only)."""
    p = np.float32(2688) * np.float32(ph)
    sb = float(np.array([p / np.float32(6)], np.float32).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)[0])
    code = float(np.array([p / np.float32(sb)], np.float32).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)[0])
    return code * sb / 2688.0


@pytest.mark.parametrize("a0,a1", [(1.0, 0.5), (0.5, 1.0)])
@pytest.mark.parametrize("sel0,sel1", [(0, 0), (1, 0), (0, 1), (1, 1)])
def test_two_constant_blocks_closed_form(a0, a1, sel0, sel1):
    """Two key blocks whose K rows are constant (a0, a1 in every channel, exact in NVFP4), Q all
    ones, V rows +1 in block 0 and -1/2 in block 1: every score of block j is s_j, exp(S - m) is
    1 on the block that holds the running maximum, and the other block's probability
    r = exp(s_low - s_high) is re-quantised at the running maximum only when it is visited
    second.  The visiting order (NVFP4 blocks first) decides which: e.g. a high NVFP4 block 0
    followed by a low NVFP4 block 1 gives the E4M3-rounded r, while a low FP16 block 0 visited
    after a high NVFP4 block 1 gives the FP16-rounded r."""
    w = small(B=1, Hq=1, Hkv=1, N=64, d=64, block_q=64, block_k=32, topk_bp=0)
    a = np.array([a0] * 32 + [a1] * 32, np.float16)
    q = np.ones((1, 1, 64, 64), np.float16)
    k = np.repeat(a[None, None, :, None], 64, axis=3).astype(np.float16)
    v = np.repeat(np.array([1.0] * 32 + [-0.5] * 32, np.float16)[None, None, :, None], 64, axis=3)
    q4, k4, v4 = _quantised(w, q, k, v)
    sel = np.array([sel0, sel1], np.uint8).reshape(1, 1, 1, 2)
    tau = 0.125
    qd = oracle.dequantize_nvfp4(q4)[0, 0, 0]
    kd = oracle.dequantize_nvfp4(k4)[0, 0]
    vd = np.swapaxes(oracle.dequantize_nvfp4(v4), -1, -2)[0, 0]
    s, vv = [], []
    for j, sj in enumerate((sel0, sel1)):
        if sj:
            s.append(tau * float(np.float64(q[0, 0, 0]) @ np.float64(k[0, 0, 32 * j])))
            vv.append(float(v[0, 0, 32 * j, 0]))
        else:
            s.append(tau * float(qd @ kd[32 * j]))
            vv.append(float(vd[32 * j, 0]))
    first, second = sorted((0, 1), key=lambda j: ((sel0, sel1)[j], j))
    if s[second] >= s[first]:  # the second block raises the running maximum: both exact
        alpha = math.exp(s[first] - s[second])
        num, den, m = alpha * vv[first] + vv[second], alpha + 1.0, s[second]
    else:
        ph = float(np.float32(math.exp(s[second] - s[first])))
        pq = float(np.float16(ph)) if (sel0, sel1)[second] else _nvfp4_requant(ph)
        num, den, m = vv[first] + pq * vv[second], 1.0 + ph, s[first]
    exp_o = num / den
    out, lse, o64 = oracle.attn_r2(q, k, v, q4, k4, v4, sel, w, tau=np.float32(tau), want_f64=True)
    assert np.all(np.abs(o64[0, 0] - exp_o) <= 1e-12)
    assert np.all(np.abs(lse[0, 0] - (m + math.log(32 * den))) <= 1e-5)
    # R1 differs exactly when an NVFP4 block is re-quantised below the running maximum
    _, _, o64_r1 = oracle.attn(q, k, v, q4, k4, v4, sel, w, tau=np.float32(tau), want_f64=True)
    differs = s[second] < s[first] and not (sel0, sel1)[second]
    assert (np.abs(o64_r1 - o64).max() > 1e-5) == differs


@pytest.mark.parametrize("bp", [0, 5000, 10000])
def test_single_key_block_equals_r1(bp):
    """With one key block per row the running maximum is the block maximum: R2 = R1."""
    w = small(B=1, Hq=2, Hkv=1, N=64, d=64, block_q=64, block_k=64, topk_abs=-1, topk_bp=bp)
    q, k, v = workloads.make_qkv(w)
    r = oracle.forward(w, q, k, v, want_f64=True)
    _, lse, o64 = oracle.attn_r2(q, k, v, r["q4"], r["k4"], r["v4"], r["sel"], w, want_f64=True)
    assert np.abs(o64 - r["out64"]).max() <= 1e-12 * np.abs(r["out64"]).max()
    assert np.abs(lse - r["lse"]).max() <= 1e-6


@pytest.mark.parametrize("causal", [False, True])
def test_all_fp16_equals_softmax_attention(causal):
    """k = all pairs: P^ = exp(S - m) rounded to FP16 (relative error <= 2^-11) is all that
    remains, whatever the first level: float64 SDPA on the FP16 inputs."""
    w = small(B=1, Hq=4, Hkv=2, N=256, d=64, causal=causal, block_q=64, block_k=32, topk_bp=10000)
    q, k, v = workloads.make_qkv(w)
    q4, k4, v4 = _quantised(w, q, k, v)
    sel = np.ones((1, 4, w.n_qb, w.n_kb), np.uint8)
    out, lse, o64 = oracle.attn_r2(q, k, v, q4, k4, v4, sel, w, want_f64=True)
    tau = float(oracle.softmax_scale(w.d))
    qq, kk, vv = (torch.from_numpy(x.astype(np.float64)) for x in (q, k, v))
    kk, vv = kk.repeat_interleave(2, 1), vv.repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=tau, is_causal=causal).numpy()
    assert np.linalg.norm(o64 - ref) / np.linalg.norm(ref) < 3e-4
    assert np.array_equal(out.view(np.uint16), oracle.double_to_half(o64).reshape(out.shape))


@pytest.mark.parametrize("bp", [0, 1000])
def test_error_within_requantisation_bound(bp):
    """Against the exact softmax of the same scores (FP16 pairs from the FP16 inputs, NVFP4 pairs
    from the dequantised ones, float64), each output element errs by at most
    sum_t |Pq_t - P^_t| |V_t| / l: per 16-key group whose running maximum is m, the E2M1 code
    errs by half a grid step (at most 1 code unit) times the E4M3 scale, i.e. by at most
    (1 + 2^-4) max_g P^ / 6, and an FP16 P^ by 2^-11 P^; l is the exact denominator at m."""
    w = small(B=1, Hq=2, Hkv=1, N=256, d=64, causal=True, block_q=64, block_k=32, topk_bp=bp)
    q, k, v = workloads.make_qkv(w)
    r = oracle.forward(w, q, k, v, want_f64=True)
    sel = r["sel"]
    _, _, o64 = oracle.attn_r2(q, k, v, r["q4"], r["k4"], r["v4"], sel, w, want_f64=True)
    tau = float(oracle.softmax_scale(w.d))
    qd = oracle.dequantize_nvfp4(r["q4"])[0]
    kd = oracle.dequantize_nvfp4(r["k4"])[0]
    vd = np.swapaxes(oracle.dequantize_nvfp4(r["v4"]), -1, -2)[0]
    for h in range(w.Hq):
        hk = h // 2
        s16 = tau * q[0, h].astype(np.float64) @ k[0, hk].astype(np.float64).T
        s4 = tau * qd[h] @ kd[hk].T
        for row in range(w.N):
            i = row // 64
            pair16 = np.repeat(sel[0, h, i].astype(bool), 32)
            srow = np.where(pair16, s16[row], s4[row])
            vrow = np.where(pair16[:, None], v[0, hk].astype(np.float64), vd[hk])
            srow[row + 1:] = -np.inf
            m = srow.max()
            p = np.exp(srow - m)
            exact = p @ vrow / p.sum()
            # per-key bound at the final maximum (a group visited at a lower running maximum has
            # a smaller absolute error after the rescale, so the bound at m covers it)
            bnd = np.zeros(w.N)
            for g in range(w.N // 16):
                sl = slice(16 * g, 16 * g + 16)
                if pair16[16 * g]:
                    bnd[sl] = 2.0 ** -11 * p[sl] + 1e-30
                else:
                    bnd[sl] = (1 + 2.0 ** -4) * p[sl].max() / 6 + 6 * 2.0 ** -10 / 2688
            err_bound = (bnd @ np.abs(vrow)) / p.sum() + 1e-3 * np.abs(exact).max() * 2.0 ** -10
            assert np.all(np.abs(o64[0, h, row] - exact) <= err_bound * 1.01 + 1e-12), (h, row)
