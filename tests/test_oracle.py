"""Pins for the CPU oracle: each test checks the oracle against something other than
itself -- values fixed by the pages (the E2M1 grid, the 4.5-bit storage, the block-mean
score), library routines (ml_dtypes FP4/FP8 casts, numpy float16, torch SDPA in float64,
BLAS matmul), closed forms and brute force on tiny inputs."""

import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(float(t) for t in line.split()))
    return rows


def small(**kw):
    base = dict(name="t", index=90, B=1, Hq=2, Hkv=2, N=256, d=64, causal=False, block_q=64,
                block_k=32, topk_abs=-1, topk_bp=1000, dist="normal")
    base.update(kw)
    return workloads.Workload(**base)


# ------------------------------------------------------------------ FP16

def test_half_decode_all_patterns_matches_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle.half_to_double(bits)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_half_encode_matches_numpy_rounding():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.normal(size=200000) * 10.0 ** rng.integers(-9, 5, 200000),
                        np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float64)])
    x = x[np.isfinite(x) & (np.abs(x) < 65504)]
    # exact midpoints between neighbouring halves exercise ties-to-even
    h = np.arange(0x0001, 0x7bff, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (h[:-1] + h[1:]) / 2
    x = np.concatenate([x, mids, -mids])
    assert np.array_equal(oracle.double_to_half(x), x.astype(np.float16).view(np.uint16))


# ------------------------------------------------------------------ E2M1

def test_e2m1_golden_table():
    for x, code in _golden("e2m1_rounding.txt"):
        assert oracle.e2m1_encode([x])[0] == int(code), x


def test_e2m1_grid_has_15_values_and_roundtrips():
    vals = oracle.e2m1_decode(np.arange(16))
    assert len(set(vals.tolist())) == 15
    assert sorted(set(np.abs(vals).tolist())) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for c in range(16):
        assert oracle.e2m1_encode([vals[c]])[0] == (c if c != 8 else 8)


def test_e2m1_matches_ml_dtypes():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.uniform(-8, 8, 300000), rng.normal(size=100000) * 0.3]).astype(np.float32)
    grid = np.array([0, 0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6], np.float32)
    eps = np.float32(1e-6)
    x = np.concatenate([x, grid, -grid, grid + eps, grid - eps, -grid + eps, -grid - eps])
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    assert np.array_equal(oracle.e2m1_encode(x), ref)


# ------------------------------------------------------------------ E4M3

def test_e4m3_decode_all_codes_matches_ml_dtypes():
    codes = np.arange(0x7f, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(oracle.e4m3_decode(codes), ref)
    assert oracle.e4m3_decode([0x7e])[0] == 448.0
    assert oracle.e4m3_decode([0x01])[0] == 2.0 ** -9


def test_e4m3_encode_matches_ml_dtypes_and_saturates():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(0, 448, 200000), 2.0 ** rng.uniform(-14, 8.8, 200000)]).astype(np.float32)
    vals = np.arange(0x7f, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, vals.astype(np.float32)])
    x = x[x <= 448]
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(oracle.e4m3_encode(x), ref)
    assert np.all(oracle.e4m3_encode(np.array([448.5, 464, 1000, 1e30], np.float32)) == 0x7e)
    for c in range(0x7f):
        assert oracle.e4m3_encode([vals[c]])[0] == c


# ------------------------------------------------------------------ NVFP4

def test_nvfp4_storage_is_4_5_bits():
    # 4-bit codes plus one 8-bit scale per 16 elements: 4.5 bits, 28.125 % of FP16 -- the
    # "+28 %" KV-cache growth from keeping an FP4 copy next to the FP16 one (ThriftAttention,
    # "Betekenis en Beweringen").
    x = np.ones((1, 1, 64, 128), np.float16)
    t = oracle.quantize_nvfp4(x, 0)
    bits = 8 * (t.codes.nbytes + t.scales.nbytes) / x.size
    assert bits == 4.5
    assert abs(bits / 16 - 0.28) < 0.002


def test_nvfp4_tensor_amax_maps_to_six():
    rng = np.random.default_rng(4)
    x = rng.normal(size=(2, 3, 64, 64)).astype(np.float16)
    t = oracle.quantize_nvfp4(x, 0)
    amax = np.abs(x.astype(np.float32)).max()
    assert t.tensor_scale == np.float32(amax) / np.float32(2688.0)
    idx = np.unravel_index(np.argmax(np.abs(x.astype(np.float32))), x.shape)
    deq = oracle.dequantize_nvfp4(t)
    codes = np.stack([t.codes & 15, t.codes >> 4], -1).reshape(deq.shape)
    assert codes[idx] & 7 == 7  # the largest element encodes to +-6
    assert abs(deq[idx] - x[idx]) <= 1e-6 * abs(float(x[idx]))


def test_nvfp4_zero_group_and_zero_tensor():
    x = np.zeros((1, 1, 16, 32), np.float16)
    x[0, 0, 3, 16:] = 1.0
    t = oracle.quantize_nvfp4(x, 0)
    assert np.all(t.codes[0, 0, :, :8] == 0) and np.all(t.scales[0, 0, :, 0] == 0)
    z = oracle.quantize_nvfp4(np.zeros((1, 1, 16, 32), np.float16), 0)
    assert z.tensor_scale == 1.0 and not z.codes.any() and not z.scales.any()


def test_nvfp4_error_bound():
    """|x - deq| <= half the E2M1 spacing at x/eff, times eff (or the saturation gap)."""
    rng = np.random.default_rng(5)
    x = (rng.standard_t(3, size=(1, 2, 128, 64)) * 3).astype(np.float16)
    t = oracle.quantize_nvfp4(x, 0)
    deq = oracle.dequantize_nvfp4(t)
    sb = np.repeat(oracle.e4m3_decode(t.scales), 16, axis=-1)
    eff = (sb.astype(np.float32) * t.tensor_scale).astype(np.float64)  # the FP32 divisor
    eff64 = sb * np.float64(t.tensor_scale)                             # the dequantisation scale
    y = np.abs(x.astype(np.float64)) / np.where(eff > 0, eff, 1)
    spacing = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    bound = np.where(y <= 6, 0.5 * spacing, y - 6) * eff * (1 + 1e-6) + 6 * np.abs(eff - eff64) + 1e-30
    assert np.all(np.abs(x.astype(np.float64) - deq) <= bound)


def test_nvfp4_matches_library_codecs():
    """Recompute each group with ml_dtypes' FP8/FP4 casts (independent codecs)."""
    rng = np.random.default_rng(6)
    x = (rng.normal(size=(1, 2, 64, 64)) * np.exp(rng.normal(size=(1, 2, 64, 1)))).astype(np.float16)
    t = oracle.quantize_nvfp4(x, 0)
    xf = x.astype(np.float32).reshape(-1, 16)
    st = np.float32(np.abs(xf).max()) / np.float32(2688)
    amax16 = np.abs(xf).max(axis=1)
    sb = ((amax16 / np.float32(6)) / st).astype(ml_dtypes.float8_e4m3fn)
    eff = sb.astype(np.float32) * st
    codes = (xf / eff[:, None]).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).reshape(t.codes.shape)
    assert np.array_equal(sb.view(np.uint8).reshape(t.scales.shape), t.scales)
    assert np.array_equal(packed, t.codes)


def test_nvfp4_token_axis_is_transpose_of_channel_axis():
    rng = np.random.default_rng(7)
    v = rng.normal(size=(2, 3, 64, 32)).astype(np.float16)
    a = oracle.quantize_nvfp4(v, 1)
    b = oracle.quantize_nvfp4(np.ascontiguousarray(np.swapaxes(v, -1, -2)), 0)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.scales, b.scales)
    assert a.tensor_scale == b.tensor_scale


# ------------------------------------------------------------------ selection

@pytest.mark.parametrize("causal", [False, True])
def test_block_scores_equal_mean_of_token_products(causal):
    w = small(B=2, Hq=4, Hkv=2, N=256, d=32, causal=causal, block_q=64, block_k=32)
    q, k, _ = workloads.make_qkv(w)
    s = oracle.block_scores(q, k, w)
    qd, kd = q.astype(np.float64), k.astype(np.float64)
    for b in range(w.B):
        for h in range(w.Hq):
            full = qd[b, h] @ kd[b, h // 2].T
            for i in range(w.n_qb):
                for j in range(w.n_kb):
                    valid = (not causal) or j * w.block_k <= (i + 1) * w.block_q - 1
                    if not valid:
                        assert s[b, h, i, j] == -np.inf
                        continue
                    ref = full[i * 64:(i + 1) * 64, j * 32:(j + 1) * 32].mean()
                    assert abs(s[b, h, i, j] - ref) <= 1e-12 * max(1.0, abs(ref))


@pytest.mark.parametrize("name,valid,k", [("tiny", 64, 4), ("n4k", 2048, 103),
                                          ("prefill32k", 65792, 3290), ("long131k", 524800, 10496)])
def test_valid_pair_counts_and_budget(name, valid, k):
    w = workloads.WORKLOADS[name]
    L = oracle.lib()
    nv = sum(L.orc_pair_valid(int(w.causal), i, j, w.block_q, w.block_k)
             for i in range(w.n_qb) for j in range(w.n_kb)) if w.N <= 32768 else None
    if nv is not None:
        assert nv == valid
    # closed forms: causal 128x64 -> sum_i (2i + 2); causal 128x128 -> sum_i (i + 1)
    assert oracle.topk_count(valid, w.topk_abs, w.topk_bp) == k


def test_diffusion_budget_sweep_counts():
    assert [oracle.topk_count(32768, -1, bp) for bp in workloads.DIFFUSION_BUDGETS_BP] == \
        [0, 328, 1639, 6554, 32768]


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(8)
    for trial in range(200):
        nqb, nkb = rng.integers(1, 6), rng.integers(1, 9)
        s = rng.integers(-3, 4, size=(1, 1, nqb, nkb)).astype(np.float64)  # many ties
        s[rng.random(s.shape) < 0.2] = -np.inf
        bp = int(rng.integers(0, 10001))
        w = small(topk_bp=bp)
        sel, kth, kc = oracle.select(s, w)
        flat = s.reshape(-1)
        valid = [t for t in range(flat.size) if np.isfinite(flat[t])]
        k = math.ceil(bp * len(valid) / 10000)
        chosen = sorted(valid, key=lambda t: (-flat[t], t))[:k]
        exp = np.zeros(flat.size, np.uint8)
        exp[chosen] = 1
        assert kc[0, 0] == k
        assert np.array_equal(sel.reshape(-1), exp)


# ------------------------------------------------------------------ attention

def _sdpa(q, k, v, tau, causal):
    qq, kk, vv = (torch.from_numpy(np.asarray(a, np.float64)) for a in (q, k, v))
    g = qq.shape[1] // kk.shape[1]
    kk = kk.repeat_interleave(g, dim=1)
    vv = vv.repeat_interleave(g, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=float(tau), is_causal=causal)
    s = float(tau) * qq @ kk.transpose(-1, -2)
    if causal:
        n = s.shape[-1]
        s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    return o.numpy(), torch.logsumexp(s, -1).numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_all_fp16_equals_softmax_attention(causal):
    """k = all pairs: only the FP16 rounding of P remains (ThriftAttention "FP16-pad")."""
    w = small(B=1, Hq=4, Hkv=2, N=256, d=64, causal=causal, block_q=64, block_k=32, topk_bp=10000)
    q, k, v = workloads.make_qkv(w)
    r = oracle.forward(w, q, k, v, want_f64=True)
    assert r["sel"][np.isfinite(r["scores"])].all()
    ref, lse_ref = _sdpa(q, k, v, oracle.softmax_scale(w.d), causal)
    rel = np.linalg.norm(r["out64"] - ref) / np.linalg.norm(ref)
    assert rel < 3e-4
    assert np.abs(r["lse"] - lse_ref).max() < 1e-5
    assert np.array_equal(r["out"].view(np.uint16), oracle.double_to_half(r["out64"]).reshape(r["out"].shape))


@pytest.mark.parametrize("fp16", [False, True])
def test_tile_scores_exact(fp16):
    """FP4 scores are exact sums of dequantised products; equal to a float64 BLAS matmul."""
    w = small(B=1, Hq=4, Hkv=2, N=256, d=64, causal=True, block_q=64, block_k=32)
    q, k, _ = workloads.make_qkv(w)
    q4, k4 = oracle.quantize_nvfp4(q, 0), oracle.quantize_nvfp4(k, 0)
    tau = oracle.softmax_scale(w.d)
    if fp16:
        qd, kd, mult = q.astype(np.float64), k.astype(np.float64), float(tau)
    else:
        qd = oracle.dequantize_nvfp4(q4) / float(q4.tensor_scale)
        kd = oracle.dequantize_nvfp4(k4) / float(k4.tensor_scale)
        mult = float(q4.tensor_scale) * float(k4.tensor_scale) * float(tau)
    for (h, i, j) in [(0, 0, 0), (1, 2, 3), (3, 3, 6), (2, 1, 3)]:
        S = oracle.tile_scores(q, k, q4, k4, w, tau, 0, h, i, j, fp16)
        ref = (qd[0, h, i * 64:(i + 1) * 64] @ kd[0, h // 2, j * 32:(j + 1) * 32].T) * mult
        rows = np.arange(i * 64, (i + 1) * 64)[:, None]
        keys = np.arange(j * 32, (j + 1) * 32)[None, :]
        ref = np.where(keys > rows, -np.inf, ref)
        if fp16:
            fin = np.isfinite(ref)
            assert np.all(np.abs(S[fin] - ref[fin]) <= 1e-12 * np.abs(ref[fin]).max())
            assert np.array_equal(np.isfinite(S), fin)
        else:
            assert np.array_equal(S, ref)


def test_pq_golden_powers_of_two():
    S = np.full(16, -np.inf)
    rows = _golden("pq_powers_of_two.txt")
    for kk, _ in rows:
        S[int(kk)] = -kk * math.log(2.0)
    M, sumP, Pq = oracle.tile_pq(S, fp16=False)
    assert M == 0.0
    assert sumP == sum(2.0 ** -kk for kk, _ in rows)
    for kk, exp in rows:
        assert Pq[int(kk)] == pytest.approx(exp, rel=0, abs=1e-15)
    assert np.all(Pq[len(rows):] == 0)


def test_pq_bounds_and_row_max():
    rng = np.random.default_rng(9)
    for trial in range(300):
        bk = int(rng.choice([16, 32, 64, 128]))
        S = rng.normal(size=bk) * rng.uniform(0.1, 8)
        S[rng.random(bk) < 0.1] = -np.inf
        if not np.isfinite(S).any():
            continue
        for fp16 in (False, True):
            M, sumP, Pq = oracle.tile_pq(S, fp16)
            ph = np.where(np.isfinite(S), np.exp(S - M).astype(np.float32), 0).astype(np.float64)
            assert sumP == pytest.approx(ph.sum(), rel=1e-15)
            if fp16:
                assert np.all(np.abs(Pq - ph) <= ph * 2.0 ** -11 + 2.0 ** -25)
                continue
            assert Pq[np.argmax(S)] == 1.0  # the block-row maximum maps to 6 * 448 / 2688
            for g in range(bk // 16):
                p = ph[g * 16:(g + 1) * 16]
                sb = oracle.e4m3_decode(oracle.e4m3_encode([np.float32(2688 * p.max()) / np.float32(6)]))[0]
                if sb == 0:  # the group lies below the smallest E4M3 scale: all codes 0
                    assert np.all(Pq[g * 16:(g + 1) * 16] == 0)
                    assert p.max() <= 6 * 2.0 ** -10 / 2688 * (1 + 1e-6)
                    continue
                y = 2688 * p / sb
                spacing = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
                bound = np.where(y <= 6, 0.5 * spacing, y - 6) * sb / 2688 * (1 + 1e-6) + 1e-300
                assert np.all(np.abs(Pq[g * 16:(g + 1) * 16] - p) <= bound)


@pytest.mark.parametrize("causal,bp", [(False, 0), (True, 0), (True, 2000), (False, 10000)])
def test_block_constant_keys_closed_form(causal, bp):
    """With every K row constant inside its key block, each block's scores are constant per
    row, exp(S - M) = 1 on the valid keys, both P quantisers are exact, and the output is the
    closed form O_r = sum_j e^{s_rj - m} sum_t V_t / sum_j e^{s_rj - m} n_rj, with s_rj
    the pair's score in its own precision and V in its own precision."""
    w = small(B=1, Hq=4, Hkv=2, N=256, d=64, causal=causal, block_q=64, block_k=32, topk_bp=bp)
    q, k, v = workloads.make_qkv(w)
    k = np.repeat(k[:, :, ::32, :], 32, axis=2).copy()  # one key per block, repeated
    r = oracle.forward(w, q, k, v, want_f64=True)
    tau = float(oracle.softmax_scale(w.d))
    q4, k4, v4 = r["q4"], r["k4"], r["v4"]
    qd4 = oracle.dequantize_nvfp4(q4)
    kd4 = oracle.dequantize_nvfp4(k4)
    vd4 = np.swapaxes(oracle.dequantize_nvfp4(v4), -1, -2)
    out = np.zeros_like(r["out64"])
    for h in range(w.Hq):
        hk = h // 2
        for row in range(w.N):
            i = row // 64
            num = np.zeros(w.d)
            terms = []
            for j in range(w.n_kb):
                keys = np.arange(j * 32, (j + 1) * 32)
                if causal:
                    keys = keys[keys <= row]
                if keys.size == 0 or (causal and j * 32 > (i + 1) * 64 - 1):
                    continue
                if r["sel"][0, h, i, j]:
                    s = tau * float(q[0, h, row].astype(np.float64) @ k[0, hk, j * 32].astype(np.float64))
                    vs = v[0, hk, keys].astype(np.float64).sum(0)
                else:
                    s = tau * float(qd4[0, h, row] @ kd4[0, hk, j * 32])
                    vs = vd4[0, hk, keys].sum(0)
                terms.append((s, vs, keys.size))
            m = max(t[0] for t in terms)
            den = sum(math.exp(s - m) * n for s, _, n in terms)
            num = sum(math.exp(s - m) * vs for s, vs, _ in terms)
            out[0, h, row] = num / den
    assert np.abs(r["out64"] - out).max() <= 1e-12 * np.abs(out).max()


@pytest.mark.parametrize("bp", [0, 1000, 10000])
def test_online_merge_equals_two_pass(bp):
    w = small(B=1, Hq=2, Hkv=1, N=512, d=64, causal=True, block_q=64, block_k=32, topk_bp=bp)
    q, k, v = workloads.make_qkv(w)
    r = oracle.forward(w, q, k, v, want_f64=True)
    order = np.random.default_rng(10).permutation(w.n_kb)
    _, lse, o64 = oracle.attn(q, k, v, r["q4"], r["k4"], r["v4"], r["sel"], w, online=True,
                              order=order, want_f64=True)
    assert np.abs(o64 - r["out64"]).max() <= 1e-9 * np.abs(r["out64"]).max()
    assert np.abs(lse - r["lse"]).max() <= 1e-5


def test_rows_of_p_sum_to_one():
    """exp(lse) is the softmax denominator: sum_t exp(S_t - lse) = 1 for k = all."""
    w = small(B=1, Hq=2, Hkv=2, N=256, d=64, causal=True, topk_bp=10000)
    q, k, v = workloads.make_qkv(w)
    r = oracle.forward(w, q, k, v)
    s = float(oracle.softmax_scale(w.d)) * q[0].astype(np.float64) @ np.swapaxes(k[0].astype(np.float64), -1, -2)
    s = np.where(np.triu(np.ones((w.N, w.N), bool), 1), -np.inf, s)
    tot = np.exp(s - r["lse"][0][..., None].astype(np.float64)).sum(-1)
    assert np.abs(tot - 1).max() < 1e-6 * math.log(w.N) * 10


def test_denominator_sums_unquantised_probabilities():
    """Reading R1: the softmax denominator sums the unquantised exp(S - M), not the re-quantised
    probabilities.  Keys alternate between two levels (c = 1 and c = 1/2, both exact in NVFP4),
    so every 16-key group holds a block maximum (code 6, scale 448) and keys whose probability
    r = exp(S_low - S_high) ~ 0.059 re-quantises to the E2M1 value 0.5 (dequantised 1/12): the
    two denominators differ by ~2 %, far above the oracle's rounding.  The lse and output are
    derived here from a float64 matmul of the dequantised inputs and the E2M1 grid."""
    w = small(B=1, Hq=1, Hkv=1, N=64, d=32, causal=False, block_q=64, block_k=32, topk_bp=0)
    q = np.ones((1, 1, 64, 32), np.float16)
    c = np.where(np.arange(64) % 2 == 0, 1.0, 0.5).astype(np.float16)
    k = np.repeat(c[None, None, :, None], 32, axis=3).astype(np.float16)
    v = workloads.make_qkv(w)[2]
    r = oracle.forward(w, q, k, v, want_f64=True)
    qd = oracle.dequantize_nvfp4(r["q4"])[0, 0]
    kd = oracle.dequantize_nvfp4(r["k4"])[0, 0]
    vd = np.swapaxes(oracle.dequantize_nvfp4(r["v4"]), -1, -2)[0, 0]
    tau = float(oracle.softmax_scale(w.d))
    S = tau * (qd @ kd.T)                                    # [64 rows, 64 keys]
    M = S.max(1, keepdims=True)                              # the same in both key blocks
    ph = np.exp(S - M).astype(np.float32).astype(np.float64)  # P^ in FP32
    assert np.all(np.isin(ph, [1.0, ph[0, 1]])) and 0.05 < ph[0, 1] < 0.07
    y = 6.0 * ph                                             # P' / s_b with s_b = 448 in every group
    pq = np.where(ph == 1.0, 6.0, 0.5) * 448 / 2688          # E2M1(6) = 6, E2M1(0.35) = 0.5
    assert np.all(np.abs(y - np.where(ph == 1.0, 6.0, 0.5)) < 0.2)
    lse = (M[:, 0] + np.log(ph.sum(1))).astype(np.float32)
    lse_wrong = (M[:, 0] + np.log(pq.sum(1))).astype(np.float32)
    assert np.abs(lse - lse_wrong).min() > 1e-2              # the two readings are far apart
    assert np.abs(r["lse"][0, 0] - lse).max() <= 1e-6
    out = (pq @ vd) / ph.sum(1, keepdims=True)
    assert np.abs(r["out64"][0, 0] - out).max() <= 1e-12 * np.abs(out).max()
