"""Host arithmetic of bench.py on CPU: the valid-pair counts and budgets of the workloads, the
effective-FLOP convention, and the algorithmic bytes of a decode step."""

import os
import sys

import numpy as np
import pytest

import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("name,valid", [("tiny", 64), ("n4k", 2048), ("prefill32k", 65792),
                                        ("long131k", 524800), ("diffusion", 32768)])
def test_valid_pairs_per_head(name, valid):
    """Valid (query block, key block) pairs per head of each workload: non-causal nQb * nKb;
    causal, key block j valid for query block i when j * bk <= (i + 1) * bq - 1."""
    w = workloads.WORKLOADS[name]
    assert bench.valid_pairs_per_head(w) == valid
    if w.causal:  # brute force over the pairs
        brute = sum(1 for i in range(w.n_qb) for j in range(w.n_kb)
                    if j * w.block_k <= (i + 1) * w.block_q - 1)
        assert brute == valid


@pytest.mark.parametrize("name", ["tiny", "n4k", "prefill16k"])
def test_unit_flops_sum_to_effective_flops(name):
    """The per-unit effective FLOPs (used by the oracle's sampled timing) add up to the whole
    problem's 4 B Hq N^2 d (halved, with the diagonal counted, when causal)."""
    w = workloads.WORKLOADS[name]
    total = w.B * w.Hq * sum(bench.unit_effective_flops(w, i) for i in range(w.n_qb))
    f = bench.effective_flops(w)
    if w.causal:  # sum over rows of (row + 1) keys = N (N + 1) / 2, against the N^2 / 2 convention
        assert total == pytest.approx(4.0 * w.B * w.Hq * w.d * w.N * (w.N + 1) / 2)
        assert total / f == pytest.approx(1 + 1 / w.N)
    else:
        assert total == f


def test_decode_bytes_by_hand():
    """One KV head with two query heads and four 64-key blocks: block 0 selected by both heads
    (FP16 only), block 1 by one head (both copies), blocks 2 and 3 by none (NVFP4 only)."""
    w = workloads.WORKLOADS["decode_tiny"].with_shape(B=1, Hq=2, Hkv=1, N=256, d=64, block_k=64)
    bits = np.zeros((1, 2, 4), bool)
    bits[0, :, 0] = True
    bits[0, 0, 1] = True
    total, b4, b16 = bench.decode_bytes(w, bits)
    assert (b4, b16) == (3, 2)
    per4 = 2 * 64 * 64 * (1 / 2 + 1 / 16)   # K and V codes + E4M3 scales of one block
    per16 = 2 * 64 * 64 * 2                 # FP16 K and V of one block
    kbar = 1 * 1 * 4 * 64 * 8               # key block means read by the selection
    assert total == 3 * per4 + 2 * per16 + kbar


def test_max_over_ranks_is_identity_for_one_process():
    import torch
    assert bench.max_over_ranks([3.0, 1.0], torch.device("cpu"), None) == [3.0, 1.0]


def test_elementwise_bound_balances_the_pipes():
    """With rates R_m (MUFU) and R_f (FMA) per SM clock, E exponentials and F = E (2 + d / bk)
    FMA-pipe operations, and c FMA operations per polynomial exponential, the balanced split puts
    x = (E R_f - F R_m) / (R_f + c R_m) exponentials on the FMA pipe; both pipes then take
    (E - x) / R_m cycles.  Worked by hand for d = 128, bk = 64 (F = 4 E), R_m = 16, R_f = 128,
    c = 8: x = E (128 - 64) / 256 = E / 4, time = 0.75 E / 16 cycles per SM."""
    e = 1.0e6
    r = bench.elementwise_bound(e, 128, 64, 16.0, 128.0, 1, 1000.0, poly_fma_ops=8)
    assert r["poly_share"] == pytest.approx(0.25)
    assert r["ms"] == pytest.approx(0.75 * e / 16 / 1e9 * 1e3)
    # the FMA side of the balance takes the same time
    assert (4 * e + 8 * 0.25 * e) / 128 == pytest.approx(0.75 * e / 16)
    # a very slow MUFU pushes every exponential to the polynomial, a very fast one none
    assert bench.elementwise_bound(e, 128, 64, 1e-6, 128.0, 1, 1000.0)["poly_share"] == pytest.approx(1.0, rel=1e-6)
    assert bench.elementwise_bound(e, 128, 64, 1e6, 128.0, 1, 1000.0)["poly_share"] == 0.0
    # the 32K prefill's elements: 2,105,344 valid 128x64 pairs
    assert bench.valid_pairs_per_head(workloads.WORKLOADS["prefill32k"]) * 32 * 128 * 64 == 2105344 * 8192


@pytest.mark.parametrize("causal", [False, True])
def test_reference_rows_equal_float64_sdpa(causal):
    import torch
    w = workloads.WORKLOADS["tiny"].with_shape(B=1, Hq=4, Hkv=2, N=256, d=64, block_k=64, causal=causal)
    q, k, v = workloads.make_qkv(w)
    tau = 0.125
    units = [(0, 0, 0), (0, 3, w.n_qb - 1), (0, 1, 1)]
    got = bench.reference_rows(q, k, v, w, units, tau)
    qq, kk, vv = (torch.from_numpy(x.astype(np.float64)) for x in (q, k, v))
    kk, vv = kk.repeat_interleave(2, 1), vv.repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=tau, is_causal=w.causal).numpy()
    exp = np.concatenate([ref[b, h, i * w.block_q:(i + 1) * w.block_q] for (b, h, i) in units])
    assert np.abs(got - exp).max() <= 1e-12 * np.abs(exp).max()


def test_gap_recovery():
    assert bench.gap_recovery(0.1, 0.01) == pytest.approx(0.9)
    assert bench.gap_recovery(0.1, 0.1) == 0.0
    assert bench.gap_recovery(0.0, 0.0) == 0.0
