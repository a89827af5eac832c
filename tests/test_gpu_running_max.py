"""The running-maximum reading of the two-level P requantisation (thrift_attn_fwd_running_max;
ThriftAttention summary, "Methodologie", "Online Samenvoeging": a two-level scheme for the
probability blocks adapted from SageAttention3): the CUDA path against
the oracle's reading R2 (first level = the row's running maximum in the kernel's visiting order,
NVFP4 key blocks ascending then FP16 ones), to the same bar as thrift_attn_fwd against R1: rel-L2
<= 1e-3, max-abs <= 1e-2 (one FP16 step where that is larger), LSE within 1e-3."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from test_gpu_parity import compare_attention, gpu_qkv, oracle_quant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pab(cuda_device):
    from precision_attention_block_b200 import build
    build.build()
    import precision_attention_block_b200 as pab
    pab.load()
    return pab


def run_r2(pab, name, bp=None, n_units=None):
    d = oracle_quant(name)
    w = d["w"] if bp is None else d["w"].with_budget(bp)
    gq, gk, gv = gpu_qkv(name)
    cfg = pab.Config.from_workload(w)
    q4, k4, v4 = pab.quantize_qkv(gq, gk, gv)
    sel = pab.block_select(gq, gk, cfg)
    out_g, lse_g = pab.attn_fwd(gq, gk, gv, q4, k4, v4, sel, cfg, running_max=True)
    out_r1, _ = pab.attn_fwd(gq, gk, gv, q4, k4, v4, sel, cfg)
    torch.cuda.synchronize()
    scores = d["scores"] if bp is None else oracle.block_scores(d["q"], d["k"], w)
    sel_o, _, _ = oracle.select(scores, w)
    if n_units is None:
        units = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.n_qb)]
    else:
        units = workloads.sample_units(w, n_units)
    out_o, lse_o, _ = oracle.attn_r2(d["q"], d["k"], d["v"], d["q4"], d["k4"], d["v4"], sel_o, w, units=units)
    compare_attention(out_g, lse_g, out_o, lse_o, w, units)
    return out_g, out_r1


@pytest.mark.parametrize("bp", [None, 0, 10000])
def test_running_max_tiny(pab, bp):
    run_r2(pab, "tiny", bp)


@pytest.mark.parametrize("bp", [None, 0])
def test_running_max_n4k(pab, bp):
    out_g, out_r1 = run_r2(pab, "n4k", bp)
    # the reading changes the result: NVFP4 blocks below the running maximum requantise differently
    assert not torch.equal(out_g, out_r1)


def test_running_max_all_fp16_equals_r1(pab):
    """With every pair in FP16 the first level only shifts exp(S - m) before its FP16 rounding:
    both readings stay within the output bar of each other (and of the same SDPA)."""
    out_g, out_r1 = run_r2(pab, "n4k", 10000)
    a, b = out_g.float().cpu().numpy(), out_r1.float().cpu().numpy()
    assert np.linalg.norm(a - b) / np.linalg.norm(b) <= 1e-3


SHAPES = {
    # 128-key blocks, causal, GQA 4:1
    "bk128": workloads.Workload("r2_bk128", 97, 1, 8, 2, 1024, 128, True, 128, 128, -1, 1500, "heavy_bias"),
    # 64-row query blocks (two per tile, each with its own entry order), causal, d = 64
    "bq64": workloads.Workload("r2_bq64", 98, 2, 4, 4, 1024, 64, True, 64, 64, -1, 2500, "normal"),
    # 128-key blocks with d = 64 (the shortest entry lists)
    "d64_bk128": workloads.Workload("r2_d64", 99, 1, 4, 1, 512, 64, True, 128, 128, -1, 3000, "student_t"),
}


@pytest.mark.parametrize("shape", list(SHAPES))
def test_running_max_shapes(pab, shape):
    w = SHAPES[shape]
    q, k, v = workloads.make_qkv(w)
    gq, gk, gv = (torch.from_numpy(x).cuda() for x in (q, k, v))
    cfg = pab.Config.from_workload(w)
    q4, k4, v4 = pab.quantize_qkv(gq, gk, gv)
    sel = pab.block_select(gq, gk, cfg)
    out_g, lse_g = pab.attn_fwd(gq, gk, gv, q4, k4, v4, sel, cfg, running_max=True)
    torch.cuda.synchronize()
    q4o, k4o, v4o = oracle.quantize_nvfp4(q, 0), oracle.quantize_nvfp4(k, 0), oracle.quantize_nvfp4(v, 1)
    sel_o, _, _ = oracle.select(oracle.block_scores(q, k, w), w)
    units = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.n_qb)]
    out_o, lse_o, _ = oracle.attn_r2(q, k, v, q4o, k4o, v4o, sel_o, w, units=units)
    compare_attention(out_g, lse_g, out_o, lse_o, w, units)


@pytest.mark.parametrize("bp", [500, 2000])
def test_running_max_diffusion_sampled(pab, bp):
    run_r2(pab, "diffusion", bp, n_units=8)


def test_running_max_prefill32k_sampled(pab):
    run_r2(pab, "prefill32k", None, n_units=24)
