"""Parity of the attention path over the shape combinations the library accepts that the named
workloads do not all reach: 64- and 128-row query blocks, 64- and 128-key blocks, d = 64 and 128,
causal and not, grouped and plain multi-head attention, an odd number of query heads, and the
three precision modes (uniform NVFP4, mixed, all FP16).  Small sizes, full tensors, same bar as
tests/test_gpu_parity.py."""

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

REL_L2 = 1e-3
MAX_ABS = 1e-2
LSE_ABS = 1e-3

# (N, Hq, Hkv, d, causal, block_q, block_k)
SHAPES = [
    (1024, 2, 2, 64, True, 64, 64),
    (1024, 4, 2, 128, True, 64, 64),
    (1024, 3, 3, 64, False, 128, 128),
    (2048, 4, 1, 64, True, 128, 128),
    (1024, 2, 2, 128, False, 64, 128),
    (1536, 6, 2, 128, True, 128, 64),
]


@pytest.fixture(scope="module")
def pab(cuda_device):
    from precision_attention_block_b200 import build
    build.build()
    import precision_attention_block_b200 as pab
    pab.load()
    return pab


def fp16_ulp(x):
    a = np.maximum(np.abs(x), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(a)) - 10)


@pytest.mark.parametrize("bp", [0, 700, 10000])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "N{}-h{}_{}-d{}-{}-q{}k{}".format(
    s[0], s[1], s[2], s[3], "causal" if s[4] else "full", s[5], s[6]))
def test_attn_shape(pab, shape, bp):
    N, Hq, Hkv, d, causal, bq, bk = shape
    w = workloads.WORKLOADS["n4k"].with_shape(N=N, Hq=Hq, Hkv=Hkv, d=d, causal=causal, block_q=bq,
                                               block_k=bk).with_budget(bp)
    q, k, v = workloads.make_qkv(w)
    gq, gk, gv = (torch.from_numpy(x).cuda() for x in (q, k, v))
    cfg = pab.Config.from_workload(w)
    ws = pab.Workspace.for_config(cfg, gq.device)
    q4, k4, v4 = pab.quantize_qkv(gq, gk, gv)
    sel = pab.block_select(gq, gk, cfg, ws=ws)
    out, lse = pab.attn_fwd(gq, gk, gv, q4, k4, v4, sel, cfg, ws=ws)
    torch.cuda.synchronize()
    assert pab.device_status(ws) == 0
    ref = oracle.forward(w, q, k, v)
    a = out.cpu().numpy().astype(np.float64)
    e = ref["out"].astype(np.float64)
    rel = np.linalg.norm(a - e) / np.linalg.norm(e)
    err = np.abs(a - e)
    lmx = np.abs(lse.cpu().numpy() - ref["lse"]).max()
    assert np.isfinite(a).all()
    assert rel <= REL_L2 and lmx <= LSE_ABS and np.all(err <= np.maximum(MAX_ABS, fp16_ulp(e))), (rel, err.max(), lmx)
