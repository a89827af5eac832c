"""Parity of the decode path (thrift_decode_select / thrift_decode_attn / thrift_decode_fwd through
the C ABI) with the CPU oracle's decode form on the same seeded inputs.

Bar, as for prefill: block scores and selected key blocks exact (pairs tied with the k-th score
within 1e-6 relative may differ); output within rel-L2 <= 1e-3 and max-abs <= 1e-2 of the
oracle (one FP16 step where that step is larger); lse within 1e-3.  Every output row is
compared: a decode step has few rows.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

REL_L2 = 1e-3
MAX_ABS = 1e-2
LSE_ABS = 1e-3
TIE_REL = 1e-6

_cache = {}


@pytest.fixture(scope="module")
def pab(cuda_device):
    from precision_attention_block_b200 import build
    build.build()
    import precision_attention_block_b200 as pab
    pab.load()
    return pab


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def problem(w):
    key = (w.name, w.B, w.Hq, w.Hkv, w.N, w.d, w.block_k, w.n_query, w.dist, w.index)
    if key not in _cache:
        q, k, v = workloads.make_qkv(w)
        k4, v4 = oracle.quantize_nvfp4(k, 0), oracle.quantize_nvfp4(v, 1)
        _cache[key] = dict(q=q, k=k, v=v, k4=k4, v4=v4, gq=dev(q), gk=dev(k), gv=dev(v))
    return _cache[key]


def fp16_ulp(x):
    a = np.maximum(np.abs(x), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(a)) - 10)


def run(pab, w, check_select=True, entry="fwd"):
    d = problem(w)
    cfg = pab.DecodeConfig.from_workload(w)
    cache = pab.KVCache.build(d["gk"], d["gv"], w.block_k)
    ws = cfg.workspace(d["gq"].device)
    ref = oracle.decode_forward(w, d["q"], d["k"], d["v"], k4=d["k4"], v4=d["v4"])
    if check_select:
        sel = pab.decode_select(d["gq"], cache, cfg, ws=ws, want_scores=True)
        torch.cuda.synchronize()
        s_g = sel.scores.cpu().numpy()
        assert np.array_equal(s_g, ref["scores"]), "decode block scores differ"
        mask = sel.mask.cpu().numpy().view(np.uint32)
        bits = ((mask[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(*mask.shape[:-1], -1)
        bits = bits[..., :cfg.n_kb].astype(bool)
        diff = bits != ref["sel"].astype(bool)
        if diff.any():
            kth = ref["kth"][..., None, None]
            band = np.abs(ref["scores"] - kth) <= TIE_REL * np.abs(kth)
            assert not (diff & ~band).any(), "selected key blocks differ outside the tie band"
        assert np.array_equal(sel.counts.cpu().numpy(), bits.sum(-1))
    if entry == "fwd":
        out, lse = pab.decode_fwd(d["gq"], cache, cfg, ws=ws)
    else:
        sel = pab.decode_select(d["gq"], cache, cfg, ws=ws)
        out, lse = pab.decode_attn(d["gq"], cache, sel, cfg, ws=ws)
    torch.cuda.synchronize()
    assert pab.device_status(ws) == 0
    og = out.cpu().numpy().astype(np.float64)
    lg = lse.cpu().numpy().astype(np.float64)
    oo = ref["out"].astype(np.float64)
    lo = ref["lse"].astype(np.float64)
    assert np.isfinite(og).all()
    rel = np.linalg.norm(og - oo) / np.linalg.norm(oo)
    err = np.abs(og - oo)
    bound = np.maximum(MAX_ABS, fp16_ulp(oo))
    lmx = np.abs(lg - lo).max()
    print(f"decode parity {w.name}: rel-L2 {rel:.3e} max-abs {err.max():.3e} lse {lmx:.3e}")
    assert rel <= REL_L2 and lmx <= LSE_ABS and np.all(err <= bound), (rel, err.max(), lmx)


@pytest.mark.parametrize("bp", [None, 0, 10000, 3000])
def test_decode_tiny(pab, bp):
    w = workloads.WORKLOADS["decode_tiny"]
    run(pab, w if bp is None else w.with_budget(bp))


def test_decode_tiny_select_then_attn(pab):
    run(pab, workloads.WORKLOADS["decode_tiny"], check_select=False, entry="attn")


# (Hq, Hkv, Nq, d, block_k, causal, N): group sizes 1..16 rows, both head dims and key blocks,
# non-causal, several key blocks per split and a ragged last split
SHAPES = [
    (8, 2, 4, 128, 64, True, 2048),
    (4, 4, 3, 64, 128, True, 1536),
    (16, 1, 1, 128, 128, False, 1024),
    (6, 3, 5, 64, 64, True, 2176),
    (2, 1, 8, 128, 64, True, 640),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("bp", [0, 1500, 10000])
def test_decode_shapes(pab, shape, bp):
    Hq, Hkv, Nq, d, bk, causal, N = shape
    w = workloads.WORKLOADS["decode_tiny"].with_shape(Hq=Hq, Hkv=Hkv, n_query=Nq, d=d, block_k=bk,
                                                      causal=causal, N=N, topk_bp=bp)
    run(pab, w)


def test_decode_batch2_heavy_bias(pab):
    w = workloads.WORKLOADS["decode_tiny"].with_shape(B=2, Hq=8, Hkv=2, N=4096, d=128, n_query=2,
                                                      dist="heavy_bias", topk_bp=500)
    run(pab, w)


def test_decode32k(pab):
    run(pab, workloads.WORKLOADS["decode32k"])


def test_decode131k(pab):
    run(pab, workloads.WORKLOADS["decode131k"])
