"""thrift_block_select_noalloc, the block-selection entry point for callers that cannot allocate
device memory (a host whose own allocator owns all device memory and only lends the library
input and output buffers, or a latency-bound caller that must not allocate while serving).

Called through the C ABI, it must give exactly what thrift_block_select gives with a caller
workspace -- the same masks, counts, lists and scores -- on two calls in a row, since every call
reuses the library's fixed device scratch array.  It must also refuse, before launching
anything, a configuration whose scratch does not fit in that array.  This file sorts last so that
a run stopping at the first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pab(cuda_device):
    from precision_attention_block_b200 import build
    build.build()
    import precision_attention_block_b200 as pab
    pab.load()
    return pab


def _outputs(pab, cfg, device):
    return pab.Selection(
        torch.full((cfg.B, cfg.Hq, cfg.n_qb, cfg.mask_words), -1, dtype=torch.int32, device=device),
        torch.full((cfg.B, cfg.Hq, cfg.n_qb), -7, dtype=torch.int32, device=device),
        torch.full((cfg.B, cfg.Hq, cfg.n_qb, cfg.n_kb), -7, dtype=torch.int16, device=device),
        torch.full((cfg.B, cfg.Hq, cfg.n_qb, cfg.n_kb), np.nan, dtype=torch.float64, device=device))


def _noalloc(pab, q, k, cfg, sel, want_scores=True):
    c = cfg.c()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return pab.load().thrift_block_select_noalloc(p(q), p(k), ctypes.byref(c), p(sel.mask), p(sel.counts),
                                                  p(sel.lists), p(sel.scores) if want_scores else None,
                                                  pab._stream())


@pytest.mark.parametrize("want_scores", [True, False])
@pytest.mark.parametrize("name", ["n4k", "tiny"])
def test_noalloc_select_matches_workspace_select(pab, name, want_scores):
    """With want_scores False the score matrix goes to the library's own array (the usual use)."""
    w = workloads.WORKLOADS[name]
    q, k, _ = workloads.make_qkv(w)
    dev = torch.device("cuda")
    gq, gk = torch.from_numpy(q).to(dev), torch.from_numpy(k).to(dev)
    cfg = pab.Config.from_workload(w)
    ref = pab.block_select(gq, gk, cfg, want_scores=True)
    torch.cuda.synchronize()
    for call in range(2):
        got = _outputs(pab, cfg, dev)
        assert _noalloc(pab, gq, gk, cfg, got, want_scores) == 0
        torch.cuda.synchronize()
        assert torch.equal(got.mask, ref.mask), f"call {call}: mask"
        assert torch.equal(got.counts, ref.counts), f"call {call}: counts"
        assert torch.equal(got.lists, ref.lists), f"call {call}: lists"
        if not want_scores:
            assert torch.isnan(got.scores).all()  # untouched
            continue
        assert torch.equal(torch.isfinite(got.scores), torch.isfinite(ref.scores))
        fin = torch.isfinite(ref.scores)
        assert torch.equal(got.scores[fin], ref.scores[fin]), f"call {call}: scores"


def test_noalloc_select_rejects_oversized_config(pab):
    w = workloads.WORKLOADS["prefill32k"]  # block means + score matrix need about 46 MB
    cfg = pab.Config.from_workload(w)
    dev = torch.device("cuda")
    tiny = torch.zeros(8, dtype=torch.float16, device=dev)
    sel = pab.Selection(*(torch.zeros(1, dtype=torch.int32, device=dev) for _ in range(3)), None)
    c = cfg.c()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = pab.load().thrift_block_select_noalloc(p(tiny), p(tiny), ctypes.byref(c), p(sel.mask), p(sel.counts),
                                                p(sel.lists), None, pab._stream())
    assert rc == 5  # THRIFT_ERR_WORKSPACE, nothing launched
