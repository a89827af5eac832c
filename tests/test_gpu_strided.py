"""Strided [B, H, N, d] layouts through the C ABI (thrift_*_strided): token-major tensors
([B, N, H, d], the layout a fused QKV projection produces) and padded rows reach the kernels as
views, without a copy.  The addressing is the only difference from the dense path, so every
result must equal the dense path's bit for bit: NVFP4 codes and scales, the selection, and the
attention output (written into a strided output view); the dense path itself is checked against
the oracle in test_gpu_parity."""

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": workloads.WORKLOADS["tiny"],
    "b2_d128": workloads.Workload("b2_d128", 96, 2, 4, 2, 1024, 128, True, 64, 64, -1, 2000, "heavy_bias"),
}


@pytest.fixture(scope="module")
def pab(cuda_device):
    from precision_attention_block_b200 import build
    build.build()
    import precision_attention_block_b200 as pab
    pab.load()
    return pab


def token_major(x: torch.Tensor) -> torch.Tensor:
    """The same values stored [B, N, H, d], returned as a [B, H, N, d] view."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


def padded_rows(x: torch.Tensor, pad: int = 8) -> torch.Tensor:
    """The same values in rows of d + pad elements, returned as a [B, H, N, d] view."""
    B, H, N, d = x.shape
    buf = torch.full((B, H, N, d + pad), float("nan"), dtype=x.dtype, device=x.device)
    buf[..., :d] = x
    return buf[..., :d]


LAYOUTS = {"token_major": token_major, "padded": padded_rows}


def inputs(name):
    w = CASES[name]
    q, k, v = workloads.make_qkv(w)
    return w, *(torch.from_numpy(x).cuda() for x in (q, k, v))


@pytest.mark.parametrize("layout", list(LAYOUTS))
@pytest.mark.parametrize("name", list(CASES))
def test_strided_quantize_equals_dense(pab, name, layout):
    w, q, k, v = inputs(name)
    for x, axis in ((q, 0), (k, 0), (v, 1)):
        xs = LAYOUTS[layout](x)
        assert not xs.is_contiguous()
        a, b = pab.quantize_nvfp4(x, axis), pab.quantize_nvfp4(xs, axis)
        torch.cuda.synchronize()
        for f in ("codes", "scales", "scales_mma", "tensor_scale"):
            assert torch.equal(getattr(a, f), getattr(b, f)), f


@pytest.mark.parametrize("layout", list(LAYOUTS))
@pytest.mark.parametrize("name", list(CASES))
def test_strided_select_equals_dense(pab, name, layout):
    w, q, k, _ = inputs(name)
    cfg = pab.Config.from_workload(w)
    a = pab.block_select(q, k, cfg, want_scores=True)
    b = pab.block_select(LAYOUTS[layout](q), LAYOUTS[layout](k), cfg, want_scores=True)
    torch.cuda.synchronize()
    for f in ("mask", "counts", "lists"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    assert torch.equal(torch.nan_to_num(a.scores, neginf=-1e300), torch.nan_to_num(b.scores, neginf=-1e300))


@pytest.mark.parametrize("layout", list(LAYOUTS))
@pytest.mark.parametrize("name", list(CASES))
def test_strided_attention_equals_dense(pab, name, layout):
    w, q, k, v = inputs(name)
    cfg = pab.Config.from_workload(w)
    q4, k4, v4 = pab.quantize_qkv(q, k, v)
    sel = pab.block_select(q, k, cfg)
    out_d, lse_d = pab.attn_fwd(q, k, v, q4, k4, v4, sel, cfg)
    f = LAYOUTS[layout]
    out_s = f(torch.zeros_like(q))  # the output in the same strided layout
    out_s.fill_(float("nan"))
    _, lse_s = pab.attn_fwd(f(q), f(k), f(v), q4, k4, v4, sel, cfg, out=out_s)
    torch.cuda.synchronize()
    assert torch.equal(out_s, out_d)
    assert torch.equal(lse_s, lse_d)


@pytest.mark.parametrize("name", list(CASES))
def test_strided_auto_equals_dense(pab, name):
    w, q, k, v = inputs(name)
    cfg = pab.Config.from_workload(w)
    out_d, lse_d = pab.attn_fwd_auto(q, k, v, cfg)
    out_s = token_major(torch.zeros_like(q))
    _, lse_s = pab.attn_fwd_auto(token_major(q), token_major(k), token_major(v), cfg, out=out_s)
    torch.cuda.synchronize()
    assert torch.equal(out_s, out_d)
    assert torch.equal(lse_s, lse_d)
    # the padding of a padded output row is never written
    buf = torch.full((w.B, w.Hq, w.N, w.d + 8), 7.0, dtype=torch.float16, device="cuda")
    pab.attn_fwd_auto(q, k, v, cfg, out=buf[..., :w.d])
    torch.cuda.synchronize()
    assert torch.equal(buf[..., :w.d], out_d)
    assert bool((buf[..., w.d:] == 7.0).all())
