"""Attn-QAT forward variant (Attn-QAT technical summary, "2. Methodik", second principle): the
kernel also writes O', the FP32 O / l of the same mixed-precision computation before the FP16
rounding.  Checked against the oracle's float64 output (rel-L2 <= 1e-3 and element-wise within
1e-2, the output bar without its FP16 step), and for consistency: the FP16 output is the round to
nearest even of O' element by element and equals thrift_attn_fwd's output bit for bit."""

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pab(cuda_device):
    from precision_attention_block_b200 import build
    build.build()
    import precision_attention_block_b200 as pab
    pab.load()
    return pab


@pytest.mark.parametrize("name,bp", [("tiny", None), ("tiny", 0), ("n4k", 500), ("n4k", 0), ("n4k", 10000)])
def test_qat_output_matches_oracle(pab, name, bp):
    w = workloads.WORKLOADS[name]
    if bp is not None:
        w = w.with_budget(bp)
    q, k, v = workloads.make_qkv(w)
    ref = oracle.forward(w, q, k, v, want_f64=True)
    gq, gk, gv = (torch.from_numpy(x).cuda() for x in (q, k, v))
    cfg = pab.Config.from_workload(w)
    q4, k4, v4 = pab.quantize_qkv(gq, gk, gv)
    sel = pab.block_select(gq, gk, cfg)
    out, out_hp, lse = pab.attn_fwd_qat(gq, gk, gv, q4, k4, v4, sel, cfg)
    out2, _ = pab.attn_fwd(gq, gk, gv, q4, k4, v4, sel, cfg)
    torch.cuda.synchronize()
    hp = out_hp.cpu().numpy().astype(np.float64)
    e = ref["out64"]
    rel = np.linalg.norm(hp - e) / np.linalg.norm(e)
    assert rel <= 1e-3, rel
    assert np.abs(hp - e).max() <= 1e-2
    assert np.array_equal(out.cpu().numpy(), out_hp.cpu().numpy().astype(np.float16))
    assert torch.equal(out, out2)
    lo = ref["lse"].astype(np.float64)
    assert np.abs(lse.cpu().numpy().astype(np.float64) - lo).max() <= 1e-3
