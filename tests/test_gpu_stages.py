"""Stage-by-stage checks of one key-block visit inside the attention kernel (thrift_debug_attn_dump):
the raw Q K^T the tensor cores leave in TMEM, the re-quantised probability operand written to shared
memory, and the raw P V product -- each against numpy on the same (GPU-produced, already
oracle-verified) NVFP4 / FP16 inputs.  These localise a layout or descriptor error to one MMA."""

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

E2M1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6], np.float64)


@pytest.fixture(scope="module")
def pab(cuda_device):
    from precision_attention_block_b200 import build
    build.build()
    import precision_attention_block_b200 as pab
    pab.load()
    return pab


def unpack_codes(c):
    c = np.asarray(c, np.uint8)
    return np.stack([c & 15, c >> 4], -1).reshape(*c.shape[:-1], c.shape[-1] * 2)


def deq_rows(codes, scales):
    """Element values code * s_b (no tensor scale) of rows of an NVFP4 tensor."""
    sb = oracle.e4m3_decode(scales)
    return E2M1[unpack_codes(codes)] * np.repeat(sb, 16, axis=-1)


def setup(pab, name, bp):
    w = workloads.WORKLOADS[name].with_budget(bp)
    q, k, v = workloads.make_qkv(w)
    gq, gk, gv = (torch.from_numpy(x).cuda() for x in (q, k, v))
    cfg = pab.Config.from_workload(w)
    q4, k4, v4 = pab.quantize_qkv(gq, gk, gv)
    sel = pab.block_select(gq, gk, cfg)
    return w, cfg, (q, k, v), (gq, gk, gv), (q4, k4, v4), sel


def first_unit(w):
    return 0, 0, w.N // 128 - 1  # b, h, query tile of CTA 0's first unit


@pytest.mark.parametrize("name", ["n4k", "tiny"])
def test_fp4_entry_stages(pab, name):
    w, cfg, (q, k, v), g, (q4, k4, v4), sel = setup(pab, name, 0)  # uniform NVFP4: entry e = key block e
    e = 1
    out, lse, dbg = pab.attn_debug_dump(*g, q4, k4, v4, sel, cfg, e)
    torch.cuda.synchronize()
    dbg = dbg.cpu().numpy()
    BK, D = w.block_k, w.d
    b, h, t = first_unit(w)
    hk = h // (w.Hq // w.Hkv)
    rows = slice(t * 128, (t + 1) * 128)
    keys = slice(e * BK, (e + 1) * BK)
    qd = deq_rows(q4.codes.cpu().numpy()[b * w.Hq + h][rows], q4.scales.cpu().numpy()[b * w.Hq + h][rows])
    kd = deq_rows(k4.codes.cpu().numpy()[b * w.Hkv + hk][keys], k4.scales.cpu().numpy()[b * w.Hkv + hk][keys])
    S_ref = qd @ kd.T
    S = dbg[:128 * BK].reshape(128, BK)
    assert np.abs(S - S_ref).max() <= 1e-5 * np.abs(S_ref).max(), "FP4 QK^T mismatch"

    # probability operand: NVFP4 codes then one E4M3 byte per 16 keys
    raw = dbg[128 * BK:128 * BK + 64 * BK].view(np.uint8).reshape(128, BK * 2)
    codes = raw[:, :BK // 2]
    sfb = raw[:, BK // 2:BK // 2 + BK // 16]
    Pdec = E2M1[unpack_codes(codes)] * np.repeat(oracle.e4m3_decode(sfb), 16, axis=-1)
    tau = float(oracle.softmax_scale(D))
    scale = float(q4.tensor_scale.item()) * float(k4.tensor_scale.item()) * tau
    flips = 0
    for r in range(128):
        res = oracle.tile_pq(S[r].astype(np.float64) * scale, False)
        Pq = res[2] * 2688.0
        flips += int((np.abs(Pdec[r] - Pq) > 1e-9 * 2688).sum())
    assert flips <= 0.01 * 128 * BK, f"{flips} probability codes differ"

    vd_all = deq_rows(v4.codes.cpu().numpy()[b * w.Hkv + hk], v4.scales.cpu().numpy()[b * w.Hkv + hk])
    vd = vd_all[:, keys].T  # [BK keys, D]
    PV_ref = Pdec @ vd
    PV = dbg[128 * BK + 64 * BK:].reshape(128, D)
    assert np.abs(PV - PV_ref).max() <= 1e-5 * np.abs(PV_ref).max(), "FP4 PV mismatch"


@pytest.mark.parametrize("name", ["n4k", "tiny"])
def test_fp16_entry_stages(pab, name):
    w, cfg, (q, k, v), g, (q4, k4, v4), sel = setup(pab, name, 10000)  # all FP16: entry e = key block e
    e = 1
    out, lse, dbg = pab.attn_debug_dump(*g, q4, k4, v4, sel, cfg, e)
    torch.cuda.synchronize()
    dbg = dbg.cpu().numpy()
    BK, D = w.block_k, w.d
    b, h, t = first_unit(w)
    hk = h // (w.Hq // w.Hkv)
    rows = slice(t * 128, (t + 1) * 128)
    keys = slice(e * BK, (e + 1) * BK)
    S_ref = q[b, h, rows].astype(np.float64) @ k[b, hk, keys].astype(np.float64).T
    S = dbg[:128 * BK].reshape(128, BK)
    assert np.abs(S - S_ref).max() <= 1e-5 * np.abs(S_ref).max(), "FP16 QK^T mismatch"
    raw = dbg[128 * BK:128 * BK + 64 * BK].view(np.uint8).reshape(128, BK * 2)
    P16 = raw.view(np.float16).astype(np.float64)
    tau = float(oracle.softmax_scale(D))
    Ms = S.max(1, keepdims=True)
    P_ref = np.exp((S - Ms) * tau)
    assert np.abs(P16 - P_ref).max() <= 2e-3
    PV_ref = P16 @ v[b, hk, keys].astype(np.float64)
    PV = dbg[128 * BK + 64 * BK:].reshape(128, D)
    assert np.abs(PV - PV_ref).max() <= 1e-5 * np.abs(PV_ref).max(), "FP16 PV mismatch"
