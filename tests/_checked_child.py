"""Child process of tests/test_gpu_checked.py: runs a set of library calls with whichever build
THRIFT_LIB selects and saves their outputs and the device status after each call to an .npz
file (argv[1]).  Not a test module itself (no test_ prefix)."""

import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import precision_attention_block_b200 as pab  # noqa: E402
import workloads  # noqa: E402


def main(out_path):
    L = pab.load()
    dev = torch.device("cuda")
    res = {"checks_enabled": np.array(L.thrift_debug_checks_enabled())}
    ws = pab.Workspace(256, dev)
    # the check probe: a failing check records THRIFT_ERR_CHECK (checked build) or nothing
    pab.check(L.thrift_debug_check(ws.ptr, 1, pab._stream()), "thrift_debug_check")
    res["probe_status"] = np.array(pab.device_status(ws))
    pab.reset_device_status(ws)
    statuses = []
    for name, bp in (("tiny", None), ("tiny", 0), ("n4k", None), ("n4k", 10000)):
        w = workloads.WORKLOADS[name] if bp is None else workloads.WORKLOADS[name].with_budget(bp)
        q, k, v = (torch.from_numpy(x).to(dev) for x in workloads.make_qkv(w))
        cfg = pab.Config.from_workload(w)
        aws = pab.Workspace.for_config(cfg, dev, auto=True)
        out, lse = pab.attn_fwd_auto(q, k, v, cfg, ws=aws)
        q4, k4, v4 = pab.quantize_qkv(q, k, v, ws=aws)
        sel = pab.block_select(q, k, cfg)
        out2, _ = pab.attn_fwd(q, k, v, q4, k4, v4, sel, cfg, ws=aws, running_max=True)
        tm = q.transpose(1, 2).contiguous().transpose(1, 2)
        out3, _ = pab.attn_fwd_auto(tm, k, v, cfg, ws=aws)
        torch.cuda.synchronize()
        tag = f"{name}_{bp}"
        res[f"out_{tag}"] = out.cpu().numpy()
        res[f"lse_{tag}"] = lse.cpu().numpy()
        res[f"r2_{tag}"] = out2.cpu().numpy()
        res[f"strided_{tag}"] = out3.cpu().numpy()
        res[f"mask_{tag}"] = sel.mask.cpu().numpy()
        statuses.append(pab.device_status(aws))
    # a long-row selection (cluster top-k) and a decode step on an appended cache
    w = workloads.WORKLOADS["prefill16k"].with_shape(Hq=4, Hkv=1)
    q, k, _ = (torch.from_numpy(x).to(dev) for x in workloads.make_qkv(w))
    sel = pab.block_select(q, k, pab.Config.from_workload(w))
    res["mask_16k"] = sel.mask.cpu().numpy()
    wd = workloads.WORKLOADS["decode_tiny"]
    qd, kd, vd = (torch.from_numpy(x).to(dev) for x in workloads.make_qkv(wd))
    cache = pab.KVCache.build(kd[:, :, :900], vd[:, :, :900], block_k=wd.block_k, capacity=wd.N)
    cache.append(kd[:, :, 900:1000], vd[:, :, 900:1000])
    dcfg = pab.DecodeConfig.from_workload(wd)
    dws = dcfg.for_cache(cache).workspace(dev)
    od, ld = pab.decode_fwd(qd, cache, dcfg, ws=dws)
    torch.cuda.synchronize()
    res["decode_out"] = od.cpu().numpy()
    statuses.append(pab.device_status(dws))
    res["statuses"] = np.array(statuses)
    np.savez(out_path, **res)


if __name__ == "__main__":
    main(sys.argv[1])
