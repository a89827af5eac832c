"""The checked build (libthrift_checked.so, THRIFT_CHECKS: every tile, list-entry and mask-word
index is checked in the kernels before use) on the GPU: a failing check is reported as
THRIFT_ERR_CHECK through the device status word without touching memory, no check fails on
the prefill (mixed, all-FP16, running-maximum, strided), long-row selection and appended-cache
decode paths, and every output equals the regular build's bit for bit.  Each build runs in its
own child process (tests/_checked_child.py)."""

import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHILD = os.path.join(ROOT, "tests", "_checked_child.py")


def run_child(lib, out, tmp_path):
    env = dict(os.environ, THRIFT_LIB=lib)
    r = subprocess.run([sys.executable, CHILD, str(out)], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    return np.load(out)


def test_checked_build_matches_regular(cuda_device, tmp_path):
    from precision_attention_block_b200 import build
    regular = build.build()
    checked = build.build(checked=True)
    a = run_child(regular, tmp_path / "regular.npz", tmp_path)
    b = run_child(checked, tmp_path / "checked.npz", tmp_path)
    assert int(a["checks_enabled"]) == 0 and int(b["checks_enabled"]) == 1
    assert int(a["probe_status"]) == 0          # checks compiled out
    assert int(b["probe_status"]) == 8          # THRIFT_ERR_CHECK
    assert (a["statuses"] == 0).all() and (b["statuses"] == 0).all()
    for key in a.files:
        if key in ("checks_enabled", "probe_status"):
            continue
        assert np.array_equal(a[key], b[key], equal_nan=True), key
