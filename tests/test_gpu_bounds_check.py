"""The debug library (librtlayer_check.so, built with -DRT_BOUNDS_CHECK): every
index the layer's kernels compute is checked against the ranges their
arguments declare, and a failed check is recorded in the error word instead
of trapping. Runs the layer on small, odd shapes (odd B, N not a power of two,
more than one row block, blocks of every size up to 1024 keys) and the block
fold on its own, each in a fresh process that loads the debug library, and
requires a clean error word and oracle parity."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import sys
sys.path.insert(0, {root!r})
import numpy as np, torch
from blocked_attention_b200 import build as Bld
from blocked_attention_b200 import rtlayer as R
R.LIB_PATH = Bld.build(bounds_check=True)
from oracle import rt_oracle as O
from tests.parity_util import TOL, problem, rel_err, to_device, to_np
for (B, N, d, H, dff) in [(3, 37, 128, 2, 256), (130, 20, 128, 2, 256), (5, 100, 192, 3, 320), (2, 1100, 128, 2, 256)]:
    x, W = problem(B, N, d, H, dff, "bf16")
    ws = R.alloc_workspace(R.workspace_bytes(B, N, d, H, dff))
    z, K, V = R.layer_forward(to_device(x, "bf16"), {{k: to_device(v, "bf16") for k, v in W.items()}}, H, workspace=ws)
    st = R.sync_status(ws)
    assert st == 0, ("error word", B, N, st)
    seqs = [0, B - 1]
    zr, Kr, Vr = O.rt_layer(x[seqs], W, H)
    errs = (rel_err(to_np(z)[seqs], zr), rel_err(to_np(K).transpose(1, 0, 2)[seqs], Kr),
            rel_err(to_np(V).transpose(1, 0, 2)[seqs], Vr))
    assert max(errs) <= TOL["bf16"], (B, N, errs)
print("bounds-checked layer ok")
'''


def test_layer_under_bounds_checks():
    r = subprocess.run([sys.executable, "-c", SCRIPT.format(root=ROOT)], capture_output=True, text=True,
                       timeout=1200, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "bounds-checked layer ok" in r.stdout
