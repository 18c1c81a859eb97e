"""The one-block kernel's launch modes: programmatic dependent launch (default) and cooperative
(SV_FUSED_COOPERATIVE=1, read once per process, so it runs in a child process). Both must give the
oracle's result; several calls back to back on one workspace exercise the launch sequence tags."""

import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import numpy as np, torch
import block_causal_linear_relu_b200 as sv
import oracle
from block_causal_linear_relu_b200.inputs import draw_qkv, to_f64
errs = []
# the flag-synchronised one-block kernel: 2 heads (static output ranges only), then 40 heads of 35
# tiles (1400 tiles: the last 172 go out in chunks through the per-launch counters, whose parity
# alternates from one call to the next on the same workspace)
for shape, seeds in (((1, 2, 700, 128), 3), ((1, 40, 4400, 96), 3)):
    ws = None
    for seed in range(seeds):
        st = draw_qkv(shape, seed, "bf16")
        q, k, v = (torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda() for x in st)
        if ws is None:
            ws = sv.make_workspace(sv.SV_OP_LINATTN_FWD, q)
        o = sv.sv_linattn_fwd(q, k, v, eps=1e-6, ws=ws)
        torch.cuda.synchronize()
        ref = oracle.linattn_fwd(*(to_f64(x, "bf16") for x in st), 1e-6)
        errs.append(oracle.max_rel_err(o.float().cpu().numpy().astype(np.float64), ref))
    assert ws.status() == 0
print("max err", max(errs))
assert max(errs) < 2e-2, errs
"""


@pytest.mark.parametrize("cooperative", ["0", "1"])
def test_one_block_kernel_launch_modes(cooperative):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    env = dict(os.environ, SV_FUSED_COOPERATIVE=cooperative, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
