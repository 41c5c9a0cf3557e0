"""The MOBA_CHECKS build (libmoba_checks.so: every index the kernels derive from data on the
device is checked against its buffer before use, a failing check reports MOBA_ERR_DEVICE_CHECK)
gives the same results as the normal build and raises no false alarm: a child process with
MOBA_CHECKS=1 loads it and runs small forward (both head dims, varlen, the long-sequence gate),
backward and decode cases against the fp64 oracle, checking the device status after each."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import math, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
from block_sparse_long_moba_b200 import moba, workloads as wl
from oracle import moba_ref as ref
from tests import parity_util as pu
lib = moba.load_library()
assert moba.LIB_PATH.endswith("libmoba_checks.so"), moba.LIB_PATH
for cu, hq, hkv, d, B, topk, keys in [
        ([0, 700, 700, 2000], 4, 2, 128, 128, 4, "clusters"),
        ([0, 1000], 2, 1, 64, 128, 3, "offset"),
        ([0, 40000], 2, 2, 64, 128, 8, "clusters")]:
    w = wl.custom(cu, hq, hkv, d, B, topk, keys)
    q, k, v, cu_t = wl.make_inputs(w, seed=1, device="cuda")
    ws = torch.empty(moba.moba_workspace_bytes(cu, hq, hkv, d, B, topk), dtype=torch.uint8,
                     device="cuda")
    idx = torch.empty((hq, cu[-1], topk), dtype=torch.int32, device="cuda")
    o, lse = moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_out=idx, workspace=ws)
    assert moba.moba_device_status(ws) == 0
    toks = wl.sample_tokens(w, 512, seed=2)
    pu.run_and_check(moba, q, k, v, cu_t, cu, B, topk, 1 / math.sqrt(d), tokens=toks)
    if cu[-1] <= 2000:
        d_o = torch.randn_like(q)
        bws = torch.empty(moba.moba_bwd_workspace_bytes(cu, hq, hkv, d, B, topk),
                          dtype=torch.uint8, device="cuda")
        dq, dk, dv = moba.moba_attn_bwd(q, k, v, o, lse, d_o, idx, cu_t, cu, B, topk,
                                        workspace=bws)
        assert moba.moba_device_status(bws) == 0
        ref_g = ref.attention_backward(q.cpu(), k.cpu(), v.cpu(), cu, B, idx.cpu().numpy(),
                                       1 / math.sqrt(d), d_o.cpu())
        for got, want in zip((dq, dk, dv), ref_g):
            err = np.abs(got.float().cpu().numpy() - want)
            assert (err <= 2e-2 * np.abs(want).max() + 2e-2 * np.abs(want)).all()
# decode
cu, cuq = [0, 5000, 9000], [0, 1, 2]
w = wl.custom(cu, 4, 2, 64, 128, 6, "clusters")
q_all, k, v, cu_t = wl.make_inputs(w, seed=3, device="cuda")
pos = ref.cache_row_positions(cu, cuq)
q = q_all[torch.as_tensor(pos, device="cuda")].contiguous()
cents = moba.moba_centroids(k, cu_t, cu, 128)
idx = torch.empty((4, 2, 6), dtype=torch.int32, device="cuda")
o, lse = moba.moba_decode_fwd(q, k, v, cents, cu_t, cu,
                              torch.tensor(cuq, dtype=torch.int32, device="cuda"), cuq, 128, 6,
                              block_idx_out=idx)
torch.cuda.synchronize()
idx_c = idx.cpu().numpy()
pu.check_routing(q_all.cpu(), ref.centroids(k.cpu(), cu, 128), cu, 128, 6, pos, idx_c)
o_ref, lse_ref = ref.attention(q_all.cpu(), k.cpu(), v.cpu(), cu, 128, idx_c, 0.125, pos)
pu.check_outputs(o.cpu().float().numpy(), lse.cpu().numpy(), o_ref, lse_ref)
print("CHECKS-BUILD-OK")
"""


def test_checks_build_matches_oracle_without_false_alarms():
    from block_sparse_long_moba_b200 import build
    build.build(checks=True)
    env = dict(os.environ, MOBA_CHECKS="1")
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], capture_output=True,
                       text=True, env=env, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "CHECKS-BUILD-OK" in r.stdout
