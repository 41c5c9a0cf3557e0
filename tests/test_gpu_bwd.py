"""Backward pass of the routed attention on the GPU (moba_attn_bwd through the C ABI) against
the fp64 oracle's attention_backward, with the routing the GPU forward pass chose held fixed.

Tolerance (derived from the arithmetic): P and dS enter the tensor cores rounded to bf16 (2^-9
relative each), products accumulate in fp32, and the gradients are returned in bf16 (2^-9). A
gradient element sums many such terms whose signs cancel (the dS of a row sum to zero), so the
error is bounded against the size of the gradient tensor, not the element:
  |g - g_ref| <= G_ATOL * max|g_ref| + G_RTOL * |g_ref|,  G_ATOL = G_RTOL = 2e-2,
about ten times the two bf16 roundings. Cases: every row of small varlen / GQA / ragged / causal
cases, both head dims, block sizes below, at and above the 128-key tile, topk above the block
count (full causal attention), and a 32K-token small-block shape.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_moba_b200 import workloads as wl
from oracle import moba_ref as ref

pytestmark = pytest.mark.gpu

G_ATOL = 2e-2
G_RTOL = 2e-2


@pytest.fixture(scope="module")
def moba():
    from block_sparse_long_moba_b200 import build, moba as m
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.load_library()
    return m


def _check(name, got, ref_, stats):
    g = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref_)
    scale = np.abs(ref_).max()
    bound = G_ATOL * scale + G_RTOL * np.abs(ref_)
    stats[name] = (float(err.max() / max(scale, 1e-30)), float(scale))
    bad = err > bound
    if bad.any():
        w = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{name} mismatch at {w}: gpu {g[w]} ref {ref_[w]} max|ref| {scale} "
                             f"({int(bad.sum())} of {bad.size} out of tolerance)")


CASES = [
    # cu, hq, hkv, d, B, topk, keys
    ([0, 1024], 2, 2, 64, 128, 3, "offset"),
    ([0, 700, 700, 2000], 4, 2, 128, 128, 4, "clusters"),    # varlen, empty sequence, ragged
    ([0, 1536], 2, 1, 128, 256, 2, "offset"),                # two key sub-tiles per block
    ([0, 2000], 2, 2, 64, 192, 3, "clusters"),               # block not a multiple of 128
    ([0, 640], 2, 1, 64, 128, 8, "offset"),                  # topk >= blocks: full causal
    ([0, 50, 1000], 2, 2, 128, 64, 5, "offset"),             # 64-key blocks, short sequence
    ([0, 8192], 4, 1, 128, 4096, 2, "offset"),               # 4096-key blocks, GQA 4:1
    ([0, 32768], 16, 16, 64, 128, 16, "clusters"),           # the small-block shape at 32K
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"T{c[0][-1]}_h{c[1]}x{c[2]}_d{c[3]}_B{c[4]}_k{c[5]}")
def test_backward_matches_oracle(moba, case):
    cu, hq, hkv, d, B, topk, keys = case
    w = wl.custom(cu, hq, hkv, d, B, topk, keys)
    q, k, v, cu_t = wl.make_inputs(w, seed=2, device="cuda")
    scale = 1.0 / math.sqrt(d)
    T = cu[-1]
    idx = torch.empty((hq, T, topk), dtype=torch.int32, device="cuda")
    o, lse = moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, scale, block_idx_out=idx)
    g = torch.Generator(device="cuda").manual_seed(9)
    d_o = torch.randn((T, hq, d), generator=g, device="cuda").to(torch.bfloat16)
    ws = torch.empty(moba.moba_bwd_workspace_bytes(cu, hq, hkv, d, B, topk), dtype=torch.uint8,
                     device="cuda")
    dq, dk, dv = moba.moba_attn_bwd(q, k, v, o, lse, d_o, idx, cu_t, cu, B, topk, scale,
                                    workspace=ws)
    torch.cuda.synchronize()
    assert moba.moba_device_status(ws) == 0
    dq_r, dk_r, dv_r = ref.attention_backward(q.cpu(), k.cpu(), v.cpu(), cu, B,
                                              idx.cpu().numpy(), scale, d_o.cpu())
    stats = {}
    _check("dv", dv, dv_r, stats)
    _check("dk", dk, dk_r, stats)
    _check("dq", dq, dq_r, stats)
    print(f"backward {case}: max|err|/max|ref| {stats}")


def test_backward_repeatable(moba):
    """Two runs agree to within rounding: every gradient row sums the same terms, in an order that
    depends on where the routing inversion placed each routed row inside its list (dK, dV) and on
    the order of the per-item additions (dQ)."""
    cu, hq, hkv, d, B, topk = [0, 3000], 4, 2, 128, 256, 4
    w = wl.custom(cu, hq, hkv, d, B, topk, "clusters")
    q, k, v, cu_t = wl.make_inputs(w, seed=4, device="cuda")
    idx = torch.empty((hq, cu[-1], topk), dtype=torch.int32, device="cuda")
    o, lse = moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_out=idx)
    d_o = torch.randn_like(q)
    r1 = moba.moba_attn_bwd(q, k, v, o, lse, d_o, idx, cu_t, cu, B, topk)
    r2 = moba.moba_attn_bwd(q, k, v, o, lse, d_o, idx, cu_t, cu, B, topk)
    torch.cuda.synchronize()
    for a, b in zip(r1, r2):
        a, b = a.float(), b.float()
        assert ((a - b).abs() <= 1e-2 * a.abs() + 1e-3 * a.abs().max()).all()
