"""MoBA decode / chunked prefill against a KV cache on the GPU (moba_decode_fwd through the C ABI)
against the fp64 oracle, and against the prefill path at the same positions.

Cases: one row per sequence (decode) over varlen caches with an empty and a one-token sequence,
chunks of several rows, many blocks (a long 128-key-block cache: the radix selection over
thousands of scores), both head dims, GQA, topk = 1, topk above the block count, and a given
routing.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_moba_b200 import workloads as wl
from oracle import moba_ref as ref
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moba():
    from block_sparse_long_moba_b200 import build, moba as m
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.load_library()
    return m


CASES = [
    # cu (cache), cuq (rows), hq, hkv, d, B, topk, keys
    ([0, 5000, 5000, 5001, 17345], [0, 1, 1, 2, 3], 4, 2, 64, 128, 8, "clusters"),
    ([0, 20000, 29000], [0, 1, 2], 8, 2, 128, 4096, 3, "offset"),
    ([0, 3000, 9000], [0, 17, 317], 4, 4, 64, 128, 6, "clusters"),        # chunked prefill
    ([0, 300000], [0, 1], 2, 1, 64, 128, 16, "clusters"),                  # 2344 blocks
    ([0, 4100, 8300], [0, 2, 4], 2, 2, 128, 512, 1, "offset"),             # topk = 1
    ([0, 1500], [0, 3], 2, 1, 128, 256, 64, "offset"),                     # topk > blocks
]


def _run(moba, cu, cuq, hq, hkv, d, B, topk, keys, seed=0, block_idx_in=None):
    w = wl.custom(cu, hq, hkv, d, B, topk, keys)
    q_all, k, v, cu_t = wl.make_inputs(w, seed=seed, device="cuda")
    pos = ref.cache_row_positions(cu, cuq)
    q = q_all[torch.as_tensor(pos, device="cuda")].contiguous()
    cuq_t = torch.tensor(cuq, dtype=torch.int32, device="cuda")
    cents = moba.moba_centroids(k, cu_t, cu, B)
    Tq = cuq[-1]
    idx = torch.empty((hq, Tq, topk), dtype=torch.int32, device="cuda")
    scale = 1.0 / math.sqrt(d)
    o, lse = moba.moba_decode_fwd(q, k, v, cents, cu_t, cu, cuq_t, cuq, B, topk, scale,
                                  block_idx_in=block_idx_in, block_idx_out=idx)
    torch.cuda.synchronize()
    return w, q_all, q, k, v, cu_t, pos, idx, o, lse, scale


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"T{c[0][-1]}_rows{c[1][-1]}_d{c[4]}_B{c[5]}_k{c[6]}")
def test_decode_matches_oracle(moba, case):
    cu, cuq, hq, hkv, d, B, topk, keys = case
    w, q_all, q, k, v, cu_t, pos, idx, o, lse, scale = _run(moba, *case)
    kc, vc = k.cpu(), v.cpu()
    cents = ref.centroids(kc, cu, B)
    idx_c = idx.cpu().numpy()
    ties = pu.check_routing(q_all.cpu(), cents, cu, B, topk, pos, idx_c)
    o_ref, lse_ref = ref.attention(q_all.cpu(), kc, vc, cu, B, idx_c, scale, pos)
    pu.check_outputs(o.cpu().float().numpy(), lse.cpu().numpy(), o_ref, lse_ref)
    print(f"decode {case}: ties={ties}")


def test_decode_equals_prefill_rows(moba):
    """The decode rows and the prefill pass over the whole cache agree at the same positions
    (same routing, O and LSE within the parity tolerances of each other)."""
    case = ([0, 6000, 14000], [0, 1, 5], 4, 2, 128, 1024, 4, "offset")
    cu, cuq, hq, hkv, d, B, topk, keys = case
    w, q_all, q, k, v, cu_t, pos, idx, o, lse, scale = _run(moba, *case)
    idx_f = torch.empty((hq, cu[-1], topk), dtype=torch.int32, device="cuda")
    o_f, lse_f = moba.moba_attn_fwd(q_all, k, v, cu_t, cu, B, topk, scale, block_idx_out=idx_f)
    torch.cuda.synchronize()
    p = torch.as_tensor(pos, device="cuda")
    assert torch.equal(idx, idx_f[:, p])
    err = (o.float() - o_f[p].float()).abs()
    assert (err <= pu.O_ATOL + pu.O_RTOL * o_f[p].float().abs()).all(), float(err.max())
    assert ((lse - lse_f[:, p]).abs() <= pu.LSE_ATOL).all()


def test_decode_with_given_routing(moba):
    cu, cuq = [0, 2000, 5000], [0, 1, 2]
    B, topk, hq = 128, 4, 2
    # a valid routing: current block plus the lowest past blocks
    pos = ref.cache_row_positions(cu, cuq)
    idx_in = torch.full((hq, 2, topk), -1, dtype=torch.int32)
    for r, t in enumerate(pos):
        s = 0 if t < cu[1] else 1
        i = (t - cu[s]) // B
        sel = list(range(min(i, topk - 1))) + [i]
        idx_in[:, r, :len(sel)] = torch.tensor(sel, dtype=torch.int32)
    idx_d = idx_in.cuda()
    w, q_all, q, k, v, cu_t, pos, idx, o, lse, scale = _run(moba, cu, cuq, hq, hq, 64, B, topk,
                                                            "offset", block_idx_in=idx_d)
    assert torch.equal(idx.cpu(), idx_in)
    o_ref, lse_ref = ref.attention(q_all.cpu(), k.cpu(), v.cpu(), cu, B, idx_in.numpy(), scale,
                                   pos)
    pu.check_outputs(o.cpu().float().numpy(), lse.cpu().numpy(), o_ref, lse_ref)
