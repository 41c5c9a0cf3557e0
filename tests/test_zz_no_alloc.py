"""moba_attn_fwd_noalloc — the entry point for callers that cannot allocate device memory.

Such callers (plug-ins whose host application owns every byte of device memory, latency-critical
paths that cannot afford an allocation) get their scratch memory from one static device array
inside the library. This test calls that entry point through the C ABI twice in a row, on two
different problems, and checks both results against the fp64 oracle on the routing the gate
chooses (itself checked against the oracle's routing), within the tolerances of the parity
tests, and against the workspace-based moba_attn_fwd; after each call the status word in the
array must read MOBA_OK. It also checks that a problem larger than the array is refused. Collected last on purpose: it must pass alone in a
fresh process and after every other test.
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
    ([0, 4096], 8, 2, 128, 256, 6, "offset"),
    ([0, 1000, 1000, 3000], 4, 4, 64, 128, 5, "clusters"),
]


def test_noalloc_matches_the_oracle_twice_in_a_row(moba):
    for n, (cu, hq, hkv, d, B, topk, keys) in enumerate(CASES):
        w = wl.custom(cu, hq, hkv, d, B, topk, keys)
        q, k, v, cu_t = wl.make_inputs(w, seed=10 + n, device="cuda")
        scale = 1.0 / math.sqrt(d)
        o = torch.full_like(q, float("nan"))
        lse = torch.full((hq, cu[-1]), float("nan"), dtype=torch.float32, device="cuda")
        moba.moba_attn_fwd_noalloc(q, k, v, cu_t, cu, B, topk, scale, o=o, lse=lse)
        assert moba.moba_noalloc_status() == 0
        # the routing the call used is the gate's (same kernels, deterministic)
        idx = moba.moba_gate_topk(q, moba.moba_centroids(k, cu_t, cu, B), cu_t, cu, B, topk)
        torch.cuda.synchronize()
        tokens = np.arange(cu[-1])
        idx_c = idx.cpu().numpy()
        pu.check_routing(q.cpu(), ref.centroids(k.cpu(), cu, B), cu, B, topk, tokens, idx_c)
        o_ref, lse_ref = ref.attention(q.cpu(), k.cpu(), v.cpu(), cu, B, idx_c, scale, tokens)
        pu.check_outputs(o.cpu().float().numpy(), lse.cpu().numpy(), o_ref, lse_ref)
        # and it agrees with the workspace-based entry point within the same tolerances
        o_ws, lse_ws = moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, scale)
        torch.cuda.synchronize()
        o_err = (o.float() - o_ws.float()).abs()
        assert (o_err <= pu.O_ATOL + pu.O_RTOL * o_ws.float().abs()).all(), float(o_err.max())
        assert ((lse - lse_ws).abs() <= pu.LSE_ATOL).all()


def test_noalloc_refuses_problems_beyond_its_scratch(moba):
    w = wl.WORKLOADS["llama8b_128k"]
    T, hq, d = w.total_tokens, w.hq, w.d
    q = torch.empty((T, hq, d), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((T, w.hkv, d), dtype=torch.bfloat16, device="cuda")
    cu_t = torch.tensor(w.cu_seqlens, dtype=torch.int32, device="cuda")
    with pytest.raises(moba.MobaError) as ei:
        moba.moba_attn_fwd_noalloc(q, k, k, cu_t, w.cu_seqlens, w.block_size, w.topk)
    assert ei.value.status == -3  # MOBA_ERR_WORKSPACE
