"""moba_attn_fwd_noalloc — the entry point for callers that cannot allocate device memory.

Such callers (plug-ins whose host application owns every byte of device memory, latency-critical
paths that cannot afford an allocation) get their scratch memory from one static device array
inside the library. This test calls that entry point through the C ABI twice in a row, on two
different problems, and checks both results against the workspace-based moba_attn_fwd within the
tolerances of the parity tests; it also checks that a problem larger than the array is refused.
Collected last on purpose: it must pass alone in a fresh process and after every other test.
"""
import math

import pytest
import torch

from block_sparse_long_moba_b200 import workloads as wl
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


def test_noalloc_matches_workspace_path_twice_in_a_row(moba):
    for n, (cu, hq, hkv, d, B, topk, keys) in enumerate(CASES):
        w = wl.custom(cu, hq, hkv, d, B, topk, keys)
        q, k, v, cu_t = wl.make_inputs(w, seed=10 + n, device="cuda")
        scale = 1.0 / math.sqrt(d)
        o_ref, lse_ref = moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, scale)
        o = torch.full_like(q, float("nan"))
        lse = torch.full((hq, cu[-1]), float("nan"), dtype=torch.float32, device="cuda")
        moba.moba_attn_fwd_noalloc(q, k, v, cu_t, cu, B, topk, scale, o=o, lse=lse)
        torch.cuda.synchronize()
        o_err = (o.float() - o_ref.float()).abs()
        assert (o_err <= pu.O_ATOL + pu.O_RTOL * o_ref.float().abs()).all(), float(o_err.max())
        assert ((lse - lse_ref).abs() <= pu.LSE_ATOL).all(), float((lse - lse_ref).abs().max())


def test_noalloc_refuses_problems_beyond_its_scratch(moba):
    w = wl.WORKLOADS["llama8b_128k"]
    T, hq, d = w.total_tokens, w.hq, w.d
    q = torch.empty((T, hq, d), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((T, w.hkv, d), dtype=torch.bfloat16, device="cuda")
    cu_t = torch.tensor(w.cu_seqlens, dtype=torch.int32, device="cuda")
    with pytest.raises(moba.MobaError) as ei:
        moba.moba_attn_fwd_noalloc(q, k, k, cu_t, w.cu_seqlens, w.block_size, w.topk)
    assert ei.value.status == -3  # MOBA_ERR_WORKSPACE
