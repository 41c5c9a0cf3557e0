"""Short key convolution before pooling on the GPU (through the C ABI) against the fp64 oracle.

Centroids of the convolved keys are checked on both forms of the centroid kernel (per kv head and
whole rows), with widths from 1 to the maximum, blocks shorter than the kernel (ragged tails) and
an empty sequence; the whole forward pass with the convolution is checked like the plain one
(routing exact outside the near-tie band, O and LSE within the parity tolerances).
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


def _conv(W, hkv, d, seed=0):
    g = torch.Generator(device="cpu").manual_seed(100 + seed)
    return (torch.randn((W, hkv, d), generator=g) / math.sqrt(W)).to("cuda")


@pytest.mark.parametrize("cu,hkv,d,B,W", [
    ([0, 1024], 1, 64, 128, 1),
    ([0, 1024], 1, 64, 128, 4),
    ([0, 300, 300, 1000, 1003], 4, 128, 64, 3),   # ragged tails, empty sequence, 3-key block
    ([0, 8192], 8, 128, 4096, 16),
    ([0, 10000], 32, 128, 128, 5),                 # whole-row form
    ([0, 65536], 16, 64, 128, 4),                  # the 128-key-block shape
    ([0, 5000, 5000, 12000], 3, 64, 64, 16),       # W > keys of the last block of sequence 2
])
def test_kconv_centroids_match_oracle(moba, cu, hkv, d, B, W):
    w = wl.custom(cu, hkv, hkv, d, B, 2)
    q, k, v, cu_t = wl.make_inputs(w, seed=0, device="cuda")
    cw = _conv(W, hkv, d)
    c = moba.moba_centroids_kconv(k, cw, cu_t, cu, B)
    torch.cuda.synchronize()
    c_ref = ref.centroids_kconv(k.cpu(), cw.cpu().double().numpy(), cu, B)
    np.testing.assert_allclose(c.cpu().numpy(), c_ref, rtol=1e-5, atol=2e-6)


@pytest.mark.parametrize("cu,hq,hkv,d,B,topk,W", [
    ([0, 2048], 2, 2, 64, 128, 4, 4),
    ([0, 700, 700, 2000], 4, 2, 128, 128, 3, 3),
    ([0, 8192], 8, 2, 128, 4096, 2, 8),
])
def test_kconv_forward_matches_oracle(moba, cu, hq, hkv, d, B, topk, W):
    w = wl.custom(cu, hq, hkv, d, B, topk, "clusters")
    q, k, v, cu_t = wl.make_inputs(w, seed=3, device="cuda")
    cw = _conv(W, hkv, d, seed=1)
    scale = 1.0 / math.sqrt(d)
    idx = torch.empty((hq, cu[-1], topk), dtype=torch.int32, device="cuda")
    o, lse = moba.moba_attn_fwd_kconv(q, k, v, cw, cu_t, cu, B, topk, scale, block_idx_out=idx)
    torch.cuda.synchronize()
    tokens = np.arange(cu[-1])
    cents = ref.centroids_kconv(k.cpu(), cw.cpu().double().numpy(), cu, B)
    idx_c = idx.cpu().numpy()
    pu.check_routing(q.cpu(), cents, cu, B, topk, tokens, idx_c)
    o_ref, lse_ref = ref.attention(q.cpu(), k.cpu(), v.cpu(), cu, B, idx_c, scale, tokens)
    pu.check_outputs(o.cpu().float().numpy(), lse.cpu().numpy(), o_ref, lse_ref)
