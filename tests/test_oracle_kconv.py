"""Pins of the oracle's short key convolution before pooling (CPU only).

key_conv is a depthwise causal convolution of width W inside each block (it never reaches into
another block) and centroids_kconv pools the convolved keys [FlashMoBA story: short convolutions
within blocks]. Pinned by: the identity kernel (plain centroids), a per-channel scale, a pure
delay with a closed-form centroid, a block-boundary case, a second (banded-matrix) formulation on
random inputs, linearity in the weights, and the routing it feeds (full forward with W = 1).
"""
import numpy as np
import pytest

from block_sparse_long_moba_b200 import workloads as wl
from oracle import moba_ref as ref


def _keys(T, G=2, d=8, seed=0):
    return np.random.default_rng(seed).standard_normal((T, G, d))


def test_identity_kernel_gives_plain_centroids():
    cu, B = [0, 37, 37, 90], 16
    k = _keys(90)
    w = np.ones((1, 2, 8))
    np.testing.assert_array_equal(ref.centroids_kconv(k, w, cu, B), ref.centroids(k, cu, B))


def test_per_channel_scale():
    cu, B = [0, 50], 16
    k = _keys(50)
    alpha = np.random.default_rng(1).standard_normal((1, 2, 8))
    np.testing.assert_allclose(ref.centroids_kconv(k, alpha, cu, B),
                               alpha[0] * ref.centroids(k, cu, B), rtol=1e-14, atol=1e-15)


def test_pure_delay_closed_form():
    """w = delta at m = 2: kconv[t] = k[t - 2] inside the block, 0 for the first two keys. With
    k[t] = (position in block) + 1 the block sum is 1 + 2 + ... + (n - 2) = (n - 2)(n - 1) / 2."""
    B = 8
    cu = [0, 8, 8, 19]  # blocks of 8, then 8 and 3 keys
    bt = ref.block_table(cu, B)
    k = np.zeros((19, 1, 2))
    for b in range(bt.num_blocks):
        for t in range(bt.start[b], bt.end[b]):
            k[t, 0, :] = t - bt.start[b] + 1
    w = np.zeros((3, 1, 2))
    w[2] = 1.0
    c = ref.centroids_kconv(k, w, cu, B)
    for b in range(bt.num_blocks):
        n = int(bt.end[b] - bt.start[b])
        want = max(n - 2, 0) * max(n - 1, 0) / 2 / n
        np.testing.assert_allclose(c[b, 0], [want, want], rtol=0, atol=1e-15)


def test_convolution_stops_at_the_block_start():
    """The previous block's keys are huge; a key at a block start only sees itself."""
    B = 4
    k = np.zeros((8, 1, 1))
    k[:4] = 1e6
    k[4:] = 1.0
    w = np.full((4, 1, 1), 0.5)
    kc = ref.key_conv(k, w, [0, 8], B)
    assert kc[4, 0, 0] == 0.5                 # first key of block 1: only m = 0
    assert kc[7, 0, 0] == 2.0                 # four keys of its own block
    np.testing.assert_allclose(ref.centroids_kconv(k, w, [0, 8], B)[1, 0, 0],
                               (0.5 + 1.0 + 1.5 + 2.0) / 4)


def test_banded_matrix_formulation_random():
    """Second formulation: per block and channel, kconv = M k with M[t, u] = w[t - u] for
    0 <= t - u < W (a banded lower-triangular Toeplitz matrix), via numpy matmul."""
    rng = np.random.default_rng(3)
    cu, B, W = [0, 45, 45, 100], 16, 5
    G, d = 2, 4
    k = rng.standard_normal((100, G, d))
    w = rng.standard_normal((W, G, d))
    kc = ref.key_conv(k, w, cu, B)
    bt = ref.block_table(cu, B)
    for b in range(bt.num_blocks):
        st, en = int(bt.start[b]), int(bt.end[b])
        n = en - st
        for g in range(G):
            for c in range(d):
                M = np.zeros((n, n))
                for t in range(n):
                    for u in range(max(0, t - W + 1), t + 1):
                        M[t, u] = w[t - u, g, c]
                np.testing.assert_allclose(kc[st:en, g, c], M @ k[st:en, g, c], rtol=1e-12,
                                           atol=1e-12)


def test_linear_in_the_weights():
    rng = np.random.default_rng(4)
    cu, B = [0, 70], 32
    k = rng.standard_normal((70, 1, 4))
    w1, w2 = rng.standard_normal((3, 1, 4)), rng.standard_normal((3, 1, 4))
    lhs = ref.centroids_kconv(k, 2.0 * w1 - w2, cu, B)
    rhs = 2.0 * ref.centroids_kconv(k, w1, cu, B) - ref.centroids_kconv(k, w2, cu, B)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_forward_with_identity_kernel_equals_plain_forward():
    w = wl.custom([0, 300], 4, 2, 16, 32, 3, "clusters")
    q, k, v, _ = wl.make_inputs(w, device="cpu")
    rt0, o0, l0 = ref.forward(q, k, v, w.cu_seqlens, 32, 3, 0.25)
    rt1, o1, l1 = ref.forward(q, k, v, w.cu_seqlens, 32, 3, 0.25, conv_w=np.ones((1, 2, 16)))
    np.testing.assert_array_equal(rt0.idx, rt1.idx)
    np.testing.assert_array_equal(o0, o1)


def test_forward_routes_on_the_convolved_keys():
    """A delay kernel moves every block's pooled signal: the routing follows the convolved
    centroids (checked against a gate run on centroids_kconv directly), while attention still
    reads the keys as given."""
    w = wl.custom([0, 400], 2, 2, 16, 32, 4, "clusters")
    q, k, v, _ = wl.make_inputs(w, device="cpu")
    conv = np.random.default_rng(5).standard_normal((3, 2, 16))
    rt, o, lse = ref.forward(q, k, v, w.cu_seqlens, 32, 4, 0.25, conv_w=conv)
    c = ref.centroids_kconv(k, conv, w.cu_seqlens, 32)
    rt2 = ref.select_blocks(q, c, w.cu_seqlens, 32, 4)
    np.testing.assert_array_equal(rt.idx, rt2.idx)
    o2, l2 = ref.attention(q, k, v, w.cu_seqlens, 32, rt.idx, 0.25, np.arange(400))
    np.testing.assert_array_equal(o, o2)
    assert (rt.idx != ref.forward(q, k, v, w.cu_seqlens, 32, 4, 0.25)[0].idx).any()
