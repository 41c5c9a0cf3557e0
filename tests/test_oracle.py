"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test ties one part of the oracle to something other than itself:
  * centroid      -> closed form on constructed keys (mean, ragged tail);
  * gate          -> a constructed case with a hand-derived answer, ties, brute-force subset
                     enumeration on random inputs, and hand-derived near-tie fields (margin,
                     boundary) and per-head scores of a GQA layout;
  * full limit    -> with topk >= #blocks MoBA is causal attention: textbook formula and torch SDPA
                     in float64 (MoBA README, "Seamlessly Transition between Full and Sparse");
  * topk = 1      -> block-diagonal causal (local) attention;
  * mask form     -> explicit T x T mask + dense softmax (MoBA repo radar, "How it works");
  * invariants    -> current block kept, no future block, |S| = min(k, i+1), softmax sums to 1,
                     LSE bounds, O inside the convex hull of the attended values;
  * golden        -> a hand-worked example in tests/golden/.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from block_sparse_long_moba_b200 import workloads as wl
from oracle import moba_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _inputs(cu, hq, hkv, d, B, topk, keys="offset", seed=0):
    w = wl.custom(cu, hq, hkv, d, B, topk, keys)
    q, k, v, cu_t = wl.make_inputs(w, seed=seed, device="cpu")
    return w, q, k, v


# ------------------------------------------------------------------------------------ centroid
def test_centroid_closed_form_with_ragged_tail():
    B, d, G = 8, 4, 2
    cu = [0, 19, 19, 30]  # ragged tails (19 = 2*8+3, 11 = 8+3) and an empty sequence
    T = cu[-1]
    bt = ref.block_table(cu, B)
    k = np.zeros((T, G, d), np.float32)
    for b in range(bt.num_blocks):
        for t in range(bt.start[b], bt.end[b]):
            for g in range(G):
                k[t, g, 0] = b + 10 * g          # constant inside the block
                k[t, g, 1] = t - bt.start[b]      # 0..n_b-1
                k[t, g, 2] = 1.0 if (t - bt.start[b]) == 0 else 0.0
    c = ref.centroids(k, cu, B)
    assert c.shape == (bt.num_blocks, G, d)
    for b in range(bt.num_blocks):
        nb = bt.end[b] - bt.start[b]
        for g in range(G):
            assert c[b, g, 0] == b + 10 * g
            assert c[b, g, 1] == pytest.approx((nb - 1) / 2, abs=1e-15)
            assert c[b, g, 2] == pytest.approx(1.0 / nb, abs=1e-15)
            assert c[b, g, 3] == 0.0
    # block counts: 19 -> 3 blocks, 0 -> none, 11 -> 2 blocks
    assert list(bt.blk_off) == [0, 3, 3, 5]


# ---------------------------------------------------------------------------------------- gate
def _const_block_keys(weights, B, d=4):
    T = len(weights) * B
    k = np.zeros((T, 1, d), np.float32)
    for j, w in enumerate(weights):
        k[j * B:(j + 1) * B, 0, 0] = w
    return k


def test_gate_constructed_case():
    B = 4
    w = [3, -1, 5, 0, 2, 7, 1, 4]
    k = _const_block_keys(w, B)
    T = k.shape[0]
    cu = [0, T]
    c = ref.centroids(k, cu, B)
    q = np.zeros((T, 2, 4), np.float32)
    q[:, 0, 0] = 1.0     # head 0 prefers large w
    q[:, 1, 0] = -1.0    # head 1 prefers small w
    rt = ref.select_blocks(q, c, cu, B, 4)  # Hkv = 1, Hq = 2: both heads use kv head 0
    idx = rt.idx
    t7 = 7 * B + 1
    assert list(idx[0, t7]) == [0, 2, 5, 7]     # past scores 3,-1,5,0,2,7,1 -> 7,5,3
    assert list(idx[1, t7]) == [1, 3, 6, 7]     # -w: 1,0,1 ... -> w=-1,0,1
    t4 = 4 * B
    assert list(idx[0, t4]) == [0, 2, 3, 4]     # past 3,-1,5,0 -> 5,3,0
    # -w past: -3, 1, -5, 0 -> top-3 are 1 (j=1), 0 (j=3), -3 (j=0)
    assert list(idx[1, t4]) == [0, 1, 3, 4]
    t3 = 3 * B + 2                              # k-1 = 3 >= i = 3: every block 0..3
    assert list(idx[0, t3]) == [0, 1, 2, 3]
    t1 = B                                      # i = 1: blocks 0,1 then -1 padding
    assert list(idx[0, t1]) == [0, 1, -1, -1]
    assert list(idx[0, 0]) == [0, -1, -1, -1]


def test_gate_ties_go_to_lower_block():
    B = 4
    w = [2, 2, 2, 1, 2, 0]
    k = _const_block_keys(w, B)
    T = k.shape[0]
    c = ref.centroids(k, [0, T], B)
    q = np.zeros((T, 1, 4), np.float32)
    q[:, 0, 0] = 1.0
    rt = ref.select_blocks(q, c, [0, T], B, 3)
    t = 5 * B
    assert list(rt.idx[0, t]) == [0, 1, 5]      # four blocks score 2: the two lowest win
    assert rt.margin[0, t] == 0.0                # exact tie at the boundary


def test_gate_margin_and_boundary_hand_derived():
    """The near-tie fields of a row with distinct scores, worked out by hand.

    Past scores of block 7 (head 0, q = e_1): w[0..6] = 3, -1, 5, 0, 2, 7, 1. With topk = 4 the
    three best past blocks score 7, 5, 3; the first unselected scores 2, so
    margin = (3 - 2) / max(|3|, |2|) = 1/3 and boundary = 2. Head 1 (q = -e_1) sees -w: the three
    best are 1, 0, -1, the first unselected -2: margin = (-1 - (-2)) / 2 = 1/2, boundary = -2.
    """
    B = 4
    w = [3, -1, 5, 0, 2, 7, 1, 4]
    k = _const_block_keys(w, B)
    T = k.shape[0]
    c = ref.centroids(k, [0, T], B)
    q = np.zeros((T, 2, 4), np.float32)
    q[:, 0, 0] = 1.0
    q[:, 1, 0] = -1.0
    rt = ref.select_blocks(q, c, [0, T], B, 4)
    t = 7 * B + 2
    assert rt.margin[0, t] == pytest.approx(1.0 / 3.0, abs=1e-15)
    assert rt.boundary[0, t] == 2.0
    assert rt.margin[1, t] == pytest.approx(0.5, abs=1e-15)
    assert rt.boundary[1, t] == -2.0
    # magnitude: q = +-e_1, so sum_i |q_i c_i| of a block is |w_j|: max(|3|, |2|) and max(1, 2)
    assert rt.magnitude[0, t] == 3.0 and rt.magnitude[1, t] == 2.0
    # block 5 (past 3, -1, 5, 0, 2; top-3 = 5, 3, 2; next 0): margin (2 - 0) / 2 = 1
    t5 = 5 * B
    assert rt.margin[0, t5] == pytest.approx(1.0, abs=1e-15)
    assert rt.boundary[0, t5] == 0.0
    # every past block kept (k - 1 >= i): no boundary, no tie possible
    assert np.isnan(rt.boundary[0, 3 * B]) and rt.margin[0, 3 * B] == np.inf
    # a positive rescale of q scales the boundary and the magnitude, not the (relative) margin
    rt2 = ref.select_blocks(2.0 * q, c, [0, T], B, 4)
    assert rt2.boundary[0, t] == 4.0 and rt2.magnitude[0, t] == 6.0
    assert rt2.margin[0, t] == pytest.approx(1.0 / 3.0, abs=1e-15)
    # topk = 1 selects no past block: margin is infinite whatever the scores
    rt1 = ref.select_blocks(q, c, [0, T], B, 1)
    assert rt1.margin[0, t] == np.inf


def test_gate_magnitude_sums_absolute_terms():
    """magnitude sums |q_i| |c_i| over the dimensions: scores that cancel keep a large magnitude.
    Block j's keys are (a_j, -a_j) in two dimensions and q = (1, 1), so every score is 0 while the
    magnitude of block j is 2 |a_j|."""
    B = 2
    a = [1.0, 3.0, 2.0, 0.5, 4.0]
    T = len(a) * B
    k = np.zeros((T, 1, 2), np.float32)
    for j, aj in enumerate(a):
        k[j * B:(j + 1) * B, 0, 0] = aj
        k[j * B:(j + 1) * B, 0, 1] = -aj
    q = np.ones((T, 1, 2), np.float32)
    c = ref.centroids(k, [0, T], B)
    rt = ref.select_blocks(q, c, [0, T], B, 3)
    t = 4 * B
    # all four past scores are 0: ties go to the lower blocks, so 0 and 1 are kept, 2 is next
    assert list(rt.idx[0, t]) == [0, 1, 4]
    assert rt.boundary[0, t] == 0.0 and rt.margin[0, t] == 0.0
    assert rt.magnitude[0, t] == max(2 * a[1], 2 * a[2])


def test_gate_scores_hand_derived_gqa():
    """gate_scores of a GQA layout (Hq = 4, Hkv = 2): query head h reads kv head h // 2.

    Keys are constant inside each block: kv head 0 carries w0[j] e_1, kv head 1 carries w1[j] e_1,
    and query head h is (h + 1) e_1, so the score of past block j is (h + 1) * w_{h // 2}[j].
    """
    B, d = 4, 4
    w0 = [1.0, -2.0, 3.0, 0.5, 4.0]
    w1 = [-1.0, 6.0, 0.25, 2.0, -3.0]
    T = len(w0) * B
    k = np.zeros((T, 2, d), np.float32)
    for j in range(len(w0)):
        k[j * B:(j + 1) * B, 0, 0] = w0[j]
        k[j * B:(j + 1) * B, 1, 0] = w1[j]
    q = np.zeros((T, 4, d), np.float32)
    for h in range(4):
        q[:, h, 0] = h + 1
    c = ref.centroids(k, [0, T], B)
    t = 4 * B + 1  # block 4: past blocks 0..3
    for h in range(4):
        want = [(h + 1) * wj for wj in (w0 if h < 2 else w1)[:4]]
        np.testing.assert_array_equal(ref.gate_scores(q, c, [0, T], B, t, h), want)
    # varlen: the second sequence's block 1 scores only that sequence's block 0
    cu = [0, 2 * B, 4 * B]
    c2 = ref.centroids(k[:4 * B], cu, B)
    s = ref.gate_scores(q[:4 * B], c2, cu, B, 3 * B, 3)
    np.testing.assert_array_equal(s, [4 * w1[2]])
    assert ref.gate_scores(q, c, [0, T], B, 2, 0).shape == (0,)  # block 0 has no past


def test_gate_brute_force_random():
    rng = np.random.default_rng(5)
    B, d, G, H = 4, 8, 2, 4
    cu = [0, 37, 70]
    T = cu[-1]
    q = rng.standard_normal((T, H, d))
    k = rng.standard_normal((T, G, d))
    c = ref.centroids(k, cu, B)
    for topk in (1, 2, 3, 5):
        rt = ref.select_blocks(q, c, cu, B, topk)
        bt = ref.block_table(cu, B)
        s_of, i_of = ref.token_position(cu, B, np.arange(T))
        for t in range(T):
            s, i = int(s_of[t]), int(i_of[t])
            base = int(bt.blk_off[s])
            for h in range(H):
                g = h // (H // G)
                scores = np.array([float(np.dot(q[t, h], c[base + j, g])) for j in range(i)])
                want = ref.topk_by_enumeration(scores, topk - 1) + [i] if i > 0 else [0]
                got = [x for x in rt.idx[h, t] if x >= 0]
                assert got == sorted(want), (t, h, topk)


# ----------------------------------------------------------------------------- full-attn limit
@pytest.mark.parametrize("cu,hq,hkv,d,B", [
    ([0, 96], 1, 1, 16, 16),
    ([0, 50, 50, 131], 4, 2, 8, 16),      # varlen, empty sequence, ragged tails, GQA 2:1
    ([0, 70], 6, 3, 32, 64),
])
def test_full_attention_limit(cu, hq, hkv, d, B):
    w, q, k, v = _inputs(cu, hq, hkv, d, B, 1)
    nb_max = max(w.seq_blocks())
    scale = 1.0 / math.sqrt(d)
    rt, out, lse = ref.forward(q, k, v, cu, B, nb_max + 1, scale)
    o_ref, lse_ref = ref.causal_attention(q, k, v, cu, scale)
    np.testing.assert_allclose(out, o_ref, atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=1e-12)
    # independent library reference: torch SDPA in float64, per sequence, GQA expanded
    r = hq // hkv
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if a == b:
            continue
        qs = q[a:b].double().permute(1, 0, 2)
        ks = k[a:b].double().permute(1, 0, 2).repeat_interleave(r, dim=0)
        vs = v[a:b].double().permute(1, 0, 2).repeat_interleave(r, dim=0)
        o_sdpa = torch.nn.functional.scaled_dot_product_attention(
            qs, ks, vs, is_causal=True, scale=scale).permute(1, 0, 2).numpy()
        np.testing.assert_allclose(out[a:b], o_sdpa, atol=1e-12, rtol=1e-10)


def test_topk1_is_block_diagonal_causal():
    cu = [0, 45, 100]
    B = 16
    w, q, k, v = _inputs(cu, 4, 2, 16, B, 1)
    scale = 0.3
    rt, out, lse = ref.forward(q, k, v, cu, B, 1, scale)
    bt = ref.block_table(cu, B)
    cu_blocks = [int(x) for x in bt.start] + [cu[-1]]
    o_bd, lse_bd = ref.causal_attention(q, k, v, cu_blocks, scale)
    np.testing.assert_allclose(out, o_bd, atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(lse, lse_bd, atol=1e-12, rtol=1e-12)


# ------------------------------------------------------------------------- second formulation
@pytest.mark.parametrize("topk", [2, 3, 5])
def test_gather_form_equals_dense_mask_form(topk):
    cu = [0, 61, 61, 160]
    B = 16
    w, q, k, v = _inputs(cu, 4, 2, 16, B, topk, keys="clusters")
    scale = 1.0 / 4.0
    rt, out, lse = ref.forward(q, k, v, cu, B, topk, scale)
    mask = ref.dense_mask(cu, B, rt.idx)
    o_d, lse_d = ref.attention_dense(q, k, v, mask, scale)
    np.testing.assert_allclose(out, o_d, atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(lse, lse_d, atol=1e-12, rtol=1e-12)


def test_sampled_rows_equal_all_rows():
    cu = [0, 200]
    B = 32
    w, q, k, v = _inputs(cu, 2, 1, 16, B, 3)
    rt_all, o_all, lse_all = ref.forward(q, k, v, cu, B, 3, 0.25)
    toks = [0, 31, 32, 100, 199]
    rt_s, o_s, lse_s = ref.forward(q, k, v, cu, B, 3, 0.25, tokens=toks)
    np.testing.assert_array_equal(rt_s.idx, rt_all.idx[:, toks])
    np.testing.assert_allclose(o_s, o_all[toks], atol=1e-13)
    np.testing.assert_allclose(lse_s, lse_all[:, toks], atol=1e-13)


# --------------------------------------------------------------------------------- invariants
def test_invariants():
    cu = [0, 90, 200]
    B, topk, scale = 16, 4, 0.2
    w, q, k, v = _inputs(cu, 4, 4, 8, B, topk, keys="clusters", seed=3)
    rt, out, lse = ref.forward(q, k, v, cu, B, topk, scale)
    T = cu[-1]
    s_of, i_of = ref.token_position(cu, B, np.arange(T))
    bt = ref.block_table(cu, B)
    qf, kf, vf = ref.to_f64(q), ref.to_f64(k), ref.to_f64(v)
    for t in range(T):
        i = int(i_of[t])
        for h in range(4):
            row = list(rt.idx[h, t])
            S = [x for x in row if x >= 0]
            assert row == S + [-1] * (topk - len(S))      # valid first, -1 padding last
            assert S == sorted(set(S))                   # ascending, distinct
            assert i in S                                # current block always selected
            assert max(S) == i                           # no future block
            assert len(S) == min(topk, i + 1)
            base = int(bt.blk_off[s_of[t]])
            keys = [u for j in S for u in range(bt.start[base + j], min(bt.end[base + j], t + 1))]
            z = scale * (kf[keys, h] @ qf[t, h])
            assert lse[h, t] >= z.max() - 1e-12
            assert lse[h, t] <= z.max() + math.log(len(keys)) + 1e-12
            vv = vf[keys, h]
            assert np.all(out[t, h] >= vv.min(axis=0) - 1e-12)
            assert np.all(out[t, h] <= vv.max(axis=0) + 1e-12)
    # softmax rows sum to one: attending constant values returns that constant
    ones = torch.ones_like(v)
    _, o1, _ = ref.forward(q, k, ones, cu, B, topk, scale)
    np.testing.assert_allclose(o1, 1.0, atol=1e-12)


# ------------------------------------------------------------------------------------- golden
def test_golden_hand_worked_example():
    with open(os.path.join(GOLDEN, "moba_tiny_handworked.json")) as f:
        gd = json.load(f)
    q = np.array(gd["q"], np.float32)[:, None, :]
    k = np.array(gd["k"], np.float32)[:, None, :]
    v = np.array(gd["v"], np.float32)[:, None, :]
    for case in gd["cases"]:
        rt, out, lse = ref.forward(q, k, v, gd["cu_seqlens"], gd["block_size"], case["topk"],
                                   gd["scale"])
        np.testing.assert_array_equal(rt.idx[0], np.array(case["idx"], np.int32))
        np.testing.assert_allclose(out[:, 0, :], _closed_form(case["o"]), atol=1e-12)
        np.testing.assert_allclose(lse[0], _closed_form(case["lse"]), atol=1e-12)


def _closed_form(expr):
    """Evaluate the hand-derived closed-form strings of the golden file (exp/log only)."""
    if isinstance(expr, list):
        return np.array([_closed_form(e) for e in expr], np.float64)
    return float(eval(expr, {"__builtins__": {}}, {"exp": math.exp, "log": math.log}))
