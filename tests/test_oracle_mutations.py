"""Plant plausible mistakes in the oracle (on the CPU) and check that some pin catches each one."""
import numpy as np
import pytest

from oracle import moba_ref as ref
from tests import test_oracle as pins
from tests import test_oracle_decode as dpins
from tests import test_oracle_kconv as kpins

_orig_centroids = ref.centroids
_orig_select = ref.select_blocks
_orig_attention = ref.attention
_orig_gate_scores = ref.gate_scores
_orig_key_conv = ref.key_conv


def _sum_not_mean(k, cu, B):
    bt = ref.block_table(cu, B)
    c = _orig_centroids(k, cu, B)
    n = (bt.end - bt.start).astype(np.float64)
    return c * n[:, None, None]


def _gqa_modulo(q, cents, cu, B, topk, tokens=None):
    # wrong head grouping inside the gate: query head h scored against kv head h % G
    # instead of h // (H/G); emulated by permuting the kv heads of the centroids
    H, G = q.shape[1], cents.shape[1]
    r = H // G
    # the gate reads kv head h // r; make that read return kv head (h % G) for the first head of
    # every group, i.e. swap kv heads through the map g -> (g * r) % G
    perm = [(g * r) % G for g in range(G)]
    return _orig_select(q, cents[:, perm, :], cu, B, topk, tokens)


def _no_causal_cut(q, k, v, cu, B, idx, scale, tokens):
    # drop the causal restriction inside the current block: attend the whole block
    t = np.asarray(tokens)
    bt = ref.block_table(cu, B)
    shifted = t.copy()
    for n, tok in enumerate(t):
        for b in range(bt.num_blocks):
            if bt.start[b] <= tok < bt.end[b]:
                shifted[n] = bt.end[b] - 1
    o, l = _orig_attention(q, k, v, cu, B, idx, scale, shifted)
    return o, l


def _negated_gate(q, cents, cu, B, topk, tokens=None):
    return _orig_select(q, -cents, cu, B, topk, tokens)


def _margin_off_by_one(q, cents, cu, B, topk, tokens=None):
    # near-tie fields taken one position too deep in the score order: the k-th and (k+1)-th best
    # past scores instead of the (k-1)-th and k-th
    rt = _orig_select(q, cents, cu, B, topk, tokens)
    H, G = q.shape[1], cents.shape[1]
    bt = ref.block_table(cu, B)
    s_of, i_of = ref.token_position(cu, B, rt.tokens)
    for n, t in enumerate(rt.tokens):
        s, i = int(s_of[n]), int(i_of[n])
        if topk - 1 >= i or topk < 2:
            continue
        for h in range(H):
            qf = ref.to_f64(q[int(t):int(t) + 1])[0, h]
            sc = cents[int(bt.blk_off[s]):int(bt.blk_off[s]) + i, h // (H // G)] @ qf
            order = np.argsort(-sc, kind="stable")
            a = sc[order[topk - 1]]
            b = sc[order[topk]] if topk < i else np.nan
            rt.boundary[h, n] = b
            den = max(abs(a), abs(b)) if not np.isnan(b) else 1.0
            rt.margin[h, n] = (a - b) / den if den > 0 else 0.0
    return rt


def _gate_scores_gqa_modulo(q, cents, cu, B, token, head):
    # wrong head grouping in the per-row scores: kv head h % G instead of h // (H/G)
    G = cents.shape[1]
    H = q.shape[1]
    perm_head = (head % G) * (H // G)  # a head of the group the modulo map picks
    return _orig_gate_scores(q, cents, cu, B, token, perm_head) * (head + 1) / (perm_head + 1)


def _magnitude_of_the_sum(q, cents, cu, B, topk, tokens=None):
    # magnitude taken as |sum_i q_i c_i| (the score itself) instead of sum_i |q_i c_i|
    rt = _orig_select(q, cents, cu, B, topk, tokens)
    rt.magnitude = np.where(np.isnan(rt.boundary), 0.0,
                            np.maximum(np.abs(rt.boundary),
                                       np.abs(rt.boundary) * (1 + np.nan_to_num(rt.margin))))
    return rt


def _conv_across_blocks(k, conv_w, cu, B):
    # the convolution reaches back into the previous block (one long sequence per cu segment)
    return _orig_key_conv(k, conv_w, cu, 10 ** 9)


def _conv_anticausal(k, conv_w, cu, B):
    # the kernel applied to later keys (t + m) instead of earlier ones
    kf = ref.to_f64(k)[::-1].copy()
    T = kf.shape[0]
    bt = ref.block_table(cu, B)
    rev_cu = [0] + [T - int(x) for x in bt.start[::-1]]
    out = _orig_key_conv(kf, conv_w, rev_cu, 10 ** 9)
    return out[::-1].copy()


def _rows_at_the_front(cu, cuq):
    # query rows taken as the first n_s tokens of each sequence instead of the last
    cu, cuq = [int(x) for x in cu], [int(x) for x in cuq]
    return np.asarray([cu[s] + x for s in range(len(cu) - 1) for x in range(cuq[s + 1] - cuq[s])],
                      np.int64)


@pytest.mark.parametrize("target,fake,pin", [
    ("centroids", _sum_not_mean, pins.test_centroid_closed_form_with_ragged_tail),
    ("select_blocks", _negated_gate, pins.test_gate_constructed_case),
    ("select_blocks", _gqa_modulo, pins.test_gate_brute_force_random),
    ("attention", _no_causal_cut, pins.test_topk1_is_block_diagonal_causal),
    ("select_blocks", _margin_off_by_one, pins.test_gate_margin_and_boundary_hand_derived),
    ("gate_scores", _gate_scores_gqa_modulo, pins.test_gate_scores_hand_derived_gqa),
    ("select_blocks", _magnitude_of_the_sum, pins.test_gate_magnitude_sums_absolute_terms),
    ("key_conv", _conv_across_blocks, kpins.test_convolution_stops_at_the_block_start),
    ("key_conv", _conv_anticausal, kpins.test_pure_delay_closed_form),
    ("cache_row_positions", _rows_at_the_front, dpins.test_row_positions),
])
def test_pin_catches_planted_mistake(monkeypatch, target, fake, pin):
    monkeypatch.setattr(ref, target, fake)
    with pytest.raises(AssertionError):
        pin()
