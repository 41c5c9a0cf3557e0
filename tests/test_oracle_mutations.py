"""Plant plausible mistakes in the oracle (on the CPU) and check that some pin catches each one."""
import numpy as np
import pytest

from oracle import moba_ref as ref
from tests import test_oracle as pins

_orig_centroids = ref.centroids
_orig_select = ref.select_blocks
_orig_attention = ref.attention


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


@pytest.mark.parametrize("target,fake,pin", [
    ("centroids", _sum_not_mean, pins.test_centroid_closed_form_with_ragged_tail),
    ("select_blocks", _negated_gate, pins.test_gate_constructed_case),
    ("select_blocks", _gqa_modulo, pins.test_gate_brute_force_random),
    ("attention", _no_causal_cut, pins.test_topk1_is_block_diagonal_causal),
])
def test_pin_catches_planted_mistake(monkeypatch, target, fake, pin):
    monkeypatch.setattr(ref, target, fake)
    with pytest.raises(AssertionError):
        pin()
