"""Pins of the oracle's decode / chunked-prefill rows (CPU only).

decode() evaluates the prefill rule at the newest n_s tokens of each cached sequence. Pinned by
closed forms (a one-token cache; a cache shorter than topk blocks is plain causal attention of one
query over all cached keys), by the prefill forward pass at the same positions (one row, a chunk
of rows, and every row of the sequence), and by the row-position rule itself.
"""
import math

import numpy as np
import pytest

from block_sparse_long_moba_b200 import workloads as wl
from oracle import moba_ref as ref


def _cache(cu, hq, hkv, d, B, topk, keys="offset", seed=0):
    w = wl.custom(cu, hq, hkv, d, B, topk, keys)
    q, k, v, _ = wl.make_inputs(w, seed=seed, device="cpu")
    return q, k, v


def test_row_positions():
    # sequence 0: 10 tokens, 1 row -> 9; sequence 1: empty; sequence 2: 15 tokens, 3 rows
    np.testing.assert_array_equal(ref.cache_row_positions([0, 10, 10, 25], [0, 1, 1, 4]),
                                  [9, 22, 23, 24])
    np.testing.assert_array_equal(ref.cache_row_positions([0, 3], [0, 3]), [0, 1, 2])
    with pytest.raises(AssertionError):
        ref.cache_row_positions([0, 3], [0, 4])   # more rows than cached tokens


def test_one_token_cache_closed_form():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 2, 8))
    k = rng.standard_normal((1, 1, 8))
    v = rng.standard_normal((1, 1, 8))
    rt, o, lse = ref.decode(q, k, v, [0, 1], [0, 1], 16, 3, 0.5)
    assert list(rt.idx[0, 0]) == [0, -1, -1]
    for h in range(2):
        np.testing.assert_allclose(o[0, h], v[0, 0], rtol=0, atol=1e-15)
        assert lse[h, 0] == pytest.approx(0.5 * float(q[0, h] @ k[0, 0]), abs=1e-14)


def test_short_cache_is_full_attention_of_the_last_query():
    """With topk >= the number of blocks the row attends every cached key: a textbook softmax
    of one query over L keys."""
    rng = np.random.default_rng(1)
    L, d, B = 45, 8, 16
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((L, 1, d))
    v = rng.standard_normal((L, 1, d))
    scale = 1 / math.sqrt(d)
    _, o, lse = ref.decode(q, k, v, [0, L], [0, 1], B, 3, scale)
    z = scale * (k[:, 0] @ q[0, 0])
    p = np.exp(z - z.max())
    np.testing.assert_allclose(o[0, 0], (p / p.sum()) @ v[:, 0], rtol=1e-12, atol=1e-14)
    assert lse[0, 0] == pytest.approx(z.max() + math.log(p.sum()), abs=1e-12)


@pytest.mark.parametrize("cuq", [[0, 1, 2, 2, 3], [0, 7, 20, 20, 21], [0, 300, 340, 340, 1040]])
def test_rows_equal_prefill_rows(cuq):
    """Decode rows (one, a chunk, or the whole sequence) equal the prefill forward pass at the
    same positions, routing included."""
    cu = [0, 300, 340, 340, 1040]  # includes an empty sequence
    B, topk, scale = 32, 4, 0.25
    q, k, v = _cache(cu, 4, 2, 16, B, topk, "clusters")
    pos = ref.cache_row_positions(cu, cuq)
    rt, o, lse = ref.decode(q[pos], k, v, cu, cuq, B, topk, scale)
    rt_f, o_f, lse_f = ref.forward(q, k, v, cu, B, topk, scale, tokens=pos)
    np.testing.assert_array_equal(rt.idx, rt_f.idx)
    np.testing.assert_allclose(o, o_f, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, lse_f, rtol=0, atol=1e-14)
