"""Shared checks of the CUDA path against the fp64 oracle (used by the GPU tests and smoke())."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moba_ref as ref

# Tolerances of the forward pass: |O - O_ref| <= O_ATOL + O_RTOL |O_ref| (elementwise, O read
# back from bf16 as fp32), |LSE - LSE_ref| <= LSE_ATOL. Gate near-tie band: rows whose last
# selected and first unselected past scores a, b differ by less than
#   max(TIE_REL * max(|a|, |b|), TIE_COND * M),   M = max over the two blocks of sum_i |q_i c_i|,
# may pick either block; attention is then checked on the GPU's own selection. The first term is
# the stated relative band. The second is the rounding of a score computed in fp32 arithmetic:
# the kernel's split-bf16 centroids leave a residual below 2^-17 of each term and fp32
# accumulation over d <= 128 terms adds below 128 * 2^-24 = 2^-17, so one score is within 2^-16 M
# and a difference of two within 2^-15 M; TIE_COND doubles that. The second term only matters
# when the two scores nearly cancel (|a|, |b| much smaller than M). TIE_ROWS_MAX bounds the share
# of checked rows that may be excused as near ties on the full-size workloads.
O_ATOL = 1e-2
O_RTOL = 1e-2
LSE_ATOL = 1e-3
TIE_REL = 1e-4
TIE_COND = 2.0 ** -14
TIE_ROWS_MAX = 1e-3


def check_routing(q_cpu, cents64, cu, B, topk, tokens, idx_gpu_rows, *, allow_ties=True):
    """Compare the GPU routing of the sampled rows with the oracle's.

    idx_gpu_rows: [H, n, topk] int32 (GPU routing of the sampled tokens).
    Exact match is required except on near-tie rows, where the GPU's set must still be valid:
    current block present, no future block, right count, ascending and distinct, and every chosen
    past block within the tie band of the oracle's boundary. Returns the number of tie rows.
    """
    rt = ref.select_blocks(q_cpu, cents64, cu, B, topk, tokens)
    H, n, _ = rt.idx.shape
    diff = np.any(rt.idx != idx_gpu_rows, axis=2)  # [H, n]
    s_of, i_of = ref.token_position(cu, B, tokens)
    ties = 0
    for h, nn in zip(*np.nonzero(diff)):
        t = int(tokens[nn])
        i = int(i_of[nn])
        got = [int(x) for x in idx_gpu_rows[h, nn]]
        sel = [x for x in got if x >= 0]
        assert got == sel + [-1] * (topk - len(sel)), (h, t, got)
        assert sel == sorted(set(sel)), (h, t, got)
        assert i in sel and max(sel) == i, (h, t, got)
        assert len(sel) == min(topk, i + 1), (h, t, got)
        scores = ref.gate_scores(q_cpu, cents64, cu, B, t, int(h))
        order = np.sort(scores)[::-1]
        a, b = order[topk - 2], order[topk - 1]
        tol = max(TIE_REL * max(abs(a), abs(b)), TIE_COND * rt.magnitude[h, nn])
        assert allow_ties and a - b <= tol, (
            f"routing mismatch outside the tie band: head {h} token {t} gpu {got} "
            f"oracle {list(rt.idx[h, nn])} margin {rt.margin[h, nn]} gap {a - b} band {tol}")
        past = [x for x in sel if x != i]
        unchosen = [j for j in range(i) if j not in past]
        assert all(scores[j] >= a - tol for j in past), (h, t, got)
        assert all(scores[j] <= b + tol for j in unchosen), (h, t, got)
        ties += 1
    return ties


def check_outputs(o_gpu_rows, lse_gpu_rows, o_ref, lse_ref):
    """o_*: [n, H, d]; lse_*: [H, n]. Raises AssertionError with the worst offender."""
    o = o_gpu_rows.astype(np.float64)
    err = np.abs(o - o_ref)
    bound = O_ATOL + O_RTOL * np.abs(o_ref)
    bad = err > bound
    if bad.any():
        w = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"O mismatch at {w}: gpu {o[w]} ref {o_ref[w]} "
                             f"({int(bad.sum())} of {bad.size} elements out of tolerance)")
    lerr = np.abs(lse_gpu_rows.astype(np.float64) - lse_ref)
    if (lerr > LSE_ATOL).any():
        w = np.unravel_index(np.argmax(lerr), lerr.shape)
        raise AssertionError(f"LSE mismatch at {w}: gpu {lse_gpu_rows[w]} ref {lse_ref[w]}")
    return float(err.max()), float(lerr.max())


def run_and_check(moba, q, k, v, cu, cu_host, B, topk, scale, tokens=None, block_idx_in=None):
    """Run moba_attn_fwd on the GPU and check routing, O and LSE of the sampled rows."""
    T = q.shape[0]
    H = q.shape[1]
    idx_out = torch.empty((H, T, topk), dtype=torch.int32, device=q.device)
    o, lse = moba.moba_attn_fwd(q, k, v, cu, cu_host, B, topk, scale,
                                block_idx_in=block_idx_in, block_idx_out=idx_out)
    torch.cuda.synchronize()
    if tokens is None:
        tokens = np.arange(T)
    tokens = np.asarray(tokens, np.int64)
    q_c, k_c, v_c = q.cpu(), k.cpu(), v.cpu()
    tok_t = torch.as_tensor(tokens)
    idx_rows = idx_out.cpu()[:, tok_t].numpy()
    ties = 0
    if block_idx_in is None:
        cents = ref.centroids(k_c, cu_host, B)
        ties = check_routing(q_c, cents, cu_host, B, topk, tokens, idx_rows)
    o_ref, lse_ref = ref.attention(q_c, k_c, v_c, cu_host, B, idx_rows, scale, tokens)
    o_rows = o.cpu()[tok_t].float().numpy()
    lse_rows = lse.cpu()[:, tok_t].numpy()
    errs = check_outputs(o_rows, lse_rows, o_ref, lse_ref)
    return {"ties": ties, "max_o_err": errs[0], "max_lse_err": errs[1], "o": o, "lse": lse,
            "idx": idx_out}
