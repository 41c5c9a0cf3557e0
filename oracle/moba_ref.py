"""Plain fp64 CPU oracle of the MoBA causal prefill forward pass.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module: only tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline / reference legs use it. It shares no code
with the CUDA path (no kernels, headers, helpers or table generators) and is slow on purpose.

What it computes, in the order the method describes it (plus, for the trainable layer, the
gradients of step 4 with the routing held fixed: attention_backward):
  1. Keys are cut into fixed-size blocks per sequence; blocks never cross cu_seqlens
     [MoBA README (rpkg.in mirror), "Introducing MoBA": the context is divided into blocks].
  2. Each block is represented by the mean of its keys, per kv head
     [MoBA paper summary (atlas.scime.ai), "Approach": query - mean-pooled-key inner product].
  3. Every query head scores each PAST block of its own sequence by q . centroid (no learned
     weights), never scores future blocks, always keeps its own current block and routes to the
     top-k blocks, the current one included [same page, "Approach"; MoBA README, "Parameter-less
     Gating Mechanism"].
  4. Attention is exact softmax attention over the keys of the selected blocks, restricted to
     key positions <= the query inside the current block [same page, "Approach": causal].

Readings where the pages are silent (the plainest reading of each, stated here):
  * centroid = mean over the keys actually present (a ragged last block averages fewer keys);
  * gate score = unscaled q . c in fp64; ties go to the lower block index;
  * the current block counts toward k; with k-1 >= i every block 0..i is selected;
  * block indices are local to the sequence, emitted ascending, padded with -1;
  * GQA: query head h uses kv head h // (Hq / Hkv);
  * LSE is the natural log of the sum of exp(scale * q . k) over the attended keys.

Evaluation order (no rescaling tricks): the logit max of every row is found in a first pass over
the blocks, then exp(z - max), its sum and the value-weighted sum are accumulated block by block
in fp64. Logits are formed with numpy matmuls (a library primitive). Every function is
pinned by tests/test_oracle.py against closed forms, textbook attention, brute force and a second
(dense-mask) formulation.
"""
from __future__ import annotations

import itertools
import math
from dataclasses import dataclass
from typing import List, Sequence

import numpy as np


def to_f64(x) -> np.ndarray:
    """bf16/fp32 torch tensor or numpy array -> fp64 numpy array (exact upcast)."""
    if isinstance(x, np.ndarray):
        return x.astype(np.float64)
    import torch  # only for the dtype conversion of torch inputs

    return x.detach().to("cpu").to(torch.float64).numpy()


@dataclass
class BlockTable:
    """Global block numbering: sequences in order, blocks of each sequence in order."""

    blk_off: np.ndarray  # [nseq+1] first global block of every sequence
    seq: np.ndarray      # [NB] sequence of each global block
    local: np.ndarray    # [NB] index of the block inside its sequence
    start: np.ndarray    # [NB] first token (absolute)
    end: np.ndarray      # [NB] one past the last token (absolute)

    @property
    def num_blocks(self) -> int:
        return int(self.seq.shape[0])


def block_table(cu_seqlens: Sequence[int], block_size: int) -> BlockTable:
    """Split every sequence [cu[s], cu[s+1]) into ceil(L_s / B) blocks of B keys (last may be short)."""
    cu = [int(x) for x in cu_seqlens]
    B = int(block_size)
    off, seq, loc, st, en = [0], [], [], [], []
    for s in range(len(cu) - 1):
        L = cu[s + 1] - cu[s]
        nb = (L + B - 1) // B
        for j in range(nb):
            seq.append(s)
            loc.append(j)
            st.append(cu[s] + j * B)
            en.append(min(cu[s] + (j + 1) * B, cu[s + 1]))
        off.append(off[-1] + nb)
    return BlockTable(np.array(off, np.int64), np.array(seq, np.int64), np.array(loc, np.int64),
                      np.array(st, np.int64), np.array(en, np.int64))


def token_position(cu_seqlens: Sequence[int], block_size: int, tokens) -> tuple:
    """For absolute token positions: (sequence s, local block i = floor((t - cu[s]) / B))."""
    cu = np.asarray([int(x) for x in cu_seqlens], np.int64)
    t = np.asarray(tokens, np.int64)
    s = np.searchsorted(cu, t, side="right") - 1
    i = (t - cu[s]) // int(block_size)
    return s, i


def centroids(k, cu_seqlens, block_size) -> np.ndarray:
    """Mean-pooled key of every block: c[b, g, :] = mean of K[t, g, :] over the block's keys.

    [MoBA paper summary (atlas.scime.ai), "Approach": mean-pooled key]. Returns [NB, Hkv, d] fp64.
    """
    bt = block_table(cu_seqlens, block_size)
    G, d = int(k.shape[1]), int(k.shape[2])
    out = np.zeros((bt.num_blocks, G, d), np.float64)
    for b in range(bt.num_blocks):
        kb = to_f64(k[int(bt.start[b]):int(bt.end[b])])  # [n_b, G, d]
        out[b] = kb.sum(axis=0) / kb.shape[0]
    return out


def key_conv(k, conv_w, cu_seqlens, block_size) -> np.ndarray:
    """Short depthwise causal convolution of the keys inside each block, per kv head and channel:

      kconv[t, g, :] = sum_{m=0}^{W-1} w[m, g, :] * k[t - m, g, :],  terms with t - m before the
      first key of t's block left out (the convolution never reaches into another block).

    [FlashMoBA story: short convolutions applied within blocks cluster related keys and raise the
    routing signal.] The pages give no kernel width, weights or activation; the plainest reading
    is a linear depthwise convolution with given weights w [W, Hkv, d], no bias or activation.
    Returns [T, Hkv, d] fp64."""
    kf = to_f64(k)
    w = to_f64(conv_w)
    W = w.shape[0]
    bt = block_table(cu_seqlens, block_size)
    out = np.zeros_like(kf)
    for b in range(bt.num_blocks):
        st, en = int(bt.start[b]), int(bt.end[b])
        for t in range(st, en):
            for m in range(W):
                if t - m >= st:
                    out[t] += w[m] * kf[t - m]
    return out


def centroids_kconv(k, conv_w, cu_seqlens, block_size) -> np.ndarray:
    """Centroids of the convolved keys: the mean over each block of key_conv(...) [FlashMoBA story:
    the short convolution is applied before the keys are pooled]. Returns [NB, Hkv, d] fp64."""
    return centroids(key_conv(k, conv_w, cu_seqlens, block_size), cu_seqlens, block_size)


@dataclass
class Routing:
    """Block selection for a set of query tokens (all heads)."""

    tokens: np.ndarray   # [n] absolute positions
    idx: np.ndarray      # [H, n, topk] int32, ascending local block ids, -1 padded
    margin: np.ndarray   # [H, n] relative gap between last selected and first unselected past score
    boundary: np.ndarray  # [H, n] the first unselected past score (nan if every past block is kept)
    # [H, n] max over those two blocks of sum_i |q_i c_i|: the size of the terms each score sums,
    # which bounds the rounding error of a score evaluated in floating point (0 if none)
    magnitude: np.ndarray


def select_blocks(q, cents: np.ndarray, cu_seqlens, block_size, topk, tokens=None) -> Routing:
    """Parameter-less causal top-k gating.

    For query t in local block i of sequence s and head h (kv head g = h // (Hq/Hkv)):
      score_j = q[t, h] . c[s, j, g]  for the past blocks j < i only (future blocks never scored);
      S = {i} U top-(k-1) past blocks by score (ties to the lower j); if k-1 >= i, S = {0..i}.
    [MoBA paper summary (atlas.scime.ai), "Approach"; MoBA README, "Parameter-less Gating".]
    """
    H = int(q.shape[1])
    G = int(cents.shape[1])
    r = H // G
    T = int(q.shape[0])
    if tokens is None:
        tokens = np.arange(T, dtype=np.int64)
    tokens = np.asarray(tokens, np.int64)
    n = tokens.shape[0]
    k = int(topk)
    bt = block_table(cu_seqlens, block_size)
    s_of, i_of = token_position(cu_seqlens, block_size, tokens)
    idx = np.full((H, n, k), -1, np.int32)
    margin = np.full((H, n), np.inf)
    boundary = np.full((H, n), np.nan)
    magnitude = np.zeros((H, n))
    # group query tokens by (sequence, local block): they share the same candidate blocks
    keys = s_of * (1 << 32) + i_of
    for key in np.unique(keys):
        rows = np.nonzero(keys == key)[0]
        s, i = int(s_of[rows[0]]), int(i_of[rows[0]])
        if k - 1 >= i:
            chosen = np.arange(i + 1, dtype=np.int32)
            idx[:, rows, : i + 1] = chosen[None, None, :]
            continue
        qf = to_f64(q[tokens[rows]])  # [m, H, d]
        base = int(bt.blk_off[s])
        for h in range(H):
            g = h // r
            c_past = cents[base:base + i, g, :]        # [i, d]
            sc = qf[:, h, :] @ c_past.T                # [m, i]
            # a stable sort of -score keeps the lower block index first on equal scores
            order = np.argsort(-sc, axis=1, kind="stable")
            top = np.sort(order[:, : k - 1], axis=1)
            idx[h, rows, : k - 1] = top
            idx[h, rows, k - 1] = i
            m = np.arange(len(rows))
            a = sc[m, order[:, k - 2]] if k >= 2 else np.full(len(rows), np.inf)
            bnd = sc[m, order[:, k - 1]]
            boundary[h, rows] = bnd
            absq = np.abs(qf[:, h, :])                                  # [m, d]
            mag_b = np.einsum("md,md->m", absq, np.abs(c_past[order[:, k - 1]]))
            mag_a = (np.einsum("md,md->m", absq, np.abs(c_past[order[:, k - 2]])) if k >= 2
                     else np.zeros(len(rows)))
            magnitude[h, rows] = np.maximum(mag_a, mag_b)
            if k >= 2:
                denom = np.maximum(np.abs(a), np.abs(bnd))
                with np.errstate(invalid="ignore", divide="ignore"):
                    margin[h, rows] = np.where(denom > 0, (a - bnd) / denom, 0.0)
            else:
                margin[h, rows] = np.inf
    return Routing(tokens, idx, margin, boundary, magnitude)


def gate_scores(q, cents: np.ndarray, cu_seqlens, block_size, token: int, head: int) -> np.ndarray:
    """All past-block scores of one (token, head): the gate's inputs, for validity checks."""
    H, G = int(q.shape[1]), int(cents.shape[1])
    bt = block_table(cu_seqlens, block_size)
    s, i = token_position(cu_seqlens, block_size, [token])
    s, i = int(s[0]), int(i[0])
    base = int(bt.blk_off[s])
    qf = to_f64(q[token:token + 1])[0, head]
    return cents[base:base + i, head // (H // G), :] @ qf


def attention(q, k, v, cu_seqlens, block_size, idx, scale, tokens) -> tuple:
    """Exact softmax attention of the given query tokens over the keys of their selected blocks.

    idx: [H, n, topk] local block ids per (head, sampled token), -1 padded (any order).
    Keys of block j are all its keys, except that in the query's own block only positions <= t
    are attended [MoBA paper summary, "Approach": causal]. Returns O [n, H, d], LSE [H, n] (fp64).
    """
    H, d = int(q.shape[1]), int(q.shape[2])
    G = int(k.shape[1])
    r = H // G
    tokens = np.asarray(tokens, np.int64)
    n = tokens.shape[0]
    bt = block_table(cu_seqlens, block_size)
    s_of, i_of = token_position(cu_seqlens, block_size, tokens)
    qf = to_f64(q[tokens])  # [n, H, d]
    sel = np.asarray(idx)
    m = np.full((H, n), -np.inf)
    lsum = np.zeros((H, n))
    acc = np.zeros((H, n, d))
    for pass_no in (0, 1):
        for b in range(bt.num_blocks):
            s, j = int(bt.seq[b]), int(bt.local[b])
            member = (sel == j).any(axis=2) & (s_of == s)[None, :]  # [H, n]
            if not member.any():
                continue
            st, en = int(bt.start[b]), int(bt.end[b])
            kb = to_f64(k[st:en])                      # [len, G, d]
            vb = to_f64(v[st:en]) if pass_no == 1 else None
            kpos = np.arange(st, en)
            for g in range(G):
                hh, nn = np.nonzero(member[g * r:(g + 1) * r])
                if hh.size == 0:
                    continue
                hh = hh + g * r
                z = scale * (qf[nn, hh, :] @ kb[:, g, :].T)          # [rows, len]
                z = np.where(kpos[None, :] <= tokens[nn][:, None], z, -np.inf)
                if pass_no == 0:
                    m[hh, nn] = np.maximum(m[hh, nn], z.max(axis=1))
                else:
                    p = np.exp(z - m[hh, nn][:, None])
                    lsum[hh, nn] += p.sum(axis=1)
                    acc[hh, nn] += p @ vb[:, g, :]
    out = (acc / lsum[..., None]).transpose(1, 0, 2)
    lse = m + np.log(lsum)
    return out, lse


def forward(q, k, v, cu_seqlens, block_size, topk, scale, tokens=None, conv_w=None):
    """Whole path: centroids -> gate -> attention. Returns (routing, O [n,H,d], LSE [H,n]).
    With conv_w the centroids pool the convolved keys (key_conv); attention reads the keys as
    given: the convolution only shapes the routing."""
    cents = (centroids(k, cu_seqlens, block_size) if conv_w is None
             else centroids_kconv(k, conv_w, cu_seqlens, block_size))
    rt = select_blocks(q, cents, cu_seqlens, block_size, topk, tokens)
    out, lse = attention(q, k, v, cu_seqlens, block_size, rt.idx, scale, rt.tokens)
    return rt, out, lse


def cache_row_positions(cu_seqlens, cu_seqlens_q) -> np.ndarray:
    """Absolute positions of query rows that are the last n_s tokens of each cached sequence:
    row r of sequence s sits at cu[s] + L_s - n_s + (r - cuq[s])."""
    cu = [int(x) for x in cu_seqlens]
    cuq = [int(x) for x in cu_seqlens_q]
    pos = []
    for s in range(len(cu) - 1):
        L, n = cu[s + 1] - cu[s], cuq[s + 1] - cuq[s]
        assert 0 <= n <= L
        pos += [cu[s] + L - n + x for x in range(n)]
    return np.asarray(pos, np.int64)


def decode(q_rows, k, v, cu_seqlens, cu_seqlens_q, block_size, topk, scale, cents=None):
    """MoBA over the newest rows of a KV cache (decode: one row per sequence).

    The rows are the last n_s tokens of each sequence, and each gets exactly what the prefill
    forward pass gives that token over its whole sequence: the same gate on the past blocks of its
    own position, the same attention up to its own position [MoBA paper summary, "Approach"; its
    "Limitations" note the paper decoded with full attention, so decode-time routing is the
    plainest reading: the prefill rule applied to the newest token]. cents: the cache's centroids
    (computed from k when None). Returns (Routing, O [Tq,H,d], LSE [H,Tq]).
    """
    tokens = cache_row_positions(cu_seqlens, cu_seqlens_q)
    qr = to_f64(q_rows)
    T = int(k.shape[0])
    q_full = np.zeros((T,) + qr.shape[1:])
    q_full[tokens] = qr
    if cents is None:
        cents = centroids(k, cu_seqlens, block_size)
    rt = select_blocks(q_full, cents, cu_seqlens, block_size, topk, tokens)
    out, lse = attention(q_full, k, v, cu_seqlens, block_size, rt.idx, scale, tokens)
    return rt, out, lse


def attention_backward(q, k, v, cu_seqlens, block_size, idx_full, scale, d_out) -> tuple:
    """Gradients of the routed attention with the routing held fixed: dQ [T,H,d], dK, dV [T,G,d].

    MoBA is trained end to end through its block-sparse attention [MoBA README, "Introducing
    MoBA": trainable block sparse attention]; the top-k gate itself is piecewise constant in q and
    the centroids, so no gradient flows through the selection, as in top-k mixture-of-experts
    routing (the pages are silent on this; it is the plainest reading). For every row (t, h)
    over its attended keys u (the keys of its selected blocks, causal inside its own block), with
    z_u = scale q.k_u, p_u = exp(z_u - LSE) and o = sum_u p_u v_u:
      dV[u] += p_u dO;  dP_u = dO . v_u;  D = dO . o;  dS_u = p_u (dP_u - D);
      dQ += scale sum_u dS_u k_u;  dK[u] += scale dS_u q.
    Keys and values of kv head g collect the terms of all query heads of its group. idx_full:
    [H, T, topk] local block ids per (head, token), -1 padded; d_out: [T, H, d]. All fp64.
    """
    qf, kf, vf, go = to_f64(q), to_f64(k), to_f64(v), to_f64(d_out)
    T, H, d = qf.shape
    G = kf.shape[1]
    r = H // G
    tokens = np.arange(T, dtype=np.int64)
    out, lse = attention(q, k, v, cu_seqlens, block_size, idx_full, scale, tokens)  # [T,H,d], [H,T]
    Dsum = np.einsum("thd,thd->ht", go, out)                                          # [H, T]
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    bt = block_table(cu_seqlens, block_size)
    s_of, _ = token_position(cu_seqlens, block_size, tokens)
    sel = np.asarray(idx_full)
    for b in range(bt.num_blocks):
        s, j = int(bt.seq[b]), int(bt.local[b])
        member = (sel == j).any(axis=2) & (s_of == s)[None, :]  # [H, T]
        if not member.any():
            continue
        st, en = int(bt.start[b]), int(bt.end[b])
        kpos = np.arange(st, en)
        for g in range(G):
            hh, tt = np.nonzero(member[g * r:(g + 1) * r])
            if hh.size == 0:
                continue
            hh = hh + g * r
            kb, vb = kf[st:en, g, :], vf[st:en, g, :]
            z = scale * (qf[tt, hh, :] @ kb.T)                      # [rows, len]
            z = np.where(kpos[None, :] <= tt[:, None], z, -np.inf)
            p = np.exp(z - lse[hh, tt][:, None])
            dov = go[tt, hh, :]                                     # [rows, d]
            dv[st:en, g, :] += p.T @ dov
            dp = dov @ vb.T
            ds = p * (dp - Dsum[hh, tt][:, None])
            np.add.at(dq, (tt, hh), scale * (ds @ kb))
            dk[st:en, g, :] += scale * (ds.T @ qf[tt, hh, :])
    return dq, dk, dv


# ---------------------------------------------------------------------------------------------
# Second, independent formulations (used only to pin the functions above)
# ---------------------------------------------------------------------------------------------

def dense_mask(cu_seqlens, block_size, idx_full: np.ndarray) -> np.ndarray:
    """Explicit [H, T, T] boolean mask of the routed attention pattern (mask-based formulation:
    MoBA repo radar, "How it works": moba_naive is attention-mask based)."""
    H, T, _ = idx_full.shape
    bt = block_table(cu_seqlens, block_size)
    s_of, i_of = token_position(cu_seqlens, block_size, np.arange(T))
    blk_global = np.full(T, -1, np.int64)
    for b in range(bt.num_blocks):
        blk_global[int(bt.start[b]):int(bt.end[b])] = b
    mask = np.zeros((H, T, T), bool)
    for h in range(H):
        for t in range(T):
            base = int(bt.blk_off[s_of[t]])
            for j in idx_full[h, t]:
                if j < 0:
                    continue
                b = base + int(j)
                u0, u1 = int(bt.start[b]), min(int(bt.end[b]), t + 1)
                mask[h, t, u0:u1] = True
    return mask


def attention_dense(q, k, v, mask: np.ndarray, scale) -> tuple:
    """Masked dense softmax attention over all T keys (small T only). O [T,H,d], LSE [H,T]."""
    qf, kf, vf = to_f64(q), to_f64(k), to_f64(v)
    T, H, d = qf.shape
    G = kf.shape[1]
    r = H // G
    out = np.zeros((T, H, d))
    lse = np.zeros((H, T))
    for h in range(H):
        g = h // r
        z = scale * (qf[:, h, :] @ kf[:, g, :].T)
        z = np.where(mask[h], z, -np.inf)
        mx = z.max(axis=1, keepdims=True)
        e = np.exp(z - mx)
        ssum = e.sum(axis=1, keepdims=True)
        out[:, h, :] = (e / ssum) @ vf[:, g, :]
        lse[h] = (mx + np.log(ssum))[:, 0]
    return out, lse


def causal_attention(q, k, v, cu_seqlens, scale) -> tuple:
    """Textbook causal softmax attention per sequence (the full-attention limit of MoBA)."""
    qf, kf, vf = to_f64(q), to_f64(k), to_f64(v)
    T, H, d = qf.shape
    G = kf.shape[1]
    r = H // G
    out = np.zeros((T, H, d))
    lse = np.zeros((H, T))
    cu = [int(x) for x in cu_seqlens]
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b == a:
            continue
        L = b - a
        tri = np.tril(np.ones((L, L), bool))
        for h in range(H):
            g = h // r
            z = scale * (qf[a:b, h] @ kf[a:b, g].T)
            z = np.where(tri, z, -np.inf)
            mx = z.max(axis=1, keepdims=True)
            e = np.exp(z - mx)
            ssum = e.sum(axis=1, keepdims=True)
            out[a:b, h] = (e / ssum) @ vf[a:b, g]
            lse[h, a:b] = (mx + np.log(ssum))[:, 0]
    return out, lse


def topk_by_enumeration(scores: np.ndarray, kk: int) -> List[int]:
    """Brute force: the kk-subset of past blocks with the largest total score (distinct scores)."""
    n = scores.shape[0]
    if kk >= n:
        return list(range(n))
    best, best_set = -math.inf, None
    for comb in itertools.combinations(range(n), kk):
        tot = float(scores[list(comb)].sum())
        if tot > best:
            best, best_set = tot, comb
    return sorted(best_set)
