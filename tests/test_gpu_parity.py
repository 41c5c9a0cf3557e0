"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on a B200.

Small cases are checked on every row; the full-size workloads on 4096 seeded, stratified query
rows x all heads (the launch configuration bench.py times). Edge cases: ragged last blocks,
sequences shorter than a block, empty sequences, topk = 1, topk >= #blocks (full attention),
block sizes that are not multiples of the 128-row tile, GQA, both head dims.
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


def _inputs(cu, hq, hkv, d, B, topk, keys="offset", seed=0):
    w = wl.custom(cu, hq, hkv, d, B, topk, keys)
    q, k, v, cu_t = wl.make_inputs(w, seed=seed, device="cuda")
    return w, q, k, v, cu_t


# ------------------------------------------------------------------------------ centroid, gate
@pytest.mark.parametrize("cu,hkv,d,B", [
    ([0, 1024], 1, 64, 128),
    ([0, 300, 300, 1000, 1100], 4, 128, 64),   # ragged tails, empty sequence, short sequence
    ([0, 8192], 8, 128, 4096),
    # at least 74 blocks: whole-row form
    ([0, 5000, 5000, 12000], 3, 64, 64),          # rows of 24 pieces: 10 rows per pass
    ([0, 10000], 32, 128, 128),                    # rows of 512 pieces: two per thread
    ([0, 9600], 64, 128, 128),                     # rows of 1024 pieces: four per thread
    ([0, 4800], 72, 128, 64),                      # wider rows: one kv head per cluster
    ([0, 65536], 16, 64, 128),                     # the 128-key-block shape
])
def test_centroids_match_oracle(moba, cu, hkv, d, B):
    w, q, k, v, cu_t = _inputs(cu, hkv, hkv, d, B, 2)
    c = moba.moba_centroids(k, cu_t, cu, B)
    torch.cuda.synchronize()
    c_ref = ref.centroids(k.cpu(), cu, B)
    np.testing.assert_allclose(c.cpu().numpy(), c_ref, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("cu,hq,hkv,d,B,topk,keys", [
    ([0, 1024], 1, 1, 64, 128, 3, "offset"),
    ([0, 4096], 16, 16, 64, 128, 16, "clusters"),
    ([0, 700, 700, 2000], 8, 2, 128, 64, 5, "offset"),
    ([0, 3000], 4, 4, 64, 64, 33, "clusters"),
    ([0, 2048], 2, 1, 128, 128, 1, "offset"),
    ([0, 6144], 2, 2, 64, 64, 40, "clusters"),          # topk above the buffered-selection limit
    ([0, 20000, 20000, 40000], 2, 1, 128, 64, 33, "clusters"),  # > 256 past blocks: chunked
    ([0, 40000], 2, 2, 64, 128, 16, "clusters"),        # 313 blocks: three-pass selection
    ([0, 33000, 33000, 70000], 2, 2, 64, 128, 32, "clusters"),  # 258 and 290 blocks, k - 1 = 31
    ([0, 90000], 2, 1, 64, 128, 8, "offset"),           # 704 blocks: centroids in two chunks
])
def test_gate_matches_oracle(moba, cu, hq, hkv, d, B, topk, keys):
    w, q, k, v, cu_t = _inputs(cu, hq, hkv, d, B, topk, keys)
    c = moba.moba_centroids(k, cu_t, cu, B)
    idx = moba.moba_gate_topk(q, c, cu_t, cu, B, topk)
    torch.cuda.synchronize()
    cents = ref.centroids(k.cpu(), cu, B)
    tokens = np.arange(cu[-1])
    pu.check_routing(q.cpu(), cents, cu, B, topk, tokens, idx.cpu().numpy())


@pytest.mark.parametrize("nblocks,topk", [(100, 12), (300, 16), (300, 32)])
def test_gate_equal_scores_take_lowest_blocks(moba, nblocks, topk):
    """All keys equal, so every past block scores the same: ties go to the lower block, so each
    row routes to blocks 0 .. topk - 2 and its own (the single-pass and three-pass selections,
    including the candidate-overflow fallback, all keep that order)."""
    B = 128
    T = nblocks * B
    cu = [0, T]
    q = torch.randn(T, 2, 64, device="cuda").to(torch.bfloat16)
    k = torch.full((T, 2, 64), 0.5, device="cuda", dtype=torch.bfloat16)
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    c = moba.moba_centroids(k, cu_t, cu, B)
    idx = moba.moba_gate_topk(q, c, cu_t, cu, B, topk).cpu()
    i = torch.arange(T) // B
    expect = torch.full((T, topk), -1, dtype=torch.int32)
    for x in range(topk):
        expect[:, x] = torch.where(x < torch.clamp(i, max=topk - 1), x, -1)
    n_sel = torch.clamp(i + 1, max=topk)
    expect[torch.arange(T), n_sel - 1] = i.to(torch.int32)
    assert torch.equal(idx[0], expect) and torch.equal(idx[1], expect)


# ----------------------------------------------------------------------- whole forward, small
SMALL = [
    # cu, hq, hkv, d, B, topk, keys
    ([0, 1024], 1, 1, 64, 128, 3, "offset"),                    # the tiny workload
    ([0, 1000], 2, 1, 64, 128, 3, "offset"),                    # ragged last block, GQA 2:1
    ([0, 333, 333, 900, 1500], 4, 2, 128, 128, 4, "clusters"),  # varlen, empty seq, d=128
    ([0, 2048], 4, 4, 64, 192, 3, "clusters"),                  # block not a multiple of 128
    ([0, 1536], 2, 2, 128, 64, 5, "offset"),                    # 64-key blocks
    ([0, 50], 1, 1, 64, 128, 3, "offset"),                      # shorter than one block
    ([0, 1], 2, 2, 64, 64, 2, "offset"),                        # a single token
    ([0, 1024], 2, 2, 64, 128, 1, "offset"),                    # topk = 1: block-diagonal
    ([0, 640], 2, 1, 128, 128, 64, "offset"),                   # topk >= #blocks: full causal
    ([0, 4096], 8, 8, 64, 128, 16, "clusters"),                 # routing stress, small
    ([0, 8192], 8, 2, 128, 4096, 3, "offset"),                  # two 4096-key blocks
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"T{c[0][-1]}_h{c[1]}x{c[2]}_d{c[3]}_B{c[4]}_k{c[5]}")
def test_forward_small_all_rows(moba, case):
    cu, hq, hkv, d, B, topk, keys = case
    w, q, k, v, cu_t = _inputs(cu, hq, hkv, d, B, topk, keys)
    res = pu.run_and_check(moba, q, k, v, cu_t, cu, B, topk, 1.0 / math.sqrt(d))
    ws = torch.empty(moba.moba_workspace_bytes(cu, hq, hkv, d, B, topk), dtype=torch.uint8,
                     device="cuda")
    moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, 1.0 / math.sqrt(d), workspace=ws)
    assert moba.moba_device_status(ws) == 0


@pytest.mark.parametrize("cu,hq,hkv,d,B,topk", [
    ([0, 40000, 40000, 75000], 2, 1, 128, 128, 8),   # 313 + 274 blocks at d = 128: two chunks
    ([0, 70000], 2, 2, 64, 128, 20),                 # 547 blocks, k - 1 = 19: three chunks
    ([0, 30000, 64000], 4, 2, 64, 128, 5),           # 235 + 266 blocks, GQA
    ([0, 80000], 2, 1, 64, 128, 16),                 # 625 blocks through a ring of four slots
    ([0, 5000, 75000], 2, 2, 64, 128, 16),           # a resident unit, then ring units
    ([0, 9000, 21000], 4, 2, 128, 128, 20),          # k - 1 = 19 at d = 128: 32-row ring slots
])
def test_forward_many_blocks_sampled_rows(moba, cu, hq, hkv, d, B, topk):
    """Sequences of more than 257 blocks take the long-sequence gate, whose centroids the forward
    pass splits into hi / lo once and keeps resident when they fit, else streams through a ring of
    slots; checked on sampled rows."""
    w, q, k, v, cu_t = _inputs(cu, hq, hkv, d, B, topk, "clusters")
    tokens = wl.sample_tokens(w, 1024, seed=3)
    pu.run_and_check(moba, q, k, v, cu_t, cu, B, topk, 1.0 / math.sqrt(d), tokens=tokens)


def test_full_attention_limit_matches_sdpa(moba):
    cu = [0, 777]
    w, q, k, v, cu_t = _inputs(cu, 4, 2, 128, 128, 8)
    o, lse = moba.moba_attn_fwd(q, k, v, cu_t, cu, 128, 8, 0.125)
    qs = q.permute(1, 0, 2).float()
    ks = k.permute(1, 0, 2).float().repeat_interleave(2, dim=0)
    vs = v.permute(1, 0, 2).float().repeat_interleave(2, dim=0)
    o_ref = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, is_causal=True,
                                                             scale=0.125).permute(1, 0, 2)
    err = (o.float() - o_ref).abs()
    assert (err <= pu.O_ATOL + pu.O_RTOL * o_ref.abs()).all(), float(err.max())


def test_given_routing_is_used(moba):
    cu = [0, 2048]
    B, topk = 128, 4
    w, q, k, v, cu_t = _inputs(cu, 2, 2, 64, B, topk)
    # a valid routing that differs from the gate's: current block plus the lowest past blocks
    T = cu[-1]
    idx = torch.full((2, T, topk), -1, dtype=torch.int32)
    for t in range(T):
        i = t // B
        sel = list(range(min(i, topk - 1))) + [i]
        idx[:, t, :len(sel)] = torch.tensor(sel, dtype=torch.int32)
    idx_d = idx.cuda()
    res = pu.run_and_check(moba, q, k, v, cu_t, cu, B, topk, 0.125, block_idx_in=idx_d)
    assert torch.equal(res["idx"].cpu(), idx)


def test_repeatable_bitwise(moba):
    cu = [0, 4096]
    w, q, k, v, cu_t = _inputs(cu, 8, 2, 128, 256, 6, "clusters")
    o1, l1 = moba.moba_attn_fwd(q, k, v, cu_t, cu, 256, 6)
    o2, l2 = moba.moba_attn_fwd(q, k, v, cu_t, cu, 256, 6)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_empty_input_is_a_noop(moba):
    q = torch.empty((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((0, 1, 64), dtype=torch.bfloat16, device="cuda")
    cu_t = torch.zeros(2, dtype=torch.int32, device="cuda")
    o, lse = moba.moba_attn_fwd(q, k, k, cu_t, [0, 0], 64, 2)
    assert o.shape == (0, 2, 64) and lse.shape == (2, 0)


# ------------------------------------------------------------------ full-size, sampled rows
FULL = ["tiny_1k", "routing_64k_b128", "llama8b_128k", "varlen_512k_b128", "llama8b_1m",
        "llama8b_10m_shard8"]


@pytest.mark.parametrize("name", FULL)
def test_workload_parity(moba, name):
    w = wl.WORKLOADS[name]
    q, k, v, cu_t = wl.make_inputs(w, seed=0, device="cuda")
    small = w.total_tokens <= 65536
    tokens = None if small else wl.sample_tokens(w, 4096, seed=0)
    res = pu.run_and_check(moba, q, k, v, cu_t, w.cu_seqlens, w.block_size, w.topk, w.scale,
                           tokens=tokens)
    rows = w.hq * (w.total_tokens if tokens is None else len(tokens))
    print(f"{name}: ties={res['ties']} of {rows} rows max|dO|={res['max_o_err']:.2e} "
          f"max|dLSE|={res['max_lse_err']:.2e}")
    # near ties are rare: a gate bug that happened to stay inside the band on many rows would
    # show up here
    assert res["ties"] <= pu.TIE_ROWS_MAX * rows + 2, (res["ties"], rows)


# --------------------------------------------------------------- gate scores that nearly cancel
@pytest.mark.parametrize("T,hkv,d,B,topk", [
    (8192, 2, 64, 128, 33),     # 64 blocks: streaming gate, boundary near the median score
    (40000, 2, 64, 128, 16),    # 313 blocks: three-pass selection
    (16384, 2, 128, 256, 24),   # d = 128
])
def test_gate_boundary_scores_near_zero(moba, T, hkv, d, B, topk):
    """Large per-block key offsets make every score a sum of large terms that nearly cancel
    (sum_i |q_i c_i| >> |q . c|), and with topk - 1 about half the past blocks the selection
    boundary sits near score zero: the regime where fp32 scoring error is largest relative to the
    score. Routing must still match the oracle outside the near-tie band."""
    g = torch.Generator(device="cuda").manual_seed(77)
    q = torch.randn((T, hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    nb = (T + B - 1) // B
    off = 2.0 * torch.randn((nb, hkv, d), generator=g, device="cuda")
    k = (torch.randn((T, hkv, d), generator=g, device="cuda") +
         off.repeat_interleave(B, dim=0)[:T]).to(torch.bfloat16)
    cu = [0, T]
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    c = moba.moba_centroids(k, cu_t, cu, B)
    idx = moba.moba_gate_topk(q, c, cu_t, cu, B, topk)
    torch.cuda.synchronize()
    cents = ref.centroids(k.cpu(), cu, B)
    tokens = np.arange(0, T, 7)
    ties = pu.check_routing(q.cpu(), cents, cu, B, topk, tokens,
                            idx.cpu()[:, torch.as_tensor(tokens)].numpy())
    rows = hkv * len(tokens)
    print(f"near-zero boundary T={T} d={d}: ties={ties} of {rows}")
    assert ties <= 0.01 * rows


# ------------------------------------------------------------------- routing contract checks
def test_routing_that_breaks_its_contract_is_reported(moba):
    """A caller routing with fewer blocks than min(topk, i + 1), or with a future block, makes the
    device status MOBA_ERR_DEVICE_CHECK (the merge would otherwise read slots nobody wrote); a
    valid routing leaves it MOBA_OK."""
    cu = [0, 2048]
    B, topk, hq = 128, 4, 2
    w, q, k, v, cu_t = _inputs(cu, hq, hq, 64, B, topk)
    idx = torch.empty((hq, cu[-1], topk), dtype=torch.int32, device="cuda")
    ws = torch.empty(moba.moba_workspace_bytes(cu, hq, hq, 64, B, topk), dtype=torch.uint8,
                     device="cuda")
    moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_out=idx, workspace=ws)
    assert moba.moba_device_status(ws) == 0
    moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_in=idx, workspace=ws)
    assert moba.moba_device_status(ws) == 0
    short = idx.clone()
    t = 5 * B + 3                       # block 5: n = 4 valid slots
    short[1, t] = torch.tensor([0, 2, 5, -1], dtype=torch.int32)
    moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_in=short, workspace=ws)
    assert moba.moba_device_status(ws) == -5
    future = idx.clone()
    future[0, 2 * B] = torch.tensor([0, 1, 3, -1], dtype=torch.int32)  # block 2 routed to 3
    moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_in=future, workspace=ws)
    assert moba.moba_device_status(ws) == -5
    first = idx.clone()
    first[0, 7] = torch.tensor([0, 0, -1, -1], dtype=torch.int32)      # block 0, repeated
    moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_in=first, workspace=ws)
    assert moba.moba_device_status(ws) == -5
    # the next valid call clears the word
    moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_in=idx, workspace=ws)
    assert moba.moba_device_status(ws) == 0


# ----------------------------------------------------------------------- bounded-wait aborts
@pytest.mark.parametrize("d", [64, 128])
def test_wait_that_runs_out_reports_timeout_and_the_context_survives(moba, d):
    """The attention kernel's MMA issuer waits first on a barrier that nothing arrives on (a
    diagnostic switch) under a 100 us pipeline-wait limit: the wait runs out, every CTA raises its
    abort flag, the other roles give up their own waits, drain the copies and matrix products they
    have in flight (under the separate fixed drain limit), free tensor memory and return, and the
    status word reads MOBA_ERR_TIMEOUT. The same workspace then serves a normal call whose output
    matches the oracle."""
    cu = [0, 1536]
    B, topk, hq, hkv = 128, 4, 4, 2
    w, q, k, v, cu_t = _inputs(cu, hq, hkv, d, B, topk, "clusters")
    scale = 1.0 / math.sqrt(d)
    idx = torch.empty((hq, cu[-1], topk), dtype=torch.int32, device="cuda")
    ws = torch.empty(moba.moba_workspace_bytes(cu, hq, hkv, d, B, topk), dtype=torch.uint8,
                     device="cuda")
    moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, scale, block_idx_out=idx, workspace=ws)
    assert moba.moba_device_status(ws) == 0
    prev = moba.set_wait_limit_ns(100_000)
    was = moba.set_diag_stall(True)
    try:
        moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, scale, block_idx_in=idx, workspace=ws)
        status = moba.moba_device_status(ws)
    finally:
        moba.set_diag_stall(False)
        moba.set_wait_limit_ns(0)
    assert prev == 2_000_000_000 and was is False
    assert status == -6, status  # MOBA_ERR_TIMEOUT
    o, lse = moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, scale, block_idx_in=idx,
                                workspace=ws)
    assert moba.moba_device_status(ws) == 0
    tokens = np.arange(cu[-1])
    o_ref, lse_ref = ref.attention(q.cpu(), k.cpu(), v.cpu(), cu, B, idx.cpu().numpy(), scale,
                                   tokens)
    pu.check_outputs(o.cpu().float().numpy(), lse.cpu().numpy(), o_ref, lse_ref)



# ------------------------------------------------------------------------- head-parallel split
def test_head_shards_reproduce_the_whole_problem(moba):
    """Running moba_attn_fwd on each rank's share of the heads (the head-parallel split, ranks
    emulated one after another on this GPU; no rank waits on another) and concatenating the heads
    gives the whole problem's result: the same routing and O / LSE within the parity tolerance of
    the single run."""
    from block_sparse_long_moba_b200 import shard

    cu = [0, 5000, 5000, 12000]
    hq, hkv, d, B, topk = 8, 4, 128, 512, 4
    w, q, k, v, cu_t = _inputs(cu, hq, hkv, d, B, topk, "clusters")
    idx = torch.empty((hq, cu[-1], topk), dtype=torch.int32, device="cuda")
    o, lse = moba.moba_attn_fwd(q, k, v, cu_t, cu, B, topk, block_idx_out=idx)
    for world in (2, 4):
        parts_o, parts_l, parts_i = [], [], []
        for rank in range(world):
            ql, kl, vl = shard.take_heads(q, k, v, world, rank)
            il = torch.empty((ql.shape[1], cu[-1], topk), dtype=torch.int32, device="cuda")
            ol, ll = shard.moba_attn_fwd_heads(ql, kl, vl, cu_t, cu, B, topk, block_idx_out=il)
            parts_o.append(ol)
            parts_l.append(ll)
            parts_i.append(il)
        torch.cuda.synchronize()
        o2, l2, i2 = torch.cat(parts_o, 1), torch.cat(parts_l, 0), torch.cat(parts_i, 0)
        mism = (i2 != idx).any(dim=2)
        assert mism.float().mean().item() <= pu.TIE_ROWS_MAX, mism.sum().item()
        ok = ~mism.T[:, :, None].expand_as(o)
        err = (o2.float() - o.float()).abs()
        assert (err[ok] <= pu.O_ATOL + pu.O_RTOL * o.float().abs()[ok]).all()
        assert ((l2 - lse).abs()[~mism] <= pu.LSE_ATOL).all()
