"""Host-side logic of bench.py (no GPU): FLOP accounting against the oracle's routing, and the
multi-rank timing reduction with 2 gloo ranks on the CPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
from block_sparse_long_moba_b200 import workloads as wl
from oracle import moba_ref as ref


@pytest.mark.parametrize("cu,B,topk", [([0, 1000], 128, 3), ([0, 300, 300, 1111], 64, 5),
                                       ([0, 4096], 256, 64)])
def test_attended_pairs_match_oracle_routing(cu, B, topk):
    w = wl.custom(cu, 2, 1, 16, B, topk)
    q, k, v, _ = wl.make_inputs(w, device="cpu")
    rt = ref.select_blocks(q, ref.centroids(k, cu, B), cu, B, topk)
    bt = ref.block_table(cu, B)
    s_of, i_of = ref.token_position(cu, B, np.arange(cu[-1]))
    pairs = 0
    for h in range(2):
        for t in range(cu[-1]):
            base = int(bt.blk_off[s_of[t]])
            for j in rt.idx[h, t]:
                if j >= 0:
                    b = base + int(j)
                    pairs += min(int(bt.end[b]), t + 1) - int(bt.start[b])
    assert bench.attended_pairs(w) == pairs


def test_workload_flops_of_the_headline_configs():
    assert abs(bench.useful_flops(wl.WORKLOADS["llama8b_128k"]) / 1e12 - 83.01) < 0.01
    assert abs(bench.useful_flops(wl.WORKLOADS["llama8b_1m"]) / 1e12 - 791.1) < 0.1


@pytest.mark.parametrize("cu,hq,hkv,d,B,topk", [
    ([0, 1000], 2, 1, 64, 128, 3),
    ([0, 300, 300, 1111], 4, 2, 128, 64, 5),
    ([0, 2500], 2, 2, 64, 256, 4),
    ([0, 9000], 2, 1, 128, 4096, 2),
])
def test_executed_flops_count_the_kernel_items(cu, hq, hkv, d, B, topk):
    """Executed tile FLOPs by brute force: build every (kv head, past block) list from the
    oracle's routing, cut it into 256-row items, add the diagonal items, and count 128 x 128
    sub-tile pairs the way the kernels issue them (both halves at d = 128; at d = 64 one half for
    items of at most 128 rows)."""
    w = wl.custom(cu, hq, hkv, d, B, topk)
    q, k, v, _ = wl.make_inputs(w, device="cpu")
    rt = ref.select_blocks(q, ref.centroids(k, cu, B), cu, B, topk)
    bt = ref.block_table(cu, B)
    s_of, i_of = ref.token_position(cu, B, np.arange(cu[-1]))
    r = hq // hkv
    lists = {}
    for h in range(hq):
        for t in range(cu[-1]):
            for j in rt.idx[h, t]:
                if 0 <= j < i_of[t]:
                    key = (h // r, int(bt.blk_off[s_of[t]]) + int(j))
                    lists[key] = lists.get(key, 0) + 1

    def rows_run(n):
        return 256 if (d == 128 or n > 128) else 128

    tiles = 0
    for (g, b), c in lists.items():
        nsub = -(-(int(bt.end[b]) - int(bt.start[b])) // 128)
        for x in range(0, c, 256):
            tiles += rows_run(min(256, c - x)) * nsub
    for b in range(bt.num_blocks):
        n = int(bt.end[b]) - int(bt.start[b])
        for q0 in range(0, n, 256):
            rows = min(256, n - q0)
            tiles += hq * rows_run(rows) * -(-(q0 + rows) // 128)
    got = bench.executed_flops(w, torch.as_tensor(rt.idx))
    assert got == 4.0 * d * 128 * tiles
    assert got >= bench.useful_flops(w)


def test_job_throughput_is_weak_scaling():
    assert bench.job_throughput(1, 131072, 100.0) == pytest.approx(1.31072e6)
    assert bench.job_throughput(4, 131072, 100.0) == pytest.approx(4 * 1.31072e6)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    mine = 10.0 + 5.0 * rank
    got = bench.max_over_ranks(mine, world, device="cpu")
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == 15.0 and out[1] == 15.0


def test_attention_traffic_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "block_sparse_long_moba_b200" / "csrc"
    csrc.mkdir(parents=True)
    def code(name):
        return "int v_%s;" % name.replace(".", "_")

    for name in bench.ATTN_SOURCES:
        (csrc / name).write_text(code(name) + "  // " + name)
    (tmp_path / "profiles").mkdir()
    rec = tmp_path / "profiles" / "attention_w_traffic.json"
    assert bench.attention_traffic("w") is None  # no record
    import json
    rec.write_text(json.dumps({"bytes_per_launch": 123.0,
                               "kernel_sources_sha256": bench.attention_source_hash()}))
    assert bench.attention_traffic("w") == 123.0
    (csrc / "attn.cu").write_text(code("attn.cu") + "  /* a comment edit */ // keeps the record")
    assert bench.attention_traffic("w") == 123.0
    (csrc / "attn.cu").write_text("int y;  // changed code")  # the kernel changed
    assert bench.attention_traffic("w") is None


def test_kernel_bytes_count_densify_at_d64_only():
    import bench
    from block_sparse_long_moba_b200 import workloads as wl
    small = bench.kernel_bytes(wl.WORKLOADS["routing_64k_b128"])
    big = bench.kernel_bytes(wl.WORKLOADS["llama8b_128k"])
    assert "densify" in small and "densify" not in big
    # every routed entry: its 4-byte entry read, its 128-byte query row read and written
    w = wl.WORKLOADS["routing_64k_b128"]
    entries = 0  # routed (t, h, slot): every selected past block of every row
    for s in range(w.nseq):
        L = w.cu_seqlens[s + 1] - w.cu_seqlens[s]
        for i in range((L + w.block_size - 1) // w.block_size):
            entries += min(w.block_size, L - i * w.block_size) * (min(w.topk, i + 1) - 1)
    entries *= w.hq
    assert entries > 0 and small["densify"] == entries * (4 + 4 * w.d)
