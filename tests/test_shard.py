"""Head-parallel sharding (CPU): the kv-group split, and 2 gloo ranks that each run the fp64
oracle on their own heads and all-gather the heads reproduce the oracle on the whole problem
(the split is exact: no head reads another rank's data)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from block_sparse_long_moba_b200 import shard
from block_sparse_long_moba_b200 import workloads as wl
from oracle import moba_ref as ref


@pytest.mark.parametrize("world,hkv", [(1, 8), (2, 8), (3, 8), (8, 8), (4, 6)])
def test_kv_groups_cover_every_head_once(world, hkv):
    seen = []
    for r in range(world):
        g0, g1 = shard.kv_groups(world, r, hkv)
        assert g1 > g0
        seen += list(range(g0, g1))
    assert seen == list(range(hkv))


def test_head_range_keeps_gqa_groups_together():
    assert shard.head_range(2, 0, 32, 8) == (0, 16, 0, 4)
    assert shard.head_range(2, 1, 32, 8) == (16, 32, 4, 8)
    assert shard.head_range(3, 2, 12, 6) == (8, 12, 4, 6)
    with pytest.raises(ValueError):
        shard.kv_groups(4, 0, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w = wl.custom([0, 300, 300, 700], 8, 4, 16, 64, 3, "clusters")
    q, k, v, _ = wl.make_inputs(w, seed=1, device="cpu")
    ql, kl, vl = shard.take_heads(q, k, v, world, rank)
    _, o_l, lse_l = ref.forward(ql, kl, vl, w.cu_seqlens, 64, 3, 0.25)
    o_full, lse_full = shard.gather_heads(torch.from_numpy(o_l), torch.from_numpy(lse_l), world,
                                          8, 4)
    out[rank] = (o_full.numpy(), lse_full.numpy())
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_parallel_oracle_equals_whole_problem(world):
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    w = wl.custom([0, 300, 300, 700], 8, 4, 16, 64, 3, "clusters")
    q, k, v, _ = wl.make_inputs(w, seed=1, device="cpu")
    _, o, lse = ref.forward(q, k, v, w.cu_seqlens, 64, 3, 0.25)
    for r in range(world):
        np.testing.assert_array_equal(out[r][0], o)
        np.testing.assert_array_equal(out[r][1], lse)
