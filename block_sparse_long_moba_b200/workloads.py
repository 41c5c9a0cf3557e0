"""Seeded synthetic inputs for the MoBA prefill forward pass.

This module only draws random tensors; it holds none of the method's arithmetic, so both the
CUDA path and the CPU oracle can consume what it produces.

Workload shapes follow the attention-layer shape of a Llama-3.1-8B model continually pre-trained
to 1M context (MoBA paper summary, "Key results": 1M-token prefill) and the small-block regime
that FlashMoBA argues for (FlashMoBA story: block size vs routing signal-to-noise). There is no
dataset or checkpoint: every tensor is drawn from a seeded generator.

Recipes (values drawn in fp32, then rounded to bf16):
  * Q, V ~ N(0, 1).
  * "offset" keys:   K[t, g, :] = N(0, 1) + o[b(t), g, :],  o ~ N(0, 0.5^2) per (block, kv head).
  * "clusters" keys: K[t, g, :] = N(0, 1) + mu[g, c(b(t), g), :], with 64 cluster means per kv head,
    mu ~ N(0, 1)^d, and each (block, kv head) assigned a cluster uniformly at random.
  Seeds: Q = 10*seed+1, K noise = 10*seed+2, V = 10*seed+3, offsets / clusters = 10*seed+4.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    cu_seqlens: List[int]
    hq: int
    hkv: int
    d: int
    block_size: int
    topk: int
    keys: str  # "offset" | "clusters"
    n_clusters: int = 64

    @property
    def total_tokens(self) -> int:
        return self.cu_seqlens[-1]

    @property
    def nseq(self) -> int:
        return len(self.cu_seqlens) - 1

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def seq_blocks(self) -> List[int]:
        b = self.block_size
        return [(self.cu_seqlens[s + 1] - self.cu_seqlens[s] + b - 1) // b for s in range(self.nseq)]

    @property
    def num_blocks(self) -> int:
        return sum(self.seq_blocks())


# The five workloads: a tiny single-head case, the Llama-3.1-8B attention shape at 128K and 1M
# tokens with 4096-token blocks, a 64K small-block routing stress case, and a packed varlen batch.
WORKLOADS = {
    "tiny_1k": Workload("tiny_1k", [0, 1024], 1, 1, 64, 128, 3, "offset"),
    "llama8b_128k": Workload("llama8b_128k", [0, 131072], 32, 8, 128, 4096, 12, "offset"),
    "llama8b_1m": Workload("llama8b_1m", [0, 1048576], 32, 8, 128, 4096, 12, "offset"),
    "routing_64k_b128": Workload("routing_64k_b128", [0, 65536], 16, 16, 64, 128, 16, "clusters"),
    "varlen_512k_b128": Workload("varlen_512k_b128", [0, 65536, 196608, 294912, 524288],
                                 16, 16, 64, 128, 32, "clusters"),
    # 10M tokens of the Llama-3.1-8B shape, one rank's share of an 8-way head split (one kv head
    # and its four query heads; MoBA paper summary, "Key results": attention time at 10M tokens)
    "llama8b_10m_shard8": Workload("llama8b_10m_shard8", [0, 10485760], 4, 1, 128, 4096, 12,
                                   "offset"),
    # small cases of the same kernels for profiler captures (a few GB on the device)
    "profile_32k_b4096": Workload("profile_32k_b4096", [0, 32768], 32, 8, 128, 4096, 4, "offset"),
    "profile_32k_b128": Workload("profile_32k_b128", [0, 32768], 16, 16, 64, 128, 16, "clusters"),
    # the gate's 256-block regime of the 1M shape (n up to 255 past blocks, k - 1 = 11) at 1 GB of Q
    "profile_128k_b512": Workload("profile_128k_b512", [0, 131072], 32, 8, 128, 512, 12, "offset"),
}
WORKLOAD_ORDER = ["tiny_1k", "llama8b_128k", "llama8b_1m", "routing_64k_b128", "varlen_512k_b128"]


def custom(cu_seqlens, hq, hkv, d, block_size, topk, keys="offset", name="custom") -> Workload:
    return Workload(name, list(int(x) for x in cu_seqlens), hq, hkv, d, block_size, topk, keys)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def block_of_token(w: Workload, device) -> torch.Tensor:
    """Global block id of every token (blocks never cross sequence boundaries)."""
    ids = []
    base = 0
    for s in range(w.nseq):
        n = w.cu_seqlens[s + 1] - w.cu_seqlens[s]
        ids.append(torch.arange(n, device=device, dtype=torch.int64) // w.block_size + base)
        base += (n + w.block_size - 1) // w.block_size
    if not ids:
        return torch.zeros(0, dtype=torch.int64, device=device)
    return torch.cat(ids)


def make_inputs(w: Workload, seed: int = 0, device="cuda"):
    """Return (q, k, v, cu_seqlens) with q [T,Hq,d], k/v [T,Hkv,d] bf16 and int32 cu_seqlens."""
    T, d = w.total_tokens, w.d
    dev = torch.device(device)
    q = torch.randn((T, w.hq, d), generator=_gen(dev, 10 * seed + 1), device=dev,
                    dtype=torch.float32).to(torch.bfloat16)
    k32 = torch.randn((T, w.hkv, d), generator=_gen(dev, 10 * seed + 2), device=dev,
                      dtype=torch.float32)
    bot = block_of_token(w, dev)
    g4 = _gen(dev, 10 * seed + 4)
    if w.keys == "offset":
        off = 0.5 * torch.randn((w.num_blocks, w.hkv, d), generator=g4, device=dev,
                                dtype=torch.float32)
        k32 += off[bot]
    elif w.keys == "clusters":
        mu = torch.randn((w.hkv, w.n_clusters, d), generator=g4, device=dev, dtype=torch.float32)
        assign = torch.randint(0, w.n_clusters, (w.num_blocks, w.hkv), generator=g4, device=dev)
        heads = torch.arange(w.hkv, device=dev)
        # mean vector for every (block, kv head): mu[g, assign[b, g]]
        blk_mean = mu[heads[None, :], assign]  # [NB, G, d]
        k32 += blk_mean[bot]
    else:
        raise ValueError(f"unknown key recipe {w.keys!r}")
    k = k32.to(torch.bfloat16)
    del k32
    v = torch.randn((T, w.hkv, d), generator=_gen(dev, 10 * seed + 3), device=dev,
                    dtype=torch.float32).to(torch.bfloat16)
    cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device=dev)
    return q, k, v, cu


def sample_tokens(w: Workload, n: int, seed: int = 0) -> List[int]:
    """Seeded, stratified sample of query positions for full-size checks.

    Always includes t=0, the first and last token of several blocks and the last token of every
    sequence; the rest are uniform draws. Returned sorted and unique.
    """
    T = w.total_tokens
    if n >= T:
        return list(range(T))
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 + seed)
    picks = {0}
    for s in range(w.nseq):
        a, b = w.cu_seqlens[s], w.cu_seqlens[s + 1]
        if b > a:
            picks.add(b - 1)
            picks.add(a)
            nb = (b - a + w.block_size - 1) // w.block_size
            for j in sorted({0, 1, nb // 2, nb - 1}):
                st = a + j * w.block_size
                if st < b:
                    picks.add(st)
                    picks.add(min(b, st + w.block_size) - 1)
    extra = torch.randint(0, T, (n * 2,), generator=g).tolist()
    for t in extra:
        if len(picks) >= n:
            break
        picks.add(int(t))
    return sorted(picks)
