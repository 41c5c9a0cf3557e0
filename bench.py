#!/usr/bin/env python
"""Throughput of the MoBA causal prefill forward pass on B200, one process per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one full forward pass (centroids, gate, routing inversion, attention, merge) over one
synthetic batch that is already resident in HBM. With N > 1 (launched by torchrun) every rank
runs its own independent problem of the same shape (weak scaling: no data-path collective; the
only collectives are the barrier and the max-over-ranks of the timed region).

Prints ONE JSON line on rank 0. `--impl reference` times the fp64 CPU oracle on a bounded sample
of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_long_moba_b200 import workloads as wl  # noqa: E402

METRIC = "MoBA prefill query-tokens/s (TFLOP/s, % of bf16 tensor peak)"
UNIT = "query-tokens/s"
L2_BYTES = 126 * 2 ** 20


# ----------------------------------------------------------------------------- problem sizes
def attended_pairs(w: wl.Workload) -> int:
    """Sum over (t, h) of the number of keys attended: (n_sel - 1) full past blocks plus the
    causal prefix of the current block, n_sel = min(topk, i + 1). Independent of which past
    blocks are chosen (past blocks are never a sequence's short last block)."""
    tot = 0
    B, k = w.block_size, w.topk
    for s in range(w.nseq):
        L = w.cu_seqlens[s + 1] - w.cu_seqlens[s]
        for i in range((L + B - 1) // B):
            n = min(B, L - i * B)
            nsel = min(k, i + 1)
            tot += n * (nsel - 1) * B + n * (n + 1) // 2
    return tot * w.hq


def useful_flops(w: wl.Workload) -> float:
    return 4.0 * w.d * attended_pairs(w)


def gate_flops(w: wl.Workload) -> float:
    """2 d per scored (t, h, past block); rows with topk-1 >= i score nothing."""
    tot = 0
    B, k = w.block_size, w.topk
    for s in range(w.nseq):
        L = w.cu_seqlens[s + 1] - w.cu_seqlens[s]
        for i in range((L + B - 1) // B):
            if k - 1 < i and k > 1:
                tot += min(B, L - i * B) * i
    return 2.0 * w.d * w.hq * tot


def kernel_bytes(w: wl.Workload) -> dict:
    """Algorithmic HBM bytes of the HBM-bound kernels over one whole step (all query chunks)."""
    T, H, G, d, k = w.total_tokens, w.hq, w.hkv, w.d, w.topk
    NB = w.num_blocks
    routed = 0
    B = w.block_size
    for s in range(w.nseq):
        L = w.cu_seqlens[s + 1] - w.cu_seqlens[s]
        for i in range((L + B - 1) // B):
            routed += min(B, L - i * B) * (min(k, i + 1) - 1)
    routed *= H
    rows = T * H  # (t, h)
    slots = rows * 0
    for s in range(w.nseq):
        L = w.cu_seqlens[s + 1] - w.cu_seqlens[s]
        for i in range((L + B - 1) // B):
            slots += min(B, L - i * B) * min(k, i + 1)
    slots *= H
    return {
        "centroid": T * G * d * 2 + NB * G * d * 4,
        "gate": T * H * d * 2 + T * H * k * 4,
        "route_count": T * H * k * 4,
        "route_scatter": T * H * k * 4 + routed * 4,
        "merge": slots * (2 * d + 4) + T * H * (2 * d + 4),
        # d = 64: each routed entry is read (4 B), its query row read and written (2 d B each)
        **({"densify": routed * (4 + 4 * d)} if d == 64 else {}),
    }


def executed_flops(w: wl.Workload, idx: torch.Tensor) -> float:
    """Tile FLOPs the attention kernel issues for one step, from the routing it was given.

    Work items are 256 query rows (two 128-row halves) against every 128-key sub-tile of one
    block: a routed item covers up to 256 rows of one (kv head, past block) list, a diagonal item
    up to 256 consecutive tokens of one head inside its own block against the keys up to its last
    query. At d = 128 both halves always run (the value product is issued for 256 rows at once);
    at d = 64 an item of at most 128 rows runs on one half. Each 128 x 128 sub-tile pair costs
    4 d 128^2 FLOPs (QK^T and PV). Routed-list lengths are counted from idx on the device."""
    T, H, G, d, B, k = w.total_tokens, w.hq, w.hkv, w.d, w.block_size, w.topk
    dev = idx.device
    r = H // G
    bot = wl.block_of_token(w, dev)                         # global block of every token
    blk_off = [0]
    for nb in w.seq_blocks():
        blk_off.append(blk_off[-1] + nb)
    seq_of_blk = torch.repeat_interleave(torch.arange(w.nseq, device=dev),
                                         torch.tensor(w.seq_blocks(), device=dev))
    base = torch.tensor(blk_off[:-1], device=dev, dtype=torch.int64)[seq_of_blk[bot]]
    i_tok = (bot - base)[:, None]                           # local block of every token
    NB = w.num_blocks
    counts = torch.zeros(G * NB, dtype=torch.int64, device=dev)
    for h in range(H):
        j = idx[h].to(torch.int64)
        ok = (j >= 0) & (j < i_tok)
        b = (base[:, None] + j)[ok]
        counts[(h // r) * NB:(h // r + 1) * NB] += torch.bincount(b, minlength=NB)
    blk_len = []
    for s in range(w.nseq):
        L = w.cu_seqlens[s + 1] - w.cu_seqlens[s]
        blk_len += [min(B, L - x * B) for x in range((L + B - 1) // B)]
    nsub = torch.tensor([(n + 127) // 128 for n in blk_len], device=dev, dtype=torch.int64)
    nsub_g = nsub.repeat(G)
    full = counts // 256
    tail = counts % 256
    if d == 128:
        rows_tail = torch.where(tail > 0, 256, 0)
    else:
        rows_tail = torch.where(tail > 128, 256, torch.where(tail > 0, 128, 0))
    routed_rows_x_sub = int(((full * 256 + rows_tail) * nsub_g).sum().item())
    diag = 0
    for n in blk_len:
        for q0 in range(0, n, 256):
            rows = min(256, n - q0)
            exec_rows = 256 if (d == 128 or rows > 128) else 128
            diag += exec_rows * ((q0 + rows + 127) // 128)
    diag *= H
    return 4.0 * d * 128 * (routed_rows_x_sub + diag)


def job_throughput(world: int, tokens_per_rank: int, ms_step_max: float) -> float:
    """Whole-job query tokens/s: every rank processes its own problem (weak scaling), timed as
    the max over ranks."""
    return world * tokens_per_rank / (ms_step_max / 1e3)


# ------------------------------------------------------------------------------------ peaks
def read_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ----------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            self.path = f"/tmp/moba_clocks_{os.getpid()}.csv"
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# -------------------------------------------------------------------------------- CPU oracle
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_target_seconds(args) -> float:
    """Seconds of oracle work per sample, the same for the reference arm's steps and the
    CPU-baseline leg (so both time the same sample size): at most --cpu-seconds, and small
    enough that --steps + --warmup samples take about four minutes."""
    return max(1.0, min(args.cpu_seconds, 240.0 / max(args.steps + args.warmup, 1)))


class OracleSampler:
    """Times the fp64 oracle (as it stands) on bounded samples of one workload's query tokens.

    One sample = one oracle call (gate + attention) on n seeded random query tokens, all heads,
    plus the centroids of the whole K, computed once and charged pro rata (n / T of its time).
    An oracle call has a fixed cost (it walks every block of K and V once) besides its per-token
    cost, so its rate depends on n: the sample size is fixed once, from an untimed calibration
    call on 64 tokens, so that one sample takes about `target_s`, and every timed sample (of the
    reference arm and of the CPU-baseline leg alike) uses that same n."""

    def __init__(self, w: wl.Workload, q, k, v, target_s: float, seed: int = 0):
        from oracle import moba_ref as ref

        self.ref, self.w = ref, w
        self.qc, self.kc, self.vc = q.cpu(), k.cpu(), v.cpu()
        t0 = time.perf_counter()
        self.cents = ref.centroids(self.kc, w.cu_seqlens, w.block_size)
        self.t_cent = time.perf_counter() - t0
        self.rng = np.random.default_rng(seed)
        T = w.total_tokens
        n0 = min(64, T)
        t_cal = self._call(n0)
        self.n = int(min(T, 4096, max(n0, round(n0 * target_s / max(t_cal, 1e-6)))))

    def _call(self, n: int) -> float:
        T = self.w.total_tokens
        toks = np.sort(self.rng.choice(T, size=min(n, T), replace=False))
        t1 = time.perf_counter()
        rt = self.ref.select_blocks(self.qc, self.cents, self.w.cu_seqlens, self.w.block_size,
                                    self.w.topk, toks)
        self.ref.attention(self.qc, self.kc, self.vc, self.w.cu_seqlens, self.w.block_size,
                           rt.idx, self.w.scale, toks)
        return time.perf_counter() - t1

    def sample(self) -> dict:
        """One timed sample; returns its rate in query-tokens/s and what it covered."""
        t_rows = self._call(self.n)
        T = self.w.total_tokens
        charged = t_rows + self.t_cent * self.n / T
        w = self.w
        return {"value": self.n / charged, "unit": UNIT, "cores": blas_threads(),
                "kind": "oracle", "seconds": charged,
                "sample": f"{self.n} random query tokens x all {w.hq} heads of {w.name} per "
                          f"sample (gate + attention {t_rows:.1f} s) + centroids of all "
                          f"{w.num_blocks} blocks ({self.t_cent:.1f} s, charged pro rata "
                          f"{self.n}/{T})"}


# ---------------------------------------------------------------------------------- traffic
ATTN_SOURCES = ("attn.cu", "sm100.cuh", "common.cuh")


def _code_only(text: str) -> str:
    """C++ source without its comments and with whitespace collapsed: what the compiler sees, so
    that editing a comment does not orphan a profile taken on the same code."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def attention_source_hash() -> str:
    """sha256 over the code (comments removed) of the attention kernel's sources, fixed order."""
    import hashlib

    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "block_sparse_long_moba_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()


def attention_traffic(workload: str):
    """DRAM bytes (read + write) of one attention launch on `workload`, from the committed ncu
    summary profiles/attention_<workload>_traffic.json, or None when there is none or it was taken
    on other kernel sources than the ones being timed."""
    path = os.path.join(ROOT, "profiles", f"attention_{workload}_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("kernel_sources_sha256") != attention_source_hash():
            return None
        return float(rec["bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------------------- distributed
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world, device="cuda") -> float:
    """Max of a per-rank timing over all ranks (the job is as slow as its slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def physical_gpu_index(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local < len(ids) and ids[local].isdigit():
            return int(ids[local])
    return local


# ----------------------------------------------------------------------------------- our arm
# Workloads timed beside the headline one (one GPU only): the 1M-token shape the metric is also
# quoted on and the two small-block shapes, each on its own buffers (freed before the next).
# The 10M-token record is one rank's share of an 8-way head-parallel split (one kv head and its
# four query heads of the Llama-3.1-8B shape over the whole sequence): the 8-GPU job runs eight
# such independent shards.
EXTRA_WORKLOADS = (("llama8b_1m", 3), ("routing_64k_b128", 10), ("varlen_512k_b128", 10),
                   ("llama8b_10m_shard8", 2))


def measure(w: wl.Workload, steps: int, warmup: int, world: int, rank: int, local: int,
            seed: int, e2e: bool, clocks_on: bool) -> dict:
    """Times `steps` forward passes of `w` (inputs resident in HBM), bracketed by a barrier and a
    device synchronisation on both sides, max over ranks; optionally the end-to-end variant with
    pinned host buffers copied in and out every step. Returns the raw figures of this rank."""
    from block_sparse_long_moba_b200 import moba

    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v, cu = wl.make_inputs(w, seed=seed, device=dev)
    T, H, d = w.total_tokens, w.hq, w.d
    o = torch.empty_like(q)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    idx = torch.empty((H, T, w.topk), dtype=torch.int32, device=dev)
    ws = torch.empty(moba.moba_workspace_bytes(w.cu_seqlens, H, w.hkv, d, w.block_size, w.topk),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        moba.moba_attn_fwd(q, k, v, cu, w.cu_seqlens, w.block_size, w.topk, w.scale,
                           block_idx_out=idx, o=o, lse=lse, workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    status = moba.moba_device_status(ws)
    if status != 0:
        raise RuntimeError(f"{w.name}: device status {status} after warm-up")

    # ---- device-timed region: inputs resident in HBM
    moba.timing_reset()
    moba.timing_enable(True)
    clocks = ClockSampler(physical_gpu_index(local)) if (rank == 0 and clocks_on) else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    n0 = moba.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = moba.launch_count() - n0
    clk = clocks.stop() if clocks else None
    moba.timing_enable(False)
    per_kernel = moba.timing_read()
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world)
    status = moba.moba_device_status(ws)
    if status != 0:
        raise RuntimeError(f"{w.name}: device status {status} after the timed region")
    out = {"ms": ms, "ms_local": ms_local, "per_kernel": per_kernel, "launches": launches,
           "clocks": clk, "executed_flops": executed_flops(w, idx)}
    if not e2e:
        return out

    # ---- end to end through the public API: pinned host inputs -> device -> host outputs.
    # Every step copies its own inputs in and its results out; the steps are pipelined over two
    # device buffer sets and three streams, as a server streaming requests would run them: the
    # copy-in of step n + 1 and the copy-out of step n - 1 overlap the compute of step n. Events
    # keep a buffer set from being refilled before the compute that reads it, or recomputed
    # before the copy-out that reads it, has finished.
    qh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True).copy_(q)
    kh = torch.empty(k.shape, dtype=k.dtype, pin_memory=True).copy_(k)
    vh = torch.empty(v.shape, dtype=v.dtype, pin_memory=True).copy_(v)
    cuh = torch.tensor(w.cu_seqlens, dtype=torch.int32).pin_memory()
    oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh, cuh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
    sets = [(q, k, v, cu, o, lse),
            (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(cu),
             torch.empty_like(o), torch.empty_like(lse))]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    computed = [torch.cuda.Event(), torch.cuda.Event()]  # compute of the set's last step done
    copied_out = [torch.cuda.Event(), torch.cuda.Event()]  # copy-out of the set's last step done
    for e in computed + copied_out:
        e.record(stream)
    n_e2e = [0]

    def e2e_step():
        b = n_e2e[0] % 2
        n_e2e[0] += 1
        qb, kb, vb, cub, ob, lb = sets[b]
        s_in.wait_event(computed[b])
        with torch.cuda.stream(s_in):
            qb.copy_(qh, non_blocking=True)
            kb.copy_(kh, non_blocking=True)
            vb.copy_(vh, non_blocking=True)
            cub.copy_(cuh, non_blocking=True)
        stream.wait_stream(s_in)
        stream.wait_event(copied_out[b])
        moba.moba_attn_fwd(qb, kb, vb, cub, w.cu_seqlens, w.block_size, w.topk, w.scale, o=ob,
                           lse=lb, workspace=ws, stream=stream)
        computed[b].record(stream)
        s_out.wait_event(computed[b])
        with torch.cuda.stream(s_out):
            oh.copy_(ob, non_blocking=True)
            lh.copy_(lb, non_blocking=True)
        copied_out[b].record(s_out)

    e2e_steps = max(2, steps)  # as many as the device-timed region; fill and drain are included
    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(s_in)
    for _ in range(e2e_steps):
        e2e_step()
    s_out.wait_stream(stream)
    s_out.wait_stream(s_in)
    ev1.record(s_out)
    torch.cuda.synchronize()
    out["e2e_ms"] = max_over_ranks(ev0.elapsed_time(ev1), world) / e2e_steps
    if not torch.equal(oh, sets[(n_e2e[0] - 1) % 2][4].cpu()):
        raise RuntimeError(f"{w.name}: end-to-end output differs from the device result")
    out["h2d"], out["d2h"] = h2d, d2h
    out["inputs"] = (q, k, v)
    return out


def summarize(w: wl.Workload, m: dict, steps: int, world: int, peaks: dict) -> dict:
    """Throughput, TFLOP/s (useful and executed), the attention roofline and per-kernel figures
    of one measured workload."""
    ms_step = m["ms"] / steps
    uf, xf = useful_flops(w), m["executed_flops"]
    per_kernel = m["per_kernel"]
    attn_ms, attn_n = per_kernel["attention"]
    attn_step_s = attn_ms / steps / 1e3                   # attention time per step
    peak = peaks["bf16_tflops_sustained"]
    achieved = uf / attn_step_s / 1e12
    kb = kernel_bytes(w)
    kern = {}
    for name, (kms, kn) in per_kernel.items():
        if kn == 0:
            continue
        ent = {"ms_per_launch": kms / kn, "launches": kn, "share": kms / max(m["ms_local"], 1e-9)}
        if name in kb:
            # kb holds the bytes of one whole step; a chunked problem launches a kernel several
            # times per step, so divide by the kernel's time per step
            gbs = kb[name] / (kms / steps / 1e3) / 1e9
            ent["gbs"] = gbs
            ent["hbm_frac"] = gbs / peaks["hbm_gbs"]
        kern[name] = ent
    if "gate" in kern:
        kern["gate"]["gate_tflops_fp32"] = gate_flops(w) / (kern["gate"]["ms_per_launch"] / 1e3) / 1e12
    cg = None
    if "centroid" in per_kernel and "gate" in per_kernel:
        cg_s = (per_kernel["centroid"][0] + per_kernel["gate"][0]) / steps / 1e3
        cg = (kb["centroid"] + kb["gate"]) / cg_s / 1e9 / peaks["hbm_gbs"]
    return {
        "ms_per_step": ms_step,
        "value": job_throughput(world, w.total_tokens, ms_step),
        "tflops_useful": uf * world / (ms_step / 1e3) / 1e12,
        "tflops_executed": xf * world / (ms_step / 1e3) / 1e12,
        "attention": {"achieved_useful": achieved, "achieved_executed": xf / attn_step_s / 1e12,
                      "frac": achieved / peak, "frac_executed": xf / attn_step_s / 1e12 / peak,
                      "frac_of_burst": achieved / peaks["bf16_tflops"],
                      "useful_tflop": uf / 1e12, "executed_tflop": xf / 1e12,
                      "ms_per_step": attn_ms / steps},
        "centroid_gate_hbm_frac": cg,
        "kernels": kern,
        "launches_per_step": m["launches"] / steps,
    }


def measure_backward(w: wl.Workload, steps: int, warmup: int, peaks: dict) -> dict:
    """Times moba_attn_bwd on `w` (one GPU): the forward pass runs once first for O, LSE and the
    routing; dO is seeded N(0, 1). Useful FLOPs: 10 d per attended (query, key) pair and head
    (S recomputed, dP, dV, dK, dQ); the key-stationary kernel issues 8 d of them per pair (S, dP,
    dV, dK) and the query-stationary one 6 d (S, dP, dQ)."""
    from block_sparse_long_moba_b200 import moba

    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v, cu = wl.make_inputs(w, seed=0, device=dev)
    T, H, d = w.total_tokens, w.hq, w.d
    idx = torch.empty((H, T, w.topk), dtype=torch.int32, device=dev)
    o, lse = moba.moba_attn_fwd(q, k, v, cu, w.cu_seqlens, w.block_size, w.topk, w.scale,
                                block_idx_out=idx)
    g = torch.Generator(device=dev).manual_seed(5)
    d_o = torch.randn(q.shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(moba.moba_bwd_workspace_bytes(w.cu_seqlens, H, w.hkv, d, w.block_size,
                                                   w.topk), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        moba.moba_attn_bwd(q, k, v, o, lse, d_o, idx, cu, w.cu_seqlens, w.block_size, w.topk,
                           w.scale, dq=dq, dk=dk, dv=dv, workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if moba.moba_device_status(ws) != 0:
        raise RuntimeError(f"{w.name} backward: device status after warm-up")
    moba.timing_reset()
    moba.timing_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    moba.timing_enable(False)
    per = moba.timing_read()
    ms = ev0.elapsed_time(ev1) / steps
    if moba.moba_device_status(ws) != 0:
        raise RuntimeError(f"{w.name} backward: device status after the timed region")
    pairs = attended_pairs(w)
    peak = peaks["bf16_tflops_sustained"]
    kern = {}
    for name, flop_per_pair in (("bwd_dkdv", 8.0 * d), ("bwd_dq", 6.0 * d), ("bwd_aux", None)):
        kms, kn = per.get(name, (0.0, 0))
        if kn == 0:
            continue
        ent = {"ms_per_step": kms / steps, "launches_per_step": kn / steps}
        if flop_per_pair:
            tf = flop_per_pair * pairs / (kms / steps / 1e3) / 1e12
            ent.update({"tflops": tf, "frac": tf / peak})
        kern[name] = ent
    for name in ("route_count", "route_scan", "route_scatter", "plan"):
        kms, kn = per.get(name, (0.0, 0))
        if kn:
            kern[name] = {"ms_per_step": kms / steps}
    useful = 10.0 * d * pairs
    return {"workload": w.name, "steps": steps, "warmup": warmup, "ms_per_step": ms,
            "tflops_useful": useful / (ms / 1e3) / 1e12,
            "frac_of_peak_sustained": useful / (ms / 1e3) / 1e12 / peak,
            "useful_tflop": useful / 1e12, "kernels": kern,
            "peak": peak, "peak_kind": f"bf16 dense sustained, {peaks['source']}"}


DECODE_CACHE = dict(nseq=8, L=131072, hq=32, hkv=8, d=128, block_size=4096, topk=12)


def measure_decode(steps: int, warmup: int, peaks: dict) -> dict:
    """Times moba_decode_fwd: one new query per sequence for 8 sequences with 128K cached tokens
    each (the Llama-3.1-8B attention shape). Algorithmic bytes: the K and V rows of the blocks the
    query heads of a kv group select (their union, read once), plus Q, the past centroids and the
    outputs; the kernels read each head's blocks separately, so the union is the floor that L2
    reuse across a group's heads can reach."""
    from block_sparse_long_moba_b200 import moba

    c = DECODE_CACHE
    cu_l = [c["L"] * s for s in range(c["nseq"] + 1)]
    w = wl.custom(cu_l, c["hq"], c["hkv"], c["d"], c["block_size"], c["topk"], "offset",
                  name="decode_128k_b8")
    dev = torch.device("cuda", torch.cuda.current_device())
    q_all, k, v, cu = wl.make_inputs(w, seed=0, device=dev)
    last = torch.tensor([x - 1 for x in cu_l[1:]], device=dev)
    q = q_all[last].contiguous()
    del q_all
    cuq_l = list(range(c["nseq"] + 1))
    cuq = torch.tensor(cuq_l, dtype=torch.int32, device=dev)
    cents = moba.moba_centroids(k, cu, cu_l, c["block_size"])
    H, d, nq = c["hq"], c["d"], c["nseq"]
    idx = torch.empty((H, nq, c["topk"]), dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((H, nq), dtype=torch.float32, device=dev)
    ws = torch.empty(moba.moba_decode_workspace_bytes(cu_l, cuq_l, H, c["hkv"], d,
                                                      c["block_size"], c["topk"]),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        moba.moba_decode_fwd(q, k, v, cents, cu, cu_l, cuq, cuq_l, c["block_size"], c["topk"],
                             w.scale, block_idx_out=idx, o=o, lse=lse, workspace=ws,
                             stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / steps
    # union of the blocks selected by the heads of each (row, kv group); every block is full
    r = H // c["hkv"]
    sel = idx.view(c["hkv"], r, nq, c["topk"]).permute(0, 2, 1, 3).reshape(c["hkv"], nq, -1)
    uniq = sum(len(set(x for x in row.tolist() if x >= 0)) for grp in sel for row in grp)
    kv_bytes = uniq * c["block_size"] * d * 2 * 2
    nb_past = c["L"] // c["block_size"] - 1
    other = nq * H * d * 2 * 2 + nq * H * nb_past * d * 4 + nq * H * 4
    per_head = nq * H * c["topk"] * c["block_size"] * d * 2 * 2
    gbs = (kv_bytes + other) / (ms / 1e3) / 1e9
    return {"workload": w.name, "steps": steps, "warmup": warmup,
            "config": {"nseq": nq, "cache_tokens_per_seq": c["L"], "rows_per_seq": 1, "hq": H,
                       "hkv": c["hkv"], "d": d, "block_size": c["block_size"],
                       "topk": c["topk"]},
            "ms_per_step": ms, "rows_per_s": nq / (ms / 1e3),
            "bytes_algorithmic": kv_bytes + other, "bytes_per_head_reads": per_head + other,
            "gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"]}


def run_ours(args):
    from block_sparse_long_moba_b200 import build, moba

    world, rank, local = dist_setup(args.gpus)
    if rank == 0:
        build.build()
    barrier(world)
    moba.load_library()
    w = wl.WORKLOADS[args.workload]
    peaks = read_peaks()
    m = measure(w, args.steps, args.warmup, world, rank, local, seed=rank, e2e=True,
                clocks_on=True)
    summ = summarize(w, m, args.steps, world, peaks) if rank == 0 else None
    T, H, d = w.total_tokens, w.hq, w.d
    q, k, v = m.pop("inputs")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sampler = OracleSampler(w, q, k, v, target_s=oracle_target_seconds(args))
        cpu = sampler.sample()
    del q, k, v
    torch.cuda.empty_cache()

    extra = {}
    if world == 1 and not args.no_extra:
        for name, steps in EXTRA_WORKLOADS:
            if name == w.name:
                continue
            wx = wl.WORKLOADS[name]
            mx = measure(wx, steps, 2, world, rank, local, seed=rank, e2e=False, clocks_on=True)
            sx = summarize(wx, mx, steps, world, peaks)
            extra[name] = {"steps": steps, "warmup": 2, **sx, "clocks": mx["clocks"],
                           "config": {"T": wx.total_tokens, "hq": wx.hq, "hkv": wx.hkv,
                                      "d": wx.d, "block_size": wx.block_size, "topk": wx.topk,
                                      "nseq": wx.nseq}}
            del mx
            torch.cuda.empty_cache()

    bwd = dec = None
    if world == 1 and not args.no_extra:
        bwd = measure_backward(w, 3, 2, peaks)
        torch.cuda.empty_cache()
        dec = measure_decode(20, 3, peaks)
        torch.cuda.empty_cache()

    if rank == 0:
        ms_step = summ["ms_per_step"]
        att = summ["attention"]
        peak = peaks["bf16_tflops_sustained"]
        traffic = attention_traffic(w.name)
        line = {
            "metric": METRIC, "value": summ["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; Q,V ~ N(0,1), K = N(0,1) + per-block offset)",
            "config": {"workload": w.name, "T": T, "hq": H, "hkv": w.hkv, "d": d,
                       "block_size": w.block_size, "topk": w.topk, "nseq": w.nseq,
                       "parallelism": f"independent problem per GPU x{world}",
                       "l2": "no flush: Q/K/V inputs are larger than L2"},
            "tflops_useful": summ["tflops_useful"],
            "tflops_executed": summ["tflops_executed"],
            "tflops_frac_of_peak_sustained": summ["tflops_useful"] / world / peak,
            "roofline": {"kernel": "attention", "bound": "tensor", "achieved": att["achieved_useful"],
                         "peak": peak, "unit": "TFLOP/s", "frac": att["frac"],
                         "peak_kind": f"bf16 dense sustained, {peaks['source']}",
                         "frac_of_burst": att["frac_of_burst"],
                         "achieved_executed": att["achieved_executed"],
                         "frac_executed": att["frac_executed"],
                         "traffic": traffic},
            "centroid_gate_hbm_frac": summ["centroid_gate_hbm_frac"],
            "kernels": summ["kernels"],
            "gpu_launches": m["launches"],
            "e2e": {"value": world * T / (m["e2e_ms"] / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": m["h2d"], "d2h_bytes_per_step": m["d2h"],
                    "ms_per_step": m["e2e_ms"],
                    "pipelining": "two device buffer sets, three streams: the copy-in of step "
                                  "n+1 and the copy-out of step n-1 overlap the compute of step n"},
            "clocks": m["clocks"],
        }
        if extra:
            line["workloads"] = extra
        if bwd:
            line["backward"] = bwd
        if dec:
            line["decode"] = dec
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------- centroid + gate only
def run_gate_only(args):
    """Times steps 1-2 alone (moba_centroids + moba_gate_topk through the C ABI, no workspace) on
    the workload's inputs, one GPU: a small-footprint command for profiling the gate kernels."""
    from block_sparse_long_moba_b200 import build, moba

    build.build()
    moba.load_library()
    torch.cuda.set_device(0)
    w = wl.WORKLOADS[args.workload]
    q, k, v, cu = wl.make_inputs(w, seed=0, device="cuda")
    del v
    c = moba.moba_centroids(k, cu, w.cu_seqlens, w.block_size)
    idx = moba.moba_gate_topk(q, c, cu, w.cu_seqlens, w.block_size, w.topk)
    for _ in range(args.warmup):
        moba.moba_centroids(k, cu, w.cu_seqlens, w.block_size, out=c)
        moba.moba_gate_topk(q, c, cu, w.cu_seqlens, w.block_size, w.topk, out=idx)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    cms = gms = 0.0
    for _ in range(args.steps):
        ev[0].record()
        moba.moba_centroids(k, cu, w.cu_seqlens, w.block_size, out=c)
        ev[1].record()
        moba.moba_gate_topk(q, c, cu, w.cu_seqlens, w.block_size, w.topk, out=idx)
        ev[2].record()
        torch.cuda.synchronize()
        cms += ev[0].elapsed_time(ev[1])
        gms += ev[1].elapsed_time(ev[2])
    cms /= args.steps
    gms /= args.steps
    kb = kernel_bytes(w)
    hbm = read_peaks()["hbm_gbs"]
    both = (kb["centroid"] + kb["gate"]) / ((cms + gms) / 1e3) / 1e9
    print(json.dumps({"metric": "centroid + gate GB/s", "value": both, "unit": "GB/s",
                      "hbm_frac": both / hbm, "workload": w.name, "steps": args.steps,
                      "centroid_ms": cms, "gate_ms": gms,
                      "centroid_gbs": kb["centroid"] / (cms / 1e3) / 1e9,
                      "gate_gbs": kb["gate"] / (gms / 1e3) / 1e9}), flush=True)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The fp64 oracle as it stands, on the host cores, on the same workload: each step is one
    sample of a fixed number of query tokens (the same sample size the CPU-baseline leg uses)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    q, k, v, cu = wl.make_inputs(w, seed=0, device="cpu")
    sampler = OracleSampler(w, q, k, v, target_s=oracle_target_seconds(args))
    for _ in range(args.warmup):
        sampler.sample()
    vals = []
    t0 = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = sampler.sample()
        vals.append(last["value"])
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "T": w.total_tokens, "hq": w.hq, "hkv": w.hkv, "d": w.d,
                   "block_size": w.block_size, "topk": w.topk},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": last["sample"] if last else ""},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama8b_128k", choices=list(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (skip the 1M and small-block sub-records)")
    ap.add_argument("--only", choices=["gate", "backward", "decode"], default=None,
                    help="time one part alone on --workload (1 GPU; for profiling): centroids + "
                         "gate, the backward pass, or decode")
    args = ap.parse_args()
    if args.only == "gate":
        run_gate_only(args)
    elif args.only in ("backward", "decode"):
        from block_sparse_long_moba_b200 import build, moba
        build.build()
        moba.load_library()
        torch.cuda.set_device(0)
        peaks = read_peaks()
        if args.only == "backward":
            rec = measure_backward(wl.WORKLOADS[args.workload], args.steps, args.warmup, peaks)
        else:
            rec = measure_decode(args.steps, args.warmup, peaks)
        print(json.dumps(rec), flush=True)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
