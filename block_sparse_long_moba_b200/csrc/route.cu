// Block tables (plan) and K3 — routing inversion.
//
// The gate emits, per (query head, token), the blocks it attends. The attention kernel instead
// works per (kv head g, key block b) on a dense tile of the queries routed to b — the queries are
// gathered from scattered rows into one dense operand [FlashMoBA story, Gather-and-Densify]. The
// inversion is a counting sort of the routed (t, h, slot) triples by bucket (g, b):
//   route_count   : per-CTA shared-memory histograms, one global atomic per (CTA, bucket);
//   route_scan    : exclusive scan of the bucket counts -> list offsets, and the list of 256-row
//                   attention work items (bucket, first entry, rows);
//   route_scatter : per-CTA reservation of a contiguous range per bucket, then shared-memory
//                   cursors place every entry.
// An entry is the index of the partial-output row of (t, h, slot): ((t - T0) * Hq + h) * k + slot,
// so the attention kernel writes its result there and the merge reads the k slots of a row
// contiguously. The current block is not routed here: the attention kernel's diagonal tiles
// cover it. Order inside a bucket is not fixed; results do not depend on it because every
// attention row is computed independently of the other rows of its tile.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moba {

// One CTA: prefix of per-sequence block counts, per-block tables, zeroed bucket counters and
// status word.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ cu, int nseq,
                                                    int B, int NB, BlockTables tb,
                                                    int* __restrict__ counts, int ncounts,
                                                    int* __restrict__ status) {
  __shared__ int warp_sums[32];
  const int tid = threadIdx.x, nt = blockDim.x;
  // contiguous range of sequences per thread
  const int per = (nseq + nt - 1) / nt;
  const int s0 = min(nseq, tid * per), s1 = min(nseq, s0 + per);
  int local = 0;
  for (int s = s0; s < s1; ++s) local += blocks_of(cu[s + 1] - cu[s], B);
  // block-wide exclusive scan of `local`
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if ((tid & 31) >= o) incl += y;
  }
  if ((tid & 31) == 31) warp_sums[tid >> 5] = incl;
  __syncthreads();
  if (tid < 32) {
    int w = (tid < (nt >> 5)) ? warp_sums[tid] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (tid >= o) w += y;
    }
    warp_sums[tid] = w;  // inclusive over warps
  }
  __syncthreads();
  int run = incl - local + ((tid >> 5) > 0 ? warp_sums[(tid >> 5) - 1] : 0);
  for (int s = s0; s < s1; ++s) {
    tb.blk_off[s] = run;
    run += blocks_of(cu[s + 1] - cu[s], B);
  }
  if (tid == nt - 1) tb.blk_off[nseq] = run;
  if (tid == 0 && nseq == 0) tb.blk_off[0] = 0;
  __syncthreads();
  __threadfence_block();
  for (int b = tid; b < NB; b += nt) {
    int lo = 0, hi = nseq;  // largest s with blk_off[s] <= b (skipping empty sequences)
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tb.blk_off[mid] <= b) lo = mid; else hi = mid;
    }
    const int s = lo;
    const int j = b - tb.blk_off[s];
    const int start = cu[s] + j * B;
    tb.blk_seq[b] = s;
    tb.blk_start[b] = start;
    tb.blk_len[b] = min(B, cu[s + 1] - start);
  }
  for (int x = tid; x < ncounts; x += nt) counts[x] = 0;
  if (tid == 0) *status = 0;
}

// Walk the routed (t, h, slot) triples of one (query block b, kv head g): slots j < i only.
// The counting pass also checks each row against the routing contract the merge relies on: with
// n = min(topk, i + 1), slots 0 .. n-2 hold strictly ascending past blocks (0 <= j < i), slot n-1
// holds the current block i and the remaining slots hold -1. The diagonal tiles write slot n-1
// and the merge reads slots 0 .. n-1, so a row that breaks this (e.g. a caller-supplied routing
// with fewer blocks) would merge slots nobody wrote: it is reported as kDevBadRouting. Only slots
// 0 .. n-2 holding 0 <= j < i are counted and scattered, so a bad row can neither index out of
// bounds nor add more than n - 1 entries (the lists are sized for exactly that many per row).
template <bool kScatter>
__global__ void __launch_bounds__(256) route_pass_kernel(
    const int32_t* __restrict__ idx, BlockTables tb, int T, int H, int G, int topk, int NB,
    int b0, int T0, int* __restrict__ counts, int* __restrict__ cursor,
    int* __restrict__ entries, int* __restrict__ status, long long ent_cap) {
  extern __shared__ int hist[];
  const int b = b0 + blockIdx.x, g = blockIdx.y;
  const int s = tb.blk_seq[b];
  const int base = tb.blk_off[s];
  const int i = b - base;
  if (kScatter && i == 0) return;
  const int len = tb.blk_len[b], tstart = tb.blk_start[b];
  const int r = H / G;
  for (int x = threadIdx.x; x < i; x += blockDim.x) hist[x] = 0;
  __syncthreads();
  const int rows = r * len;
  const int n = min(topk, i + 1);
  bool bad = false;
  for (int row = threadIdx.x; row < rows; row += blockDim.x) {
    const int hh = row / len, t = tstart + row % len;
    const int32_t* rp = idx + (static_cast<size_t>(g * r + hh) * T + t) * topk;
    int prev = -1;
    for (int slot = 0; slot < topk; ++slot) {
      const int j = __ldg(rp + slot);
      if (!kScatter) {
        bad |= slot < n - 1 ? (j <= prev || j >= i) : slot == n - 1 ? (j != i) : (j != -1);
        prev = j;
      }
      if (slot < n - 1 && j >= 0 && j < i) atomicAdd(&hist[j], 1);
    }
  }
  if (!kScatter) {
    if (__syncthreads_or(bad) && threadIdx.x == 0 && status)
      atomicCAS(status, 0, kDevBadRouting);
    if (i == 0) return;
  } else {
    __syncthreads();
  }
  int* gbucket = (kScatter ? cursor : counts) + static_cast<size_t>(g) * NB + base;
  for (int x = threadIdx.x; x < i; x += blockDim.x) {
    const int c = hist[x];
    if (c) {
      const int pos = atomicAdd(&gbucket[x], c);
      if (kScatter) hist[x] = pos;
    }
  }
  if (!kScatter) return;
  __syncthreads();
  for (int row = threadIdx.x; row < rows; row += blockDim.x) {
    const int hh = row / len, t = tstart + row % len;
    const int h = g * r + hh;
    const int32_t* rp = idx + (static_cast<size_t>(h) * T + t) * topk;
    const int prow = ((t - T0) * H + h) * topk;
    for (int slot = 0; slot < n - 1; ++slot) {
      const int j = __ldg(rp + slot);
      if (j >= 0 && j < i) {
        const int pos = atomicAdd(&hist[j], 1);
        if (in_range(pos, ent_cap, status)) entries[pos] = prow + slot;
      }
    }
  }
}

// One CTA of 1024 threads: offsets, cursors and the 256-row work-item list of every bucket; resets the
// bucket counters for the next chunk.
__global__ void __launch_bounds__(1024) route_scan_kernel(int* __restrict__ counts, int nbk,
                                                          int* __restrict__ cursor,
                                                          int4* __restrict__ tiles,
                                                          int* __restrict__ n_tiles,
                                                          long long tiles_cap,
                                                          int* __restrict__ status) {
  __shared__ int ws_c[32], ws_t[32];
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (nbk + nt - 1) / nt;
  const int k0 = min(nbk, tid * per), k1 = min(nbk, k0 + per);
  int lc = 0, lt = 0;
  for (int x = k0; x < k1; ++x) {
    const int c = counts[x];
    lc += c;
    lt += (c + kItemRows - 1) / kItemRows;
  }
  int ic = lc, it = lt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yc = __shfl_up_sync(0xffffffffu, ic, o);
    const int yt = __shfl_up_sync(0xffffffffu, it, o);
    if ((tid & 31) >= o) {
      ic += yc;
      it += yt;
    }
  }
  if ((tid & 31) == 31) {
    ws_c[tid >> 5] = ic;
    ws_t[tid >> 5] = it;
  }
  __syncthreads();
  if (tid < 32) {
    int wc = (tid < (nt >> 5)) ? ws_c[tid] : 0;
    int wt = (tid < (nt >> 5)) ? ws_t[tid] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yc = __shfl_up_sync(0xffffffffu, wc, o);
      const int yt = __shfl_up_sync(0xffffffffu, wt, o);
      if (tid >= o) {
        wc += yc;
        wt += yt;
      }
    }
    ws_c[tid] = wc;
    ws_t[tid] = wt;
  }
  __syncthreads();
  const int wprev_c = (tid >> 5) > 0 ? ws_c[(tid >> 5) - 1] : 0;
  const int wprev_t = (tid >> 5) > 0 ? ws_t[(tid >> 5) - 1] : 0;
  int off = ic - lc + wprev_c;
  int toff = it - lt + wprev_t;
  for (int x = k0; x < k1; ++x) {
    const int c = counts[x];
    cursor[x] = off;
    for (int y = 0; y * kItemRows < c; ++y)
      if (in_range(toff + y, tiles_cap, status))
        tiles[toff + y] = make_int4(x, off + y * kItemRows, min(kItemRows, c - y * kItemRows), 0);
    toff += (c + kItemRows - 1) / kItemRows;
    off += c;
    counts[x] = 0;
  }
  if (tid == nt - 1) {
    n_tiles[0] = toff;
    n_tiles[1] = off;  // routed entries of the chunk
  }
}

// Densify (d = 64): row p of qdense = the query row of routed entry p, so that the attention
// kernel reads a work item's gathered rows as dense 128-row tiles. Consecutive entries are written
// to consecutive rows (coalesced: eight lanes per 128-byte row, four rows per warp instruction);
// the query rows are read at random and are mostly L2-resident.
__global__ void __launch_bounds__(256) densify_kernel(const int* __restrict__ entries,
                                                      const int* __restrict__ n_entries,
                                                      const __nv_bfloat16* __restrict__ q, int H,
                                                      int topk, int T0,
                                                      __nv_bfloat16* __restrict__ qdense,
                                                      long long cap, long long q_rows,
                                                      int* __restrict__ status) {
  const int n = *n_entries;
  const int lane8 = threadIdx.x & 7;
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x >> 3);
  for (long long p = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3; p < n;
       p += stride) {
    if (!in_range(p, cap, status)) break;
    const int e = __ldg(entries + p);
    const long long row = static_cast<long long>(T0) * H + e / topk;  // t * H + h
    if (!in_range(row, q_rows, status)) continue;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(q + row * 64) + lane8);
    __stcs(reinterpret_cast<uint4*>(qdense + p * 64) + lane8, v);
  }
}

cudaError_t launch_plan(const int32_t* cu_dev, int nseq, int B, int NB, const BlockTables& tb,
                        int* counts, int ncounts, int* status, cudaStream_t stream) {
  plan_kernel<<<1, 1024, 0, stream>>>(cu_dev, nseq, B, NB, tb, counts, ncounts, status);
  return cudaGetLastError();
}

cudaError_t launch_route_count(const int32_t* idx, const BlockTables& tb, int T, int H, int G,
                               int topk, int NB, int b0, int nblk, int T0, int max_nb,
                               int* counts, int* status, cudaStream_t stream) {
  const int smem = max_nb * 4;
  cudaError_t e = cudaFuncSetAttribute(route_pass_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  route_pass_kernel<false><<<dim3(nblk, G), 256, smem, stream>>>(
      idx, tb, T, H, G, topk, NB, b0, T0, counts, nullptr, nullptr, status, 0);
  return cudaGetLastError();
}

cudaError_t launch_route_scan(int* counts, int nbk, int* cursor, int4* tiles, int* n_tiles,
                              long long tiles_cap, int* status, cudaStream_t stream) {
  route_scan_kernel<<<1, 1024, 0, stream>>>(counts, nbk, cursor, tiles, n_tiles, tiles_cap,
                                            status);
  return cudaGetLastError();
}

cudaError_t launch_densify(const int* entries, const int* n_entries, const void* q, int H,
                           int topk, int T0, long long max_entries, void* qdense, int num_sms,
                           long long q_rows, int* status, cudaStream_t stream) {
  const long long want = (max_entries + 31) / 32;  // 32 rows per CTA pass
  const int grid = static_cast<int>(std::min<long long>(std::max(want, 1LL), 8LL * num_sms));
  densify_kernel<<<grid, 256, 0, stream>>>(entries, n_entries,
                                           static_cast<const __nv_bfloat16*>(q), H, topk, T0,
                                           static_cast<__nv_bfloat16*>(qdense), max_entries,
                                           q_rows, status);
  return cudaGetLastError();
}

cudaError_t launch_route_scatter(const int32_t* idx, const BlockTables& tb, int T, int H, int G,
                                 int topk, int NB, int b0, int nblk, int T0, int max_nb,
                                 int* cursor, int* entries, long long ent_cap, int* status,
                                 cudaStream_t stream) {
  const int smem = max_nb * 4;
  cudaError_t e = cudaFuncSetAttribute(route_pass_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  route_pass_kernel<true><<<dim3(nblk, G), 256, smem, stream>>>(
      idx, tb, T, H, G, topk, NB, b0, T0, nullptr, cursor, entries, status, ent_cap);
  return cudaGetLastError();
}

}  // namespace moba
