// K6 — backward pass of the routed attention on the tcgen05 tensor cores [MoBA README (rpkg.in
// mirror), "Introducing MoBA": trainable block sparse attention]. The routing is held fixed (the
// top-k gate is piecewise constant in q and the centroids, as in top-k mixture-of-experts
// routing, so no gradient flows through it). For every row (t, h) over its attended keys u, with
// p_u = exp(scale q.k_u - LSE), D = dO . O and dS_u = p_u (dO . v_u - D):
//   dV[u] += p_u dO,   dK[u] += scale dS_u q,   dQ += scale sum_u dS_u k_u,
// and a kv head's dK / dV collect the terms of every query head of its group.
//
// The query range is processed in chunks of whole blocks (as in the forward pass), so that the
// routing lists and the densified rows of one chunk fit a fixed memory budget.
//   bwd_pre_kernel   D = dO . O per row (fp32), and the fp32 dQ accumulator zeroed.
//   bwd_densify      per chunk: the query and dO rows of every routed entry copied in list order
//                    into dense arrays, with the row's log2-domain LSE, D and position, so that a
//                    routed query tile is one 128-row TMA tile load [FlashMoBA story, Gather-and-
//                    Densify] — every key sub-tile of the block reads the same tiles again.
//   bwd_dkdv_kernel  key-stationary: one work item per (kv head g, block b, 128-key sub-tile j)
//                    walks every 128-row query tile of the chunk that attends those keys — the rows
//                    routed to b (dense tiles) and the rows of block b itself at or after the
//                    sub-tile (causal; 128 consecutive tokens of one head, a strided TMA tile) —
//                    and keeps dK, dV of its 128 keys in tensor memory, then adds them to the fp32
//                    dK, dV rows it owns (one owner per row in a launch: no atomics):
//                      S^T  = K_j Q^T      (M = 128 keys, N = 128 rows, K = d)
//                      dP^T = V_j dO^T
//                      P^T  = exp2(S^T scale log2e - LSE2), dS^T = P^T (dP^T - D), written back
//                             over S^T and dP^T in tensor memory as bf16
//                      dV  += P^T dO,  dK += dS^T Q   (A from tensor memory, B MN-major)
//   bwd_dq_kernel    query-stationary: one item per 128 query rows of one (g, b) routing list (a
//                    run of the densified rows) or of one head inside its own block (causal),
//                    loaded as TMA tiles, walks the 128-key sub-tiles of b:
//                      S = Q K_j^T, dP = dO V_j^T, dS = P (dP - D) over dP in tensor memory,
//                      dQ += dS K_j
//                    and adds scale * dQ once per item into the fp32 accumulator (red.global.add;
//                    a row collects one addition per selected block).
//   bwd_finish       dQ, dK, dV = bf16(accumulators).
// Warp roles: warp 0 = TMA producer (tiles and, for the query tiles, the per-row LSE / D
// columns), warp 1 = TMEM owner and MMA issuer, then one thread per tensor-memory lane for the
// elementwise softmax-gradient step and the epilogues: warps 4-7 and 8-11 (384 threads; each
// warpgroup takes half of the tile's columns: query rows in the dK/dV kernel, keys in the dQ
// kernel). Every wait is
// bounded; on a timeout the CTA raises its abort flag, records a status code, lets its copies and
// matrix products in flight finish (under the fixed drain limit) and returns. No TMA multicast.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace moba {

constexpr int kKvThreads = 384;  // dK/dV and dQ kernels: two elementwise warpgroups
constexpr int kOneCtaPerSmBytes = 120 * 1024;  // more than half of an SM's shared memory

struct BwdArgs {
  const float* lse;         // [H, T] natural log
  const float* dsum;        // [T * H] D = dO . O
  const int* entries;       // chunk's routed entries (((t - T0) * H + h) * topk + slot) by (g, b)
  const int* bucket_end;    // [G * NB] end offset of every (g, b) list of the chunk
  const int4* tiles;        // routed 256-row items {bucket, first entry, rows}
  const int* n_routed;      // device count of routed items
  const float* col_lse;     // densified entries: log2-domain LSE, D and position of each row
  const float* col_d;
  const int* col_t;
  BlockTables tb;
  float* dq_acc;            // [T * H, D]
  float* dk_acc;            // [T, G, D]
  float* dv_acc;
  int* status;
  int T, H, G, r, topk, NB, SPB;
  int T0, b0, nblk;         // the chunk: first token, first query block, query blocks
  long long dense_rows;     // capacity of the chunk's entries and densified arrays (checks)
  float scale_log2, scale;
  unsigned long long wait_ns;
};

// Operand layout of one 128-row tile of D columns: D / 64 swizzle atoms of [128 rows][128 bytes]
// (128-byte swizzle), atom stride 16 KB — the layout a (64, 1, 128) TMA box or four-row
// tile::gather4 copies write.
template <int D>
struct BwdTile {
  static constexpr int BYTES = 128 * D * 2;
};

// K-major descriptor step for 16 columns (k-step ks) of a [128][D] tile.
__device__ __forceinline__ uint32_t kmajor_step(int ks) { return (ks >> 2) * 16384 + (ks & 3) * 32; }

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// ------------------------------------------------------------------------------------- D, zero
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      long long rows, float* __restrict__ dsum,
                                                      float* __restrict__ dq_acc) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int PER = D / 32;
  const __nv_bfloat16* po = o + row * D + lane * PER;
  const __nv_bfloat16* pd = dout + row * D + lane * PER;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) acc = fmaf(__bfloat162float(po[e]), __bfloat162float(pd[e]), acc);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) dsum[row] = acc;
#pragma unroll
  for (int e = 0; e < PER; ++e) dq_acc[row * D + lane * PER + e] = 0.f;
}

__global__ void __launch_bounds__(256) bwd_zero_kernel(float4* __restrict__ p, long long n4) {
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < n4;
       x += static_cast<long long>(gridDim.x) * blockDim.x)
    p[x] = make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void __launch_bounds__(256) bwd_finish_kernel(const float4* __restrict__ acc,
                                                         long long n4, uint2* __restrict__ out) {
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < n4;
       x += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = acc[x];
    out[x] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
}

// Densify one chunk's routed entries: dense row p = query row and dO row of entry p, plus the
// row's log2-domain LSE, D and position. Consecutive entries go to consecutive rows (coalesced
// 16-byte stores, D / 8 lanes per row); the source rows are read at random.
template <int D>
__global__ void __launch_bounds__(256) bwd_densify_kernel(
    const int* __restrict__ entries, const int* __restrict__ n_entries,
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ dsum, int T, int H, int topk, int T0,
    __nv_bfloat16* __restrict__ qd, __nv_bfloat16* __restrict__ dd, float* __restrict__ col_lse,
    float* __restrict__ col_d, int* __restrict__ col_t, long long cap, int* __restrict__ status) {
  constexpr int LPR = D / 8;  // lanes per row
  const int n = *n_entries;
  const int sub = threadIdx.x % LPR;
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x / LPR);
  for (long long p = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / LPR; p < n;
       p += stride) {
    if (!in_range(p, cap, status)) break;
    const long long row = static_cast<long long>(T0) * H + __ldg(entries + p) / topk;
    if (!in_range(row, static_cast<long long>(T) * H, status)) continue;
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(q + row * D) + sub);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + sub);
    __stcs(reinterpret_cast<uint4*>(qd + p * D) + sub, a);
    __stcs(reinterpret_cast<uint4*>(dd + p * D) + sub, b);
    if (sub == 0) {
      const int t = static_cast<int>(row / H), h = static_cast<int>(row % H);
      col_lse[p] = __ldg(lse + static_cast<size_t>(h) * T + t) * 1.4426950408889634f;
      col_d[p] = __ldg(dsum + row);
      col_t[p] = t;
    }
  }
}

// ------------------------------------------------------------------------------- dK, dV kernel
// Query tiles of item (g, b, j): first the routed rows of (g, b) in 128-row tiles, then, for each
// query head of the group, the rows of block b from the sub-tile's first key to the block's end.
struct KvItem {
  bool valid;
  int g, b, j;
  int key0, klen;         // first key of the sub-tile, keys in it (<= 128)
  int bend;               // one past the block's last key
  int rstart, rcount;     // routed list range
  int nrt, ndt_head, ntile;  // routed tiles, diagonal tiles per head, total
};

__device__ __forceinline__ KvItem kv_item(const BwdArgs& a, int w) {
  KvItem it;
  it.j = w % a.SPB;
  const int x = w / a.SPB;  // bucket g * NB + b: a bucket's sub-tiles are consecutive items
  it.g = x / a.NB;
  it.b = x % a.NB;
  const int bstart = a.tb.blk_start[it.b], blen = a.tb.blk_len[it.b];
  it.key0 = bstart + it.j * 128;
  it.klen = min(128, blen - it.j * 128);
  it.bend = bstart + blen;
  it.rstart = x > 0 ? a.bucket_end[x - 1] : 0;
  it.rcount = a.bucket_end[x] - it.rstart;
  if (it.rcount > 0 && (!in_range(it.rstart, a.dense_rows, a.status) ||
                        !in_range(static_cast<long long>(it.rstart) + it.rcount - 1, a.dense_rows,
                                  a.status)))
    it.rcount = 0;  // (MOBA_CHECKS) a corrupt list is skipped by every role alike
  it.nrt = (it.rcount + 127) / 128;
  // the block's own rows belong to the chunk that holds the block
  const bool own = it.b >= a.b0 && it.b < a.b0 + a.nblk;
  it.ndt_head = own ? (it.bend - it.key0 + 127) / 128 : 0;
  it.ntile = it.nrt + a.r * it.ndt_head;
  it.valid = it.j * 128 < blen && it.ntile > 0;
  return it;
}

template <int D>
struct KvCfg {
  static constexpr int TILE = BwdTile<D>::BYTES;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;             // stage s: Q at OFF_Q + s * 2 TILE
  static constexpr int OFF_DO = 3 * TILE;            //          dO at OFF_DO + s * 2 TILE
  static constexpr int OFF_COL = 6 * TILE;           // [2 stages][128] {lse2, D} per column
  static constexpr int OFF_BARS = OFF_COL + 2 * 128 * 8;
  static constexpr int SMEM = OFF_BARS + 256;
};

struct KvBars {
  uint64_t kv_full, kv_empty;
  uint64_t qd_full[2], qd_empty[2];
  uint64_t s_full, p_full, acc_full, acc_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kKvThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v,
                    const __grid_constant__ CUtensorMap map_q3,
                    const __grid_constant__ CUtensorMap map_do3,
                    const __grid_constant__ CUtensorMap map_qd,
                    const __grid_constant__ CUtensorMap map_dd, const BwdArgs a, int n_items) {
  using C = KvCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  KvBars* bars = reinterpret_cast<KvBars*>(smem + C::OFF_BARS);
  float2* col = reinterpret_cast<float2*>(smem + C::OFF_COL);  // [stage][128] {lse2, D}
  volatile int* abort_flag = &bars->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicCAS(a.status, 0, kDevSmemAlign);
    return;
  }
  if (tid == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->qd_full[s], 33);  // lane 0's expected bytes + the 32 lanes' columns
      mbar_init(&bars->qd_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 256);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_free, 256);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
    prefetch_tensormap(&map_q3);
    prefetch_tensormap(&map_do3);
    prefetch_tensormap(&map_qd);
    prefetch_tensormap(&map_dd);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint64_t TO = a.wait_ns;
  int* err = a.status;
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu,
                      mbar_wait_bounded(bar, parity, abort_flag, err, kDevTimeoutAttn, TO));
  };
  constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DK = 256, TM_DV = 256 + D;

  if (warp == 0) {
    // ------------------------------------------------------------------------ producer
    uint32_t gt = 0, li = 0;  // query tiles and items issued
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvItem it = kv_item(a, w);
      if (!it.valid) continue;
      ok = wait_all(&bars->kv_empty, (li & 1) ^ 1);
      if (!ok) break;
      mbar_arrive_expect_tx_elect(&bars->kv_full, 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d_elect(smem + C::OFF_K + c * 16384, &map_k, &bars->kv_full, c * 64, it.g,
                          it.key0);
        tma_load_3d_elect(smem + C::OFF_V + c * 16384, &map_v, &bars->kv_full, c * 64, it.g,
                          it.key0);
      }
      ++li;
      for (int n = 0; n < it.ntile; ++n, ++gt) {
        const int st = gt & 1;
        ok = wait_all(&bars->qd_empty[st], ((gt >> 1) & 1) ^ 1);
        if (!ok) break;
        // columns 4 lane .. 4 lane + 3 of the tile: {log2-domain LSE, D} of the row (padding
        // columns: LSE2 = +inf, so that p = 0); the rows themselves arrive as one 128-row TMA
        // tile (dense routed rows, or 128 consecutive tokens of one head)
        float2* cl = col + st * 128;
        uint8_t* dq_ = smem + C::OFF_Q + st * 2 * C::TILE;
        uint8_t* dd_ = smem + C::OFF_DO + st * 2 * C::TILE;
        if (n < it.nrt) {
          const int p0 = it.rstart + n * 128;
          const int rows = min(128, it.rcount - n * 128);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * lane + e;
            const bool on = c < rows;
            cl[c] = make_float2(on ? __ldg(a.col_lse + p0 + c) : INFINITY,
                                on ? __ldg(a.col_d + p0 + c) : 0.f);
          }
          if (lane == 0) mbar_arrive_expect_tx(&bars->qd_full[st], 2 * C::TILE);
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              tma_load_2d(dq_ + c * 16384, &map_qd, &bars->qd_full[st], c * 64, p0);
              tma_load_2d(dd_ + c * 16384, &map_dd, &bars->qd_full[st], c * 64, p0);
            }
          }
        } else {
          const int dn = n - it.nrt;
          const int h = it.g * a.r + dn / it.ndt_head;
          const int t0 = it.key0 + (dn % it.ndt_head) * 128;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * lane + e;
            const int t = t0 + c;
            const bool on = t < it.bend;
            cl[c] = make_float2(
                on ? __ldg(a.lse + static_cast<size_t>(h) * a.T + t) * 1.4426950408889634f
                   : INFINITY,
                on ? __ldg(a.dsum + static_cast<size_t>(t) * a.H + h) : 0.f);
          }
          if (lane == 0) mbar_arrive_expect_tx(&bars->qd_full[st], 2 * C::TILE);
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              tma_load_3d(dq_ + c * 16384, &map_q3, &bars->qd_full[st], c * 64, h, t0);
              tma_load_3d(dd_ + c * 16384, &map_do3, &bars->qd_full[st], c * 64, h, t0);
            }
          }
        }
        mbar_arrive(&bars->qd_full[st]);  // this lane's columns are written
      }
    }
    if (!ok) {
      // let the copies in flight land before the CTA exits (bounded)
      volatile int no_abort = 0;
      if (li > 0)
        mbar_wait_bounded(&bars->kv_full, (li - 1) & 1, &no_abort, err, kDevDrainTimeout,
                          kDrainTimeoutNs);
      for (uint32_t x = 0; x < 2 && x < gt; ++x) {
        const uint32_t g2 = gt - 1 - x;
        mbar_wait_bounded(&bars->qd_full[g2 & 1], (g2 >> 1) & 1, &no_abort, err,
                          kDevDrainTimeout, kDrainTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, 0, 1);  // B = dO / Q, MN-major
    const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
    uint32_t gt = 0, li = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvItem it = kv_item(a, w);
      if (!it.valid) continue;
      ok = wait_all(&bars->kv_full, li & 1);
      if (!ok) break;
      tc_fence_after();
      for (int n = 0; n < it.ntile; ++n, ++gt) {
        const int st = gt & 1;
        ok = wait_all(&bars->qd_full[st], (gt >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sQ = smem_u32(smem + C::OFF_Q + st * 2 * C::TILE);
        const uint32_t sD = smem_u32(smem + C::OFF_DO + st * 2 * C::TILE);
        {
          const uint64_t ak = smem_desc_sw128(sK, 16, 1024), bq = smem_desc_sw128(sQ, 16, 1024);
          const uint64_t av = smem_desc_sw128(sV, 16, 1024), bd = smem_desc_sw128(sD, 16, 1024);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ss_elect(tmem + TM_S, desc_advance(ak, kmajor_step(ks)),
                         desc_advance(bq, kmajor_step(ks)), IDESC_S, ks > 0 ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ss_elect(tmem + TM_DP, desc_advance(av, kmajor_step(ks)),
                         desc_advance(bd, kmajor_step(ks)), IDESC_S, ks > 0 ? 1u : 0u);
          mma_commit_elect(&bars->s_full);
        }
        ok = wait_all(&bars->p_full, gt & 1);
        if (!ok) break;
        if (n == 0 && li > 0) {
          // the previous item's dK / dV must have been read out before they are overwritten
          ok = wait_all(&bars->acc_free, (li - 1) & 1);
          if (!ok) break;
        }
        tc_fence_after();
        {
          const uint64_t bd = smem_desc_sw128(sD, 16384, 1024), bq = smem_desc_sw128(sQ, 16384, 1024);
          // packed rows 0..63 sit in columns 0..31 (first warpgroup), rows 64..127 in columns
          // 64..95 (second warpgroup): each half writes only columns it has read itself
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ts_elect(tmem + TM_DV, tmem + TM_S + (ks >> 2) * 64 + (ks & 3) * 8,
                         desc_advance(bd, ks * 2048), IDESC_ACC, (n > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ts_elect(tmem + TM_DK, tmem + TM_DP + (ks >> 2) * 64 + (ks & 3) * 8,
                         desc_advance(bq, ks * 2048), IDESC_ACC, (n > 0 || ks > 0) ? 1u : 0u);
          mma_commit_elect(&bars->qd_empty[st]);
        }
      }
      if (!ok) break;
      mma_commit_elect(&bars->kv_empty);
      mma_commit_elect(&bars->acc_full);
      ++li;
    }
    if (!ok) {
      volatile int no_abort = 0;
      mma_commit_elect(&bars->drain);
      mbar_wait_bounded(&bars->drain, 0, &no_abort, err, kDevDrainTimeout, kDrainTimeoutNs);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------- P, dS (thread = key) and dK, dV
    // two warpgroups on the same keys: half hw takes the tile's query columns 64 hw .. 64 hw + 63
    // and the d columns hw D/2 .. hw D/2 + D/2 - 1 of the epilogue
    const int hw = (warp - 4) >> 2;
    const int row = (warp & 3) * 32 + (tid & 31);  // tensor-memory lane = key of the sub-tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    uint32_t gt = 0, li = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvItem it = kv_item(a, w);
      if (!it.valid) continue;
      const bool kvalid = row < it.klen;
      const int u = it.key0 + row;
      for (int n = 0; n < it.ntile; ++n, ++gt) {
        const int st = gt & 1;
        ok = wait_all(&bars->qd_full[st], (gt >> 1) & 1);  // the tile's columns are in place
        if (!ok) break;
        ok = wait_all(&bars->s_full, gt & 1);
        if (!ok) break;
        tc_fence_after();
        const float4* cl4 = reinterpret_cast<const float4*>(col + st * 128);  // 2 columns each
        // columns c < cmin are queries before this key (the causal cut of the block's own rows:
        // u <= t0 + c); routed rows all follow the block
        int cmin = 0;
        if (n >= it.nrt) cmin = u - (it.key0 + ((n - it.nrt) % it.ndt_head) * 128);
        if (!kvalid) cmin = 128;
        // this half's two 32-column chunks; the second chunk's tensor-memory loads are in flight
        // while the first is computed. Packed P / dS of chunk ch of half hw go to columns
        // 64 hw + 16 ch .. + 15, inside this half's own (already read) columns.
        const int cbase = 64 * hw;
        uint32_t sr[2][32], dr[2][32];
        tmem_ld32(tmem + lane_off + TM_S + cbase, sr[0]);
        tmem_ld32(tmem + lane_off + TM_DP + cbase, dr[0]);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int cur = ch & 1;
          if (ch < 1) {
            tmem_ld32(tmem + lane_off + TM_S + cbase + 32, sr[1]);
            tmem_ld32(tmem + lane_off + TM_DP + cbase + 32, dr[1]);
          }
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            reg_fence(sr[cur][x]);
            reg_fence(dr[cur][x]);
          }
          uint32_t pp[16], dd[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const int c = cbase + 32 * ch + x;
            const float4 cc = cl4[c >> 1];  // {lse2, D} of columns c and c + 1
            const float p0 = c >= cmin ? ex2_approx(fmaf(__uint_as_float(sr[cur][x]), sl2, -cc.x))
                                       : 0.f;
            const float p1 = c + 1 >= cmin
                                 ? ex2_approx(fmaf(__uint_as_float(sr[cur][x + 1]), sl2, -cc.z))
                                 : 0.f;
            pp[x >> 1] = pack_bf16x2(p0, p1);
            dd[x >> 1] = pack_bf16x2(p0 * (__uint_as_float(dr[cur][x]) - cc.y),
                                     p1 * (__uint_as_float(dr[cur][x + 1]) - cc.w));
          }
          tmem_st16(tmem + lane_off + TM_S + cbase + 16 * ch, pp);
          tmem_st16(tmem + lane_off + TM_DP + cbase + 16 * ch, dd);
          if (ch < 1) tmem_wait_ld();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full);
      }
      if (!ok) break;
      // ---- epilogue: dK (scaled) and dV rows of this sub-tile's keys
      ok = wait_all(&bars->acc_full, li & 1);
      if (!ok) break;
      tc_fence_after();
      float* dka = a.dk_acc + (static_cast<size_t>(u) * a.G + it.g) * D;
      float* dva = a.dv_acc + (static_cast<size_t>(u) * a.G + it.g) * D;
#pragma unroll 1
      for (int c0 = hw * (D / 2); c0 < (hw + 1) * (D / 2); c0 += 32) {
        uint32_t kr[32], vr[32];
        tmem_ld32(tmem + lane_off + TM_DK + c0, kr);
        tmem_ld32(tmem + lane_off + TM_DV + c0, vr);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          reg_fence(kr[x]);
          reg_fence(vr[x]);
        }
        if (kvalid) {
          // this item owns rows (u, g): earlier chunks' sums are read back and extended
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            float4 kk = *reinterpret_cast<const float4*>(dka + c0 + x);
            float4 vv = *reinterpret_cast<const float4*>(dva + c0 + x);
            kk.x = fmaf(__uint_as_float(kr[x]), a.scale, kk.x);
            kk.y = fmaf(__uint_as_float(kr[x + 1]), a.scale, kk.y);
            kk.z = fmaf(__uint_as_float(kr[x + 2]), a.scale, kk.z);
            kk.w = fmaf(__uint_as_float(kr[x + 3]), a.scale, kk.w);
            vv.x += __uint_as_float(vr[x]);
            vv.y += __uint_as_float(vr[x + 1]);
            vv.z += __uint_as_float(vr[x + 2]);
            vv.w += __uint_as_float(vr[x + 3]);
            *reinterpret_cast<float4*>(dka + c0 + x) = kk;
            *reinterpret_cast<float4*>(dva + c0 + x) = vv;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_free);
      ++li;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------- dQ kernel
struct QItem {
  int kind;               // 0 empty, 1 routed, 2 diagonal
  int g, h, b;
  int rows, start;        // routed: first entry of the 128 rows; diagonal: first token
  int key0, klen, nsub;   // block's first key, keys attended (diagonal: up to the last row)
};

__device__ __forceinline__ QItem q_item(const BwdArgs& a, int w, int n_routed) {
  QItem it;
  it.kind = 0;
  it.h = 0;
  if (w < 2 * n_routed) {
    const int4 tl = a.tiles[w >> 1];
    const int half = w & 1;
    it.rows = min(128, tl.z - half * 128);
    if (it.rows <= 0) return it;
    if (!in_range(tl.x, static_cast<long long>(a.G) * a.NB, a.status) ||
        !in_range(static_cast<long long>(tl.y) + tl.z - 1, a.dense_rows, a.status))
      return it;  // (MOBA_CHECKS) a corrupt work item is skipped by every role alike
    it.kind = 1;
    it.g = tl.x / a.NB;
    it.b = tl.x % a.NB;
    it.start = tl.y + half * 128;
    it.key0 = a.tb.blk_start[it.b];
    it.klen = a.tb.blk_len[it.b];
    it.nsub = (it.klen + 127) / 128;
    return it;
  }
  const int wd = w - 2 * n_routed;
  it.h = wd % a.H;
  const int rest = wd / a.H;
  const int bl = a.b0 + rest % a.nblk;
  const int p = a.SPB - 1 - rest / a.nblk;  // longest first
  it.b = bl;
  const int len = a.tb.blk_len[bl];
  if (p * 128 >= len) return it;
  it.kind = 2;
  it.g = it.h / a.r;
  it.key0 = a.tb.blk_start[bl];
  it.rows = min(128, len - p * 128);
  it.start = it.key0 + p * 128;
  it.klen = p * 128 + it.rows;
  it.nsub = p + 1;
  return it;
}

template <int D>
struct QCfg {
  static constexpr int TILE = BwdTile<D>::BYTES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE;
  static constexpr int OFF_KV = 2 * TILE;  // stage s: K at OFF_KV + s * 2 TILE, V after it
  static constexpr int OFF_BARS = 6 * TILE;
  static constexpr int SMEM = OFF_BARS + 256;
};

struct QBars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t s_full, ds_full, dq_full, dq_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kKvThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_q3,
                  const __grid_constant__ CUtensorMap map_do3,
                  const __grid_constant__ CUtensorMap map_qd,
                  const __grid_constant__ CUtensorMap map_dd, const BwdArgs a) {
  using C = QCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  QBars* bars = reinterpret_cast<QBars*>(smem + C::OFF_BARS);
  volatile int* abort_flag = &bars->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicCAS(a.status, 0, kDevSmemAlign);
    return;
  }
  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->ds_full, 256);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, 256);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
    prefetch_tensormap(&map_q3);
    prefetch_tensormap(&map_do3);
    prefetch_tensormap(&map_qd);
    prefetch_tensormap(&map_dd);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_routed = *a.n_routed;
  const int n_items = 2 * n_routed + a.H * a.nblk * a.SPB;
  const uint64_t TO = a.wait_ns;
  int* err = a.status;
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu,
                      mbar_wait_bounded(bar, parity, abort_flag, err, kDevTimeoutAttn, TO));
  };
  constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256;

  if (warp == 0) {
    // ------------------------------------------------------------------------ producer
    uint32_t li = 0, J = 0;  // items and K/V sub-tiles issued
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const QItem it = q_item(a, w, n_routed);
      if (it.kind == 0) continue;
      ok = wait_all(&bars->q_empty, (li & 1) ^ 1);
      if (!ok) break;
      // the item's 128 query / dO rows as one TMA tile each: a run of the chunk's densified
      // routed rows, or 128 consecutive tokens of one head (rows past the item are never used)
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          if (it.kind == 1) {
            tma_load_2d(smem + C::OFF_Q + c * 16384, &map_qd, &bars->q_full, c * 64, it.start);
            tma_load_2d(smem + C::OFF_DO + c * 16384, &map_dd, &bars->q_full, c * 64, it.start);
          } else {
            tma_load_3d(smem + C::OFF_Q + c * 16384, &map_q3, &bars->q_full, c * 64, it.h,
                        it.start);
            tma_load_3d(smem + C::OFF_DO + c * 16384, &map_do3, &bars->q_full, c * 64, it.h,
                        it.start);
          }
        }
      }
      __syncwarp();
      ++li;
      for (int j = 0; j < it.nsub; ++j, ++J) {
        const int st = J & 1;
        ok = wait_all(&bars->kv_empty[st], ((J >> 1) & 1) ^ 1);
        if (!ok) break;
        mbar_arrive_expect_tx_elect(&bars->kv_full[st], 2 * C::TILE);
        uint8_t* sk = smem + C::OFF_KV + st * 2 * C::TILE;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d_elect(sk + c * 16384, &map_k, &bars->kv_full[st], c * 64, it.g,
                            it.key0 + j * 128);
          tma_load_3d_elect(sk + C::TILE + c * 16384, &map_v, &bars->kv_full[st], c * 64, it.g,
                            it.key0 + j * 128);
        }
      }
    }
    if (!ok) {
      volatile int no_abort = 0;
      if (li > 0)
        mbar_wait_bounded(&bars->q_full, (li - 1) & 1, &no_abort, err, kDevDrainTimeout,
                          kDrainTimeoutNs);
      for (uint32_t x = 0; x < 2 && x < J; ++x) {
        const uint32_t Jx = J - 1 - x;
        mbar_wait_bounded(&bars->kv_full[Jx & 1], (Jx >> 1) & 1, &no_abort, err, kDevDrainTimeout,
                          kDrainTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, D, 0, 1);  // B = K, MN-major
    const uint32_t sQ = smem_u32(smem + C::OFF_Q), sD = smem_u32(smem + C::OFF_DO);
    uint32_t li = 0, J = 0, cs = 0;  // items, K/V sub-tiles, S/dS rounds
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const QItem it = q_item(a, w, n_routed);
      if (it.kind == 0) continue;
      ok = wait_all(&bars->q_full, li & 1);
      if (!ok) break;
      tc_fence_after();
      for (int j = 0; j < it.nsub; ++j, ++J, ++cs) {
        const int st = J & 1;
        ok = wait_all(&bars->kv_full[st], (J >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + C::OFF_KV + st * 2 * C::TILE);
        const uint32_t sV = sK + C::TILE;
        {
          const uint64_t aq = smem_desc_sw128(sQ, 16, 1024), bk = smem_desc_sw128(sK, 16, 1024);
          const uint64_t ad = smem_desc_sw128(sD, 16, 1024), bv = smem_desc_sw128(sV, 16, 1024);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ss_elect(tmem + TM_S, desc_advance(aq, kmajor_step(ks)),
                         desc_advance(bk, kmajor_step(ks)), IDESC_S, ks > 0 ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ss_elect(tmem + TM_DP, desc_advance(ad, kmajor_step(ks)),
                         desc_advance(bv, kmajor_step(ks)), IDESC_S, ks > 0 ? 1u : 0u);
          mma_commit_elect(&bars->s_full);
          if (j == it.nsub - 1) mma_commit_elect(&bars->q_empty);  // Q, dO read for the item
        }
        ok = wait_all(&bars->ds_full, cs & 1);
        if (!ok) break;
        if (j == 0 && li > 0) {
          ok = wait_all(&bars->dq_free, (li - 1) & 1);  // previous item's dQ has been read
          if (!ok) break;
        }
        tc_fence_after();
        {
          const uint64_t bk = smem_desc_sw128(sK, 16384, 1024);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            // packed keys 0..63 in columns 0..31 (first warpgroup), 64..127 in 64..95
            mma_ts_elect(tmem + TM_DQ, tmem + TM_DP + (ks >> 2) * 64 + (ks & 3) * 8,
                         desc_advance(bk, ks * 2048), IDESC_DQ, (j > 0 || ks > 0) ? 1u : 0u);
          mma_commit_elect(&bars->kv_empty[st]);
        }
      }
      if (!ok) break;
      mma_commit_elect(&bars->dq_full);
      ++li;
    }
    if (!ok) {
      volatile int no_abort = 0;
      mma_commit_elect(&bars->drain);
      mbar_wait_bounded(&bars->drain, 0, &no_abort, err, kDevDrainTimeout, kDrainTimeoutNs);
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- dS (thread = query row), dQ
    // two warpgroups on the same rows: half hw takes key columns 64 hw .. 64 hw + 63 and d
    // columns hw D/2 .. hw D/2 + D/2 - 1 of the epilogue
    const int hw = (warp - 4) >> 2;
    const int m = (warp & 3) * 32 + (tid & 31);
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    uint32_t li = 0, cs = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const QItem it = q_item(a, w, n_routed);
      if (it.kind == 0) continue;
      const bool rvalid = m < it.rows;
      int row = 0, t = 0;
      float lse2 = INFINITY, dsv = 0.f;  // padding rows: p = 0
      if (rvalid) {
        if (it.kind == 1) {
          // the densified row's columns (entry order = dense order)
          row = a.T0 * a.H + __ldg(a.entries + it.start + m) / a.topk;
          t = __ldg(a.col_t + it.start + m);
          lse2 = __ldg(a.col_lse + it.start + m);
          dsv = __ldg(a.col_d + it.start + m);
        } else {
          t = it.start + m;
          row = t * a.H + it.h;
          lse2 = __ldg(a.lse + static_cast<size_t>(it.h) * a.T + t) * 1.4426950408889634f;
          dsv = __ldg(a.dsum + row);
        }
      }
      for (int j = 0; j < it.nsub; ++j, ++cs) {
        ok = wait_all(&bars->s_full, cs & 1);
        if (!ok) break;
        tc_fence_after();
        const int u0 = it.key0 + j * 128;
        // valid key columns: inside the block, and (own block) not after the query
        int kmax = min(it.klen - j * 128, 128);
        if (it.kind == 2) kmax = min(kmax, t - u0 + 1);
        const int cbase = 64 * hw;
        uint32_t sr[2][32], dr[2][32];
        tmem_ld32(tmem + lane_off + TM_S + cbase, sr[0]);
        tmem_ld32(tmem + lane_off + TM_DP + cbase, dr[0]);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int cur = ch & 1;
          if (ch < 1) {
            tmem_ld32(tmem + lane_off + TM_S + cbase + 32, sr[1]);
            tmem_ld32(tmem + lane_off + TM_DP + cbase + 32, dr[1]);
          }
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            reg_fence(sr[cur][x]);
            reg_fence(dr[cur][x]);
          }
          uint32_t dd[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const int c = cbase + 32 * ch + x;
            const float p0 = c < kmax ? ex2_approx(fmaf(__uint_as_float(sr[cur][x]), sl2, -lse2))
                                      : 0.f;
            const float p1 = c + 1 < kmax
                                 ? ex2_approx(fmaf(__uint_as_float(sr[cur][x + 1]), sl2, -lse2))
                                 : 0.f;
            dd[x >> 1] = pack_bf16x2(p0 * (__uint_as_float(dr[cur][x]) - dsv),
                                     p1 * (__uint_as_float(dr[cur][x + 1]) - dsv));
          }
          tmem_st16(tmem + lane_off + TM_DP + cbase + 16 * ch, dd);
          if (ch < 1) tmem_wait_ld();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->ds_full);
      }
      if (!ok) break;
      ok = wait_all(&bars->dq_full, li & 1);
      if (!ok) break;
      tc_fence_after();
      float* dst = a.dq_acc + static_cast<size_t>(row) * D;
#pragma unroll 1
      for (int c0 = hw * (D / 2); c0 < (hw + 1) * (D / 2); c0 += 32) {
        uint32_t qr[32];
        tmem_ld32(tmem + lane_off + TM_DQ + c0, qr);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) reg_fence(qr[x]);
        if (rvalid && in_range(row, static_cast<long long>(a.T) * a.H, a.status)) {
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            red_add_v4(dst + c0 + x, __uint_as_float(qr[x]) * a.scale,
                       __uint_as_float(qr[x + 1]) * a.scale, __uint_as_float(qr[x + 2]) * a.scale,
                       __uint_as_float(qr[x + 3]) * a.scale);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->dq_free);
      ++li;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------- host side
static BwdArgs bwd_args(const BwdLaunch& L) {
  BwdArgs a;
  a.lse = L.lse;
  a.dsum = L.dsum;
  a.entries = L.entries;
  a.bucket_end = L.bucket_end;
  a.tiles = L.tiles;
  a.n_routed = L.n_routed;
  a.col_lse = L.col_lse;
  a.col_d = L.col_d;
  a.col_t = L.col_t;
  a.tb = L.tb;
  a.dq_acc = L.dq_acc;
  a.dk_acc = L.dk_acc;
  a.dv_acc = L.dv_acc;
  a.status = L.status;
  a.T = L.T;
  a.H = L.H;
  a.G = L.G;
  a.r = L.H / L.G;
  a.topk = L.topk;
  a.NB = L.NB;
  a.SPB = (L.B + 127) / 128;
  a.T0 = L.T0;
  a.b0 = L.b0;
  a.nblk = L.nblk;
  a.dense_rows = L.dense_rows;
  a.scale = L.scale;
  a.scale_log2 = L.scale * 1.4426950408889634f;
  a.wait_ns = L.wait_ns > 0 ? L.wait_ns : kWaitTimeoutNs;
  return a;
}

// [rows, D] bf16 dense rows -> 2-D map (D, rows), box (64, 128), 128-byte swizzle, zero fill past
// the last row.
static bool make_rows_tile_map(CUtensorMap* map, const void* base, long long rows, int D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static unsigned grid_for(long long n, int per_block, int num_sms) {
  return static_cast<unsigned>(
      std::max<long long>(1, std::min<long long>((n + per_block - 1) / per_block, 8LL * num_sms)));
}

cudaError_t launch_bwd_pre(const BwdLaunch& L, cudaStream_t stream) {
  const long long rows = static_cast<long long>(L.T) * L.H;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  const auto* o = static_cast<const __nv_bfloat16*>(L.o);
  const auto* dout = static_cast<const __nv_bfloat16*>(L.dout);
  if (L.d == 64)
    bwd_pre_kernel<64><<<grid, 256, 0, stream>>>(o, dout, rows, L.dsum, L.dq_acc);
  else
    bwd_pre_kernel<128><<<grid, 256, 0, stream>>>(o, dout, rows, L.dsum, L.dq_acc);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long n4 = static_cast<long long>(L.T) * L.G * L.d / 4;
  bwd_zero_kernel<<<grid_for(n4, 256, L.num_sms), 256, 0, stream>>>(
      reinterpret_cast<float4*>(L.dk_acc), n4);
  bwd_zero_kernel<<<grid_for(n4, 256, L.num_sms), 256, 0, stream>>>(
      reinterpret_cast<float4*>(L.dv_acc), n4);
  return cudaGetLastError();
}

cudaError_t launch_bwd_densify(const BwdLaunch& L, cudaStream_t stream) {
  const auto* q = static_cast<const __nv_bfloat16*>(L.q);
  const auto* dout = static_cast<const __nv_bfloat16*>(L.dout);
  auto* qd = static_cast<__nv_bfloat16*>(L.qd);
  auto* dd = static_cast<__nv_bfloat16*>(L.dd);
  const unsigned grid = grid_for(L.dense_rows, 256 / (L.d / 8), L.num_sms);
  if (L.d == 64)
    bwd_densify_kernel<64><<<grid, 256, 0, stream>>>(L.entries, L.n_routed + 1, q, dout, L.lse,
                                                     L.dsum, L.T, L.H, L.topk, L.T0, qd, dd,
                                                     L.col_lse, L.col_d, L.col_t, L.dense_rows,
                                                     L.status);
  else
    bwd_densify_kernel<128><<<grid, 256, 0, stream>>>(L.entries, L.n_routed + 1, q, dout, L.lse,
                                                      L.dsum, L.T, L.H, L.topk, L.T0, qd, dd,
                                                      L.col_lse, L.col_d, L.col_t, L.dense_rows,
                                                      L.status);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dkdv_d(const BwdLaunch& L, cudaStream_t stream) {
  CUtensorMap mk, mv, mq3, mdo3, mqd, mdd;
  if (!make_kv_map(&mk, L.k, L.T, L.G, D) || !make_kv_map(&mv, L.v, L.T, L.G, D) ||
      !make_kv_map(&mq3, L.q, L.T, L.H, D) || !make_kv_map(&mdo3, L.dout, L.T, L.H, D) ||
      !make_rows_tile_map(&mqd, L.qd, std::max(L.dense_rows, 1LL), D) ||
      !make_rows_tile_map(&mdd, L.dd, std::max(L.dense_rows, 1LL), D))
    return cudaErrorInvalidValue;
  const BwdArgs a = bwd_args(L);
  const int n_kv = a.NB * a.G * a.SPB;
  // each CTA allocates all 512 tensor-memory columns: ask for enough shared memory that two CTAs
  // never share an SM (the second would wait in tcgen05.alloc for the first to finish)
  const int smem = std::max(KvCfg<D>::SMEM, kOneCtaPerSmBytes);
  cudaError_t e =
      cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<std::min(L.num_sms, std::max(n_kv, 1)), kKvThreads, smem, stream>>>(
      mk, mv, mq3, mdo3, mqd, mdd, a, n_kv);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dq_d(const BwdLaunch& L, cudaStream_t stream) {
  CUtensorMap mk, mv, mq3, mdo3, mqd, mdd;
  if (!make_kv_map(&mk, L.k, L.T, L.G, D) || !make_kv_map(&mv, L.v, L.T, L.G, D) ||
      !make_kv_map(&mq3, L.q, L.T, L.H, D) || !make_kv_map(&mdo3, L.dout, L.T, L.H, D) ||
      !make_rows_tile_map(&mqd, L.qd, std::max(L.dense_rows, 1LL), D) ||
      !make_rows_tile_map(&mdd, L.dd, std::max(L.dense_rows, 1LL), D))
    return cudaErrorInvalidValue;
  const BwdArgs a = bwd_args(L);
  const int smem = std::max(QCfg<D>::SMEM, kOneCtaPerSmBytes);
  cudaError_t e =
      cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D><<<L.num_sms, kKvThreads, smem, stream>>>(mk, mv, mq3, mdo3, mqd, mdd, a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv(const BwdLaunch& L, cudaStream_t stream) {
  return L.d == 64 ? launch_dkdv_d<64>(L, stream) : launch_dkdv_d<128>(L, stream);
}

cudaError_t launch_bwd_dq(const BwdLaunch& L, cudaStream_t stream) {
  return L.d == 64 ? launch_dq_d<64>(L, stream) : launch_dq_d<128>(L, stream);
}

cudaError_t launch_bwd_finish(const BwdLaunch& L, cudaStream_t stream) {
  const long long nq4 = static_cast<long long>(L.T) * L.H * L.d / 4;
  const long long nk4 = static_cast<long long>(L.T) * L.G * L.d / 4;
  bwd_finish_kernel<<<grid_for(nq4, 256, L.num_sms), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(L.dq_acc), nq4, static_cast<uint2*>(L.dq));
  bwd_finish_kernel<<<grid_for(nk4, 256, L.num_sms), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(L.dk_acc), nk4, static_cast<uint2*>(L.dk));
  bwd_finish_kernel<<<grid_for(nk4, 256, L.num_sms), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(L.dv_acc), nk4, static_cast<uint2*>(L.dv));
  return cudaGetLastError();
}

}  // namespace moba
