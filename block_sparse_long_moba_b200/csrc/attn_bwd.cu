// K6 — backward pass of the routed attention on the tcgen05 tensor cores [MoBA README (rpkg.in
// mirror), "Introducing MoBA": trainable block sparse attention]. The routing is held fixed (the
// top-k gate is piecewise constant in q and the centroids, as in top-k mixture-of-experts
// routing, so no gradient flows through it). For every row (t, h) over its attended keys u, with
// p_u = exp(scale q.k_u - LSE), D = dO . O and dS_u = p_u (dO . v_u - D):
//   dV[u] += p_u dO,   dK[u] += scale dS_u q,   dQ += scale sum_u dS_u k_u,
// and a kv head's dK / dV collect the terms of every query head of its group.
//
//   bwd_pre_kernel   D = dO . O per row (fp32), and the fp32 dQ accumulator zeroed.
//   bwd_dkdv_kernel  key-stationary: one work item per (kv head g, block b, 128-key sub-tile j)
//                    walks every 128-row query tile that attends those keys — the rows routed to b
//                    (the routing inversion's list of (g, b), gathered from scattered rows) and the
//                    rows of block b itself at or after the sub-tile (causal) — and keeps dK, dV of
//                    its 128 keys in tensor memory; each key row has one owner, so no atomics:
//                      S^T  = K_j Q^T      (M = 128 keys, N = 128 rows, K = d)
//                      dP^T = V_j dO^T
//                      P^T  = exp2(S^T scale log2e - LSE2), dS^T = P^T (dP^T - D), written back
//                             over S^T and dP^T in tensor memory as bf16
//                      dV  += P^T dO,  dK += dS^T Q   (A from tensor memory, B MN-major)
//   bwd_dq_kernel    query-stationary: one item per 128 query rows of one (g, b) routing list, or
//                    of one head inside its own block (causal), walks the 128-key sub-tiles of b:
//                      S = Q K_j^T, dP = dO V_j^T, dS = P (dP - D) over dP in tensor memory,
//                      dQ += dS K_j
//                    and adds scale * dQ once per item into the fp32 accumulator (red.global.add;
//                    a row collects one addition per selected block).
//   bwd_dq_finish    dQ = bf16(accumulator).
// Warp roles (256 threads): warp 0 = TMA producer (tiles and, for the query tiles, the per-row
// LSE / D / position columns), warp 1 = TMEM owner and MMA issuer, warps 4-7 = one thread per
// tensor-memory lane (the elementwise softmax-gradient step and the epilogues). Every wait is
// bounded; on a timeout the CTA raises its abort flag, records a status code, lets its copies and
// matrix products in flight finish (under the fixed drain limit) and returns. No TMA multicast.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace moba {

constexpr int kBwdThreads = 256;
constexpr int kOneCtaPerSmBytes = 120 * 1024;  // more than half of an SM's shared memory

struct BwdArgs {
  const float* lse;         // [H, T] natural log
  const float* dsum;        // [T * H] D = dO . O
  const int* entries;       // routed entries ((t * H + h) * topk + slot), grouped by (g, b)
  const int* bucket_end;    // [G * NB] end offset of every (g, b) list
  const int4* tiles;        // routed 256-row items {bucket, first entry, rows}
  const int* n_routed;      // device count of routed items
  BlockTables tb;
  __nv_bfloat16* dk;        // [T, G, D]
  __nv_bfloat16* dv;
  float* dq_acc;            // [T * H, D]
  int* status;
  int T, H, G, r, topk, NB, SPB;
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

__global__ void __launch_bounds__(256) bwd_dq_finish_kernel(const float4* __restrict__ acc,
                                                            long long n4,
                                                            uint2* __restrict__ dq) {
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < n4;
       x += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = acc[x];
    dq[x] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
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
  const int bg = w / a.SPB;
  it.g = bg % a.G;
  it.b = bg / a.G;
  const int bstart = a.tb.blk_start[it.b], blen = a.tb.blk_len[it.b];
  it.valid = it.j * 128 < blen;
  it.key0 = bstart + it.j * 128;
  it.klen = min(128, blen - it.j * 128);
  it.bend = bstart + blen;
  const int x = it.g * a.NB + it.b;
  it.rstart = x > 0 ? a.bucket_end[x - 1] : 0;
  it.rcount = a.bucket_end[x] - it.rstart;
  it.nrt = (it.rcount + 127) / 128;
  it.ndt_head = (it.bend - it.key0 + 127) / 128;
  it.ntile = it.nrt + a.r * it.ndt_head;
  return it;
}

template <int D>
struct KvCfg {
  static constexpr int TILE = BwdTile<D>::BYTES;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;             // stage s: Q at OFF_Q + s * 2 TILE
  static constexpr int OFF_DO = 3 * TILE;            //          dO at OFF_DO + s * 2 TILE
  static constexpr int OFF_COL = 6 * TILE;           // [2 stages][3][128] lse2, D, position
  static constexpr int OFF_BARS = OFF_COL + 2 * 3 * 128 * 4;
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
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v,
                    const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_do, const BwdArgs a, int n_items) {
  using C = KvCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  KvBars* bars = reinterpret_cast<KvBars*>(smem + C::OFF_BARS);
  float* col = reinterpret_cast<float*>(smem + C::OFF_COL);  // [stage][lse2 | D | t][128]
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
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_free, 128);
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
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_do);
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
        // columns 4 lane .. 4 lane + 3 of the tile: query row (t * H + h), log2-domain LSE, D,
        // position; padding columns repeat a valid row and get LSE2 = +inf (p = 0)
        int rows4[4];
        float* cl = col + st * 3 * 128;
        int first_row = 0;
        for (int e = 0; e < 4; ++e) {
          const int c = 4 * lane + e;
          int row = -1, t = -1;
          if (n < it.nrt) {
            const int m = n * 128 + c;
            if (m < it.rcount) {
              row = __ldg(a.entries + it.rstart + m) / a.topk;
              t = row / a.H;
            }
            if (e == 0 && lane == 0) first_row = __ldg(a.entries + it.rstart + n * 128) / a.topk;
          } else {
            const int dn = n - it.nrt;
            const int h = it.g * a.r + dn / it.ndt_head;
            const int tt = it.key0 + (dn % it.ndt_head) * 128 + c;
            if (tt < it.bend) {
              t = tt;
              row = t * a.H + h;
            }
            if (e == 0 && lane == 0) first_row = (it.key0 + (dn % it.ndt_head) * 128) * a.H + h;
          }
          rows4[e] = row;
          if (row >= 0) {
            cl[c] = __ldg(a.lse + static_cast<size_t>(row % a.H) * a.T + t) * 1.4426950408889634f;
            cl[128 + c] = __ldg(a.dsum + row);
            reinterpret_cast<int*>(cl)[256 + c] = t;
          } else {
            cl[c] = INFINITY;
            cl[128 + c] = 0.f;
            reinterpret_cast<int*>(cl)[256 + c] = -1;
          }
        }
        first_row = __shfl_sync(0xffffffffu, first_row, 0);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (rows4[e] < 0) rows4[e] = first_row;
        if (lane == 0) mbar_arrive_expect_tx(&bars->qd_full[st], 2 * C::TILE);
        __syncwarp();
        uint8_t* dq_ = smem + C::OFF_Q + st * 2 * C::TILE + lane * 512;
        uint8_t* dd_ = smem + C::OFF_DO + st * 2 * C::TILE + lane * 512;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_gather4(dq_ + c * 16384, &map_q, &bars->qd_full[st], c * 64, rows4[0], rows4[1],
                      rows4[2], rows4[3]);
          tma_gather4(dd_ + c * 16384, &map_do, &bars->qd_full[st], c * 64, rows4[0], rows4[1],
                      rows4[2], rows4[3]);
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
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ts_elect(tmem + TM_DV, tmem + TM_S + ks * 8, desc_advance(bd, ks * 2048), IDESC_ACC,
                         (n > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ts_elect(tmem + TM_DK, tmem + TM_DP + ks * 8, desc_advance(bq, ks * 2048),
                         IDESC_ACC, (n > 0 || ks > 0) ? 1u : 0u);
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
    const int row = tid - 128;  // tensor-memory lane = key of the sub-tile
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
        const float* cl = col + st * 3 * 128;
        const int* ct = reinterpret_cast<const int*>(cl) + 256;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tmem + lane_off + TM_S + c0, sr);
          tmem_ld32(tmem + lane_off + TM_DP + c0, dr);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            reg_fence(sr[x]);
            reg_fence(dr[x]);
          }
          uint32_t pp[16], dd[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            float p[2], ds[2];
#pragma unroll
            for (int y = 0; y < 2; ++y) {
              const int c = c0 + x + y;
              const bool on = kvalid && u <= ct[c];
              p[y] = on ? ex2_approx(fmaf(__uint_as_float(sr[x + y]), sl2, -cl[c])) : 0.f;
              ds[y] = p[y] * (__uint_as_float(dr[x + y]) - cl[128 + c]);
            }
            pp[x >> 1] = pack_bf16x2(p[0], p[1]);
            dd[x >> 1] = pack_bf16x2(ds[0], ds[1]);
          }
          // packed in place: columns c0/2 .. c0/2 + 15 of S and dP were read by this or an
          // earlier chunk
          tmem_st16(tmem + lane_off + TM_S + c0 / 2, pp);
          tmem_st16(tmem + lane_off + TM_DP + c0 / 2, dd);
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
      __nv_bfloat16* dkr = a.dk + (static_cast<size_t>(u) * a.G + it.g) * D;
      __nv_bfloat16* dvr = a.dv + (static_cast<size_t>(u) * a.G + it.g) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
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
#pragma unroll
          for (int x = 0; x < 32; x += 8) {
            uint4 kk, vv;
            kk.x = pack_bf16x2(__uint_as_float(kr[x]) * a.scale, __uint_as_float(kr[x + 1]) * a.scale);
            kk.y = pack_bf16x2(__uint_as_float(kr[x + 2]) * a.scale, __uint_as_float(kr[x + 3]) * a.scale);
            kk.z = pack_bf16x2(__uint_as_float(kr[x + 4]) * a.scale, __uint_as_float(kr[x + 5]) * a.scale);
            kk.w = pack_bf16x2(__uint_as_float(kr[x + 6]) * a.scale, __uint_as_float(kr[x + 7]) * a.scale);
            vv.x = pack_bf16x2(__uint_as_float(vr[x]), __uint_as_float(vr[x + 1]));
            vv.y = pack_bf16x2(__uint_as_float(vr[x + 2]), __uint_as_float(vr[x + 3]));
            vv.z = pack_bf16x2(__uint_as_float(vr[x + 4]), __uint_as_float(vr[x + 5]));
            vv.w = pack_bf16x2(__uint_as_float(vr[x + 6]), __uint_as_float(vr[x + 7]));
            *reinterpret_cast<uint4*>(dkr + c0 + x) = kk;
            *reinterpret_cast<uint4*>(dvr + c0 + x) = vv;
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
  const int bl = rest % a.NB;
  const int p = a.SPB - 1 - rest / a.NB;  // longest first
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
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_q,
                  const __grid_constant__ CUtensorMap map_do, const BwdArgs a) {
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
    mbar_init(&bars->ds_full, 128);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, 128);
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
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_routed = *a.n_routed;
  const int n_items = 2 * n_routed + a.H * a.NB * a.SPB;
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
      int rows4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = 4 * lane + e;
        const int mm = m < it.rows ? m : 0;  // padding rows repeat row 0 (never written)
        rows4[e] = it.kind == 1 ? __ldg(a.entries + it.start + mm) / a.topk
                                : (it.start + mm) * a.H + it.h;
      }
      if (lane == 0) mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE);
      __syncwarp();
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_gather4(smem + C::OFF_Q + lane * 512 + c * 16384, &map_q, &bars->q_full, c * 64,
                    rows4[0], rows4[1], rows4[2], rows4[3]);
        tma_gather4(smem + C::OFF_DO + lane * 512 + c * 16384, &map_do, &bars->q_full, c * 64,
                    rows4[0], rows4[1], rows4[2], rows4[3]);
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
            mma_ts_elect(tmem + TM_DQ, tmem + TM_DP + ks * 8, desc_advance(bk, ks * 2048), IDESC_DQ,
                         (j > 0 || ks > 0) ? 1u : 0u);
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
    const int m = tid - 128;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    uint32_t li = 0, cs = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const QItem it = q_item(a, w, n_routed);
      if (it.kind == 0) continue;
      const bool rvalid = m < it.rows;
      int row = 0, t = 0;
      if (rvalid) {
        if (it.kind == 1) {
          row = __ldg(a.entries + it.start + m) / a.topk;
          t = row / a.H;
        } else {
          t = it.start + m;
          row = t * a.H + it.h;
        }
      }
      const float lse2 = rvalid ? __ldg(a.lse + static_cast<size_t>(row % a.H) * a.T + t) *
                                      1.4426950408889634f
                                : INFINITY;
      const float dsv = rvalid ? __ldg(a.dsum + row) : 0.f;
      const int tlim = (it.kind == 2) ? t : 0x7fffffff;  // causal inside the query's own block
      for (int j = 0; j < it.nsub; ++j, ++cs) {
        ok = wait_all(&bars->s_full, cs & 1);
        if (!ok) break;
        tc_fence_after();
        const int u0 = it.key0 + j * 128;
        const int kmax = min(it.klen - j * 128, 128);  // valid key columns of the sub-tile
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tmem + lane_off + TM_S + c0, sr);
          tmem_ld32(tmem + lane_off + TM_DP + c0, dr);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            reg_fence(sr[x]);
            reg_fence(dr[x]);
          }
          uint32_t dd[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            float ds[2];
#pragma unroll
            for (int y = 0; y < 2; ++y) {
              const int c = c0 + x + y;
              const bool on = c < kmax && u0 + c <= tlim;
              const float p = on ? ex2_approx(fmaf(__uint_as_float(sr[x + y]), sl2, -lse2)) : 0.f;
              ds[y] = p * (__uint_as_float(dr[x + y]) - dsv);
            }
            dd[x >> 1] = pack_bf16x2(ds[0], ds[1]);
          }
          tmem_st16(tmem + lane_off + TM_DP + c0 / 2, dd);
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
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t qr[32];
        tmem_ld32(tmem + lane_off + TM_DQ + c0, qr);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) reg_fence(qr[x]);
        if (rvalid) {
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
  a.tb = L.tb;
  a.dk = static_cast<__nv_bfloat16*>(L.dk);
  a.dv = static_cast<__nv_bfloat16*>(L.dv);
  a.dq_acc = L.dq_acc;
  a.status = L.status;
  a.T = L.T;
  a.H = L.H;
  a.G = L.G;
  a.r = L.H / L.G;
  a.topk = L.topk;
  a.NB = L.NB;
  a.SPB = (L.B + 127) / 128;
  a.scale = L.scale;
  a.scale_log2 = L.scale * 1.4426950408889634f;
  a.wait_ns = L.wait_ns > 0 ? L.wait_ns : kWaitTimeoutNs;
  return a;
}

static bool bwd_maps(const BwdLaunch& L, CUtensorMap* mk, CUtensorMap* mv, CUtensorMap* mq,
                     CUtensorMap* mdo) {
  return make_kv_map(mk, L.k, L.T, L.G, L.d) && make_kv_map(mv, L.v, L.T, L.G, L.d) &&
         make_q_rows_map(mq, L.q, static_cast<long long>(L.T) * L.H, L.d) &&
         make_q_rows_map(mdo, L.dout, static_cast<long long>(L.T) * L.H, L.d);
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
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dkdv_d(const BwdLaunch& L, cudaStream_t stream) {
  CUtensorMap mk, mv, mq, mdo;
  if (!bwd_maps(L, &mk, &mv, &mq, &mdo)) return cudaErrorInvalidValue;
  const BwdArgs a = bwd_args(L);
  const int n_kv = a.NB * a.G * a.SPB;
  // each CTA allocates all 512 tensor-memory columns: ask for enough shared memory that two CTAs
  // never share an SM (the second would wait in tcgen05.alloc for the first to finish)
  const int smem = std::max(KvCfg<D>::SMEM, kOneCtaPerSmBytes);
  cudaError_t e =
      cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<std::min(L.num_sms, std::max(n_kv, 1)), kBwdThreads, smem, stream>>>(
      mk, mv, mq, mdo, a, n_kv);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_dq_d(const BwdLaunch& L, cudaStream_t stream) {
  CUtensorMap mk, mv, mq, mdo;
  if (!bwd_maps(L, &mk, &mv, &mq, &mdo)) return cudaErrorInvalidValue;
  const BwdArgs a = bwd_args(L);
  const int smem = std::max(QCfg<D>::SMEM, kOneCtaPerSmBytes);
  cudaError_t e =
      cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D><<<L.num_sms, kBwdThreads, smem, stream>>>(mk, mv, mq, mdo, a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv(const BwdLaunch& L, cudaStream_t stream) {
  return L.d == 64 ? launch_dkdv_d<64>(L, stream) : launch_dkdv_d<128>(L, stream);
}

cudaError_t launch_bwd_dq(const BwdLaunch& L, cudaStream_t stream) {
  return L.d == 64 ? launch_dq_d<64>(L, stream) : launch_dq_d<128>(L, stream);
}

cudaError_t launch_bwd_finish(const BwdLaunch& L, cudaStream_t stream) {
  const long long n4 = static_cast<long long>(L.T) * L.H * L.d / 4;
  const unsigned grid =
      static_cast<unsigned>(std::min<long long>((n4 + 255) / 256, 8LL * L.num_sms));
  if (grid == 0) return cudaSuccess;
  bwd_dq_finish_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(L.dq_acc), n4,
                                                 static_cast<uint2*>(L.dq));
  return cudaGetLastError();
}

}  // namespace moba
