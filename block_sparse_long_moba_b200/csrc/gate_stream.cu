// K2, streaming form — parameter-less causal top-k gate [MoBA paper summary (atlas.scime.ai),
// "Approach"; MoBA README, "Parameter-less Gating Mechanism"] for sequences of at most 257 blocks
// (every past block id fits in 8 bits; the Llama-3.1-8B shapes at 128K and 1M tokens with
// 4096-key blocks have 32 and 256).
//
// The gate reads every query row once, so it is bound by the HBM stream of Q. The kernel is
// organised around keeping that stream full:
//   * each CTA owns one contiguous range of 128-row query tiles, cut on the host so that the
//     ranges carry equal estimated work (a tile costs a Q load plus a selection that grows with
//     its number of past blocks);
//   * a producer warp walks the range and keeps NQ query tiles in flight on the TMA unit (NQ is
//     sized from the shared memory left after the centroids: 6 at 32 blocks, 2 at 256, d = 128);
//   * the fp32 centroids of the sequence's past blocks are split once per (sequence, kv head)
//     into two bf16 terms (c = c_hi + c_lo, ~2^-17 relative) by two converter warps;
//   * one MMA warp computes S[128, n] = Q . (C_hi + C_lo)^T for all n past blocks of a tile in one
//     tcgen05 accumulation (N = n rounded up to 16, at most 256; every product exact, fp32 sums);
//   * two selection warpgroups take alternate tiles, one thread per query row (= TMEM lane):
//     the first 32 scores are sorted by a bitonic network into the row's top list, later columns
//     are filtered against the list's current k-th entry and inserted only when they beat it.
// The T x NB score matrix never exists in memory [FlashMoBA story, FlashTopK].
//
// Keys: a score's order-preserving 32-bit image with its low 8 bits replaced by 255 - block, so
// keys are distinct, a larger key is a better score and equal truncated scores rank the lower
// block first; the truncation reorders only scores within 2^-15 (relative) of each other.
//
// Every wait is bounded (2 s); on a timeout the CTA raises an abort flag, records a status code,
// drains what it has in flight and returns.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace moba {

namespace {

constexpr int kGsRing = 16;     // published tiles
constexpr int kGsSegRing = 4;   // published (sequence, kv head) segments
constexpr int kGsMaxQ = 8;      // query tile buffers
constexpr int kGsCapMax = 256;  // centroid rows resident (past blocks of one sequence)

struct GsTile {
  int kind;     // 1 scored tile; 2 run of rows whose selection is fixed (few causal blocks or
                // topk == 1); -1 end
  int seg_ord;  // ordinal of the tile's segment within this CTA
  int i, h, t0, rows;  // block, head, first token, tokens (<= 128 when scored)
  int qslot;
};

struct GsSeg {
  int kind;  // 1, or -1 end
  int g, base, nrows;
};

struct GsBars {
  uint64_t q_full[kGsMaxQ], q_empty[kGsMaxQ];
  uint64_t t_full[kGsRing], t_empty[kGsRing];
  uint64_t s_full[kGsSegRing], s_empty[kGsSegRing];
  uint64_t mma_done[2], tm_free[2];
  uint64_t c_full, c_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  GsTile tiles[kGsRing];
  GsSeg segs[kGsSegRing];
};
constexpr int kGsBarsBytes = 2048;
static_assert(sizeof(GsBars) <= kGsBarsBytes, "barrier block");

// Order-preserving map of fp32 to uint32 (a larger float gives a larger unsigned) and back.
__device__ __forceinline__ uint32_t gs_f2ord(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float gs_ord2f(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// Bitonic sorting network over 32 registers, descending (static indices only).
__device__ __forceinline__ void bitonic32_desc(uint32_t (&k)[32]) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int a = 0; a < 32; ++a) {
        const int b = a ^ stride;
        if (b > a) {
          const uint32_t hi = max(k[a], k[b]), lo = min(k[a], k[b]);
          if ((a & size) == 0) {
            k[a] = hi;
            k[b] = lo;
          } else {
            k[a] = lo;
            k[b] = hi;
          }
        }
      }
    }
  }
}

// Bitonic sorting network over N (a power of two) keys, descending (static indices only).
template <int N>
__device__ __forceinline__ void bitonic_desc(uint32_t (&k)[N]) {
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int a = 0; a < N; ++a) {
        const int b = a ^ stride;
        if (b > a) {
          const uint32_t hi = max(k[a], k[b]), lo = min(k[a], k[b]);
          if ((a & size) == 0 || size == N) {
            k[a] = hi;
            k[b] = lo;
          } else {
            k[a] = lo;
            k[b] = hi;
          }
        }
      }
    }
  }
}

// Sorts a bitonic sequence of N keys descending (the merge stages of the network).
template <int N>
__device__ __forceinline__ void bitonic_clean_desc(uint32_t (&k)[N]) {
#pragma unroll
  for (int stride = N >> 1; stride > 0; stride >>= 1) {
#pragma unroll
    for (int a = 0; a < N; ++a) {
      const int b = a ^ stride;
      if (b > a) {
        const uint32_t hi = max(k[a], k[b]), lo = min(k[a], k[b]);
        k[a] = hi;
        k[b] = lo;
      }
    }
  }
}

// Bitonic sorting network over N (a power of two) int registers, ascending.
template <int N>
__device__ __forceinline__ void bitonic_asc(int (&k)[N]) {
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int a = 0; a < N; ++a) {
        const int b = a ^ stride;
        if (b > a) {
          const int lo = min(k[a], k[b]), hi = max(k[a], k[b]);
          if ((a & size) == 0) {
            k[a] = lo;
            k[b] = hi;
          } else {
            k[a] = hi;
            k[b] = lo;
          }
        }
      }
    }
  }
}

__device__ __forceinline__ uint32_t gs_key(float s, int j) {
  return (gs_f2ord(s) & ~0xffu) | static_cast<uint32_t>(255 - j);
}

struct GsArgs {
  const float* cents;  // [NB, G, D] fp32
  const int32_t* cu;   // [nseq + 1]
  int32_t* idx;        // [H, T, topk]
  int* status;
  int nseq, T, H, G, B, topk;
  int nq, cap;  // query buffers; centroid rows (multiple of 16, <= 256)
  uint32_t off_c, off_stage, off_bars;
};

}  // namespace

template <int D, int KCAP>
__global__ void __launch_bounds__(384, 1)
    gate_stream_kernel(const __grid_constant__ CUtensorMap map_q, const GsArgs a,
                       const __grid_constant__ GateSched sched) {
  constexpr int NCB = D / 64;
  constexpr uint32_t Q_BYTES = kTile * D * 2;
  extern __shared__ __align__(1024) uint8_t smem_gs[];
  GsBars* bars = reinterpret_cast<GsBars*>(smem_gs + a.off_bars);
  volatile int* abort_flag = &bars->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem_gs) & 1023u) {  // the swizzled layouts need a 1024-byte aligned base
    if (tid == 0 && a.status) atomicCAS(a.status, 0, kDevTimeoutAttn);
    return;
  }
  if (tid == 0) {
    for (int x = 0; x < kGsMaxQ; ++x) {
      mbar_init(&bars->q_full[x], 1);
      mbar_init(&bars->q_empty[x], 1);
    }
    for (int x = 0; x < kGsRing; ++x) {
      mbar_init(&bars->t_full[x], 1);
      mbar_init(&bars->t_empty[x], 5);  // the MMA warp + the four warps of one selection group
    }
    for (int x = 0; x < kGsSegRing; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->s_empty[x], 2);  // the two converter warps
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->mma_done[x], 1);
      mbar_init(&bars->tm_free[x], 4);
    }
    mbar_init(&bars->c_full, 64);
    mbar_init(&bars->c_empty, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == 0) prefetch_tensormap(&map_q);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint64_t TO = kWaitTimeoutNs;
  int* err = a.status;
  const int r = a.H / a.G;
  const int ksel = a.topk - 1;
  const int cta = static_cast<int>(blockIdx.x);
  uint8_t* sC = smem_gs + a.off_c;

  if (warp == 0) {
    // ------------------------------------------------------------ producer: tiles and Q loads
    if (lane == 0) {
      bool ok = true;
      int seg = sched.seg[cta], i = sched.blk[cta], p = sched.pos[cta], base = sched.base[cta];
      int left = sched.count[cta];
      int s = seg / a.G, g = seg % a.G;
      int seq0 = a.cu[s], L = a.cu[s + 1] - seq0, nb = blocks_of(L, a.B);
      int cur_seg = -1, seg_ord = -1;
      uint32_t k = 0, nq = 0, nsg = 0;
      auto publish_seg = [&](const GsSeg& e) -> bool {
        const uint32_t sl = nsg % kGsSegRing;
        if (!mbar_wait_bounded(&bars->s_empty[sl], ((nsg / kGsSegRing) & 1) ^ 1, abort_flag, err,
                               kDevTimeoutAttn, TO))
          return false;
        bars->segs[sl] = e;
        mbar_arrive(&bars->s_full[sl]);
        ++nsg;
        return true;
      };
      auto publish_tile = [&](const GsTile& e) -> bool {
        const uint32_t sl = k % kGsRing;
        if (!mbar_wait_bounded(&bars->t_empty[sl], ((k / kGsRing) & 1) ^ 1, abort_flag, err,
                               kDevTimeoutAttn, TO))
          return false;
        bars->tiles[sl] = e;
        mbar_arrive(&bars->t_full[sl]);
        ++k;
        return true;
      };
      while (ok && left > 0) {
        const int blen = min(a.B, L - i * a.B);
        const int ntt = (blen + kTile - 1) / kTile;
        const int hh = p / ntt, tt = p % ntt;
        GsTile e;
        e.i = i;
        e.h = g * r + hh;
        e.t0 = seq0 + i * a.B + tt * kTile;
        e.kind = (ksel > 0 && i > ksel) ? 1 : 2;
        // a fixed-selection entry covers this head's remaining pieces of the block in the range
        const int run = (e.kind == 1) ? 1 : min(left, ntt - tt);
        e.rows = min(run * kTile, blen - tt * kTile);
        if (seg != cur_seg) {
          GsSeg sg;
          sg.kind = 1;
          sg.g = g;
          sg.base = base;
          sg.nrows = min(max(nb - 1, 0), a.cap);
          ok = publish_seg(sg);
          if (!ok) break;
          cur_seg = seg;
          ++seg_ord;
        }
        e.seg_ord = seg_ord;
        e.qslot = -1;
        if (e.kind == 1) {
          const uint32_t sl = nq % static_cast<uint32_t>(a.nq);
          ok = mbar_wait_bounded(&bars->q_empty[sl], ((nq / a.nq) & 1) ^ 1, abort_flag, err,
                                 kDevTimeoutAttn, TO);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->q_full[sl], Q_BYTES);
#pragma unroll
          for (int c = 0; c < NCB; ++c)
            tma_load_3d(smem_gs + sl * Q_BYTES + c * 16384, &map_q, &bars->q_full[sl], c * 64,
                        e.h, e.t0);
          e.qslot = static_cast<int>(sl);
          ++nq;
        }
        ok = publish_tile(e);
        if (!ok) break;
        left -= run;
        // next tile: heads and 128-row pieces of this block, then the next block, then the next
        // kv head of the sequence, then the next non-empty sequence
        p += run;
        if (p == r * ntt) {
          p = 0;
          if (++i == nb) {
            i = 0;
            if (++g == a.G) {
              g = 0;
              base += nb;
              do {
                ++s;
                if (s >= a.nseq) break;
                seq0 = a.cu[s];
                L = a.cu[s + 1] - seq0;
                nb = blocks_of(L, a.B);
              } while (nb == 0);
            }
            seg = s * a.G + g;
          }
        }
      }
      if (ok) {
        GsTile end;
        end.kind = -1;
        end.seg_ord = end.i = end.h = end.t0 = end.rows = 0;
        end.qslot = -1;
        ok = publish_tile(end) && publish_tile(end);  // one end marker for each selection group
      }
      if (ok) {
        GsSeg end;
        end.kind = -1;
        end.g = end.base = end.nrows = 0;
        ok = publish_seg(end);
      }
      if (!ok) {
        // after an abort, let the query loads still in flight land (bounded)
        volatile int no_abort = 0;
        for (uint32_t x = 0; x < static_cast<uint32_t>(a.nq) && x < nq; ++x) {
          const uint32_t l = nq - 1 - x;
          mbar_wait_bounded(&bars->q_full[l % a.nq], (l / a.nq) & 1, &no_abort, nullptr, 0,
                            TO / 4);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------ MMA issuer
    bool ok = true;
    uint32_t nq = 0, nsc[2] = {0u, 0u};
    int cur_ord = -1;
    const uint32_t sCa = smem_u32(sC);
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu,
                        mbar_wait_bounded(bar, parity, abort_flag, err, kDevTimeoutAttn, TO));
    };
    for (uint32_t k = 0;; ++k) {
      const uint32_t sl = k % kGsRing;
      ok = wait(&bars->t_full[sl], (k / kGsRing) & 1);
      if (!ok) break;
      const GsTile e = bars->tiles[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->t_empty[sl]);
      if (e.kind < 0) break;
      if (e.seg_ord != cur_ord) {
        // the previous segment's products are done with the centroid buffer once they complete
        if (cur_ord >= 0) mma_commit_elect(&bars->c_empty);
        cur_ord = e.seg_ord;
        ok = wait(&bars->c_full, static_cast<uint32_t>(cur_ord) & 1);
        if (!ok) break;
        tc_fence_after();
      }
      if (e.kind != 1) continue;
      const int w = static_cast<int>(k & 1);
      if (nsc[w] > 0) {
        ok = wait(&bars->tm_free[w], (nsc[w] - 1) & 1);
        if (!ok) break;
      }
      const uint32_t qs = nq % static_cast<uint32_t>(a.nq);
      ok = wait(&bars->q_full[qs], (nq / a.nq) & 1);
      if (!ok) break;
      tc_fence_after();
      const int nmma = (e.i + 15) & ~15;  // past blocks, rounded up to the MMA's N granule
      const uint32_t idesc = idesc_bf16_f32(128, nmma, 0, 0);
      const uint32_t qa = smem_u32(smem_gs + qs * Q_BYTES);
#pragma unroll
      for (int sp = 0; sp < 2; ++sp) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t aoff = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t boff = static_cast<uint32_t>((sp * NCB + (ks >> 2)) * a.cap * 128 +
                                                      (ks & 3) * 32);
          mma_ss_elect(tmem + static_cast<uint32_t>(w * 256), smem_desc_sw128(qa + aoff, 16, 1024),
                       smem_desc_sw128(sCa + boff, 16, 1024), idesc,
                       (sp > 0 || ks > 0) ? 1u : 0u);
        }
      }
      mma_commit_elect(&bars->mma_done[w]);
      mma_commit_elect(&bars->q_empty[qs]);
      ++nsc[w];
      ++nq;
    }
    if (!ok) {
      volatile int no_abort = 0;
      mma_commit_elect(&bars->drain);
      mbar_wait_bounded(&bars->drain, 0, &no_abort, nullptr, 0, TO / 4);
    }
  } else if (warp < 4) {
    // ------------------------------------------- converters: fp32 centroids -> bf16 hi + lo
    const int ct = tid - 64;
    bool ok = true;
    for (uint32_t m = 0;; ++m) {
      const uint32_t sl = m % kGsSegRing;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->s_full[sl], (m / kGsSegRing) & 1,
                                                     abort_flag, err, kDevTimeoutAttn, TO));
      if (!ok) break;
      const GsSeg sg = bars->segs[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_empty[sl]);
      if (sg.kind < 0) break;
      if (m > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->c_empty, (m - 1) & 1, abort_flag,
                                                       err, kDevTimeoutAttn, TO));
        if (!ok) break;
      }
      const int nrows16 = (sg.nrows + 15) & ~15;
      const int ngroups = nrows16 * (D / 8);
      for (int e0 = ct; e0 < ngroups; e0 += 8 * 64) {
        float4 va[8], vb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = e0 + u * 64;
          const int rr = e / (D / 8), c8 = (e % (D / 8)) * 8;
          va[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          vb[u] = va[u];
          if (e < ngroups && rr < sg.nrows) {
            const float4* src = reinterpret_cast<const float4*>(
                a.cents + (static_cast<size_t>(sg.base + rr) * a.G + sg.g) * D + c8);
            va[u] = __ldg(src);
            vb[u] = __ldg(src + 1);
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = e0 + u * 64;
          if (e >= ngroups) break;
          const int rr = e / (D / 8), c8 = (e % (D / 8)) * 8;
          const float x[8] = {va[u].x, va[u].y, va[u].z, va[u].w,
                              vb[u].x, vb[u].y, vb[u].z, vb[u].w};
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * q]);
            const __nv_bfloat16 h1 = __float2bfloat16_rn(x[2 * q + 1]);
            const __nv_bfloat16 l0 = __float2bfloat16_rn(x[2 * q] - __bfloat162float(h0));
            const __nv_bfloat16 l1 = __float2bfloat16_rn(x[2 * q + 1] - __bfloat162float(h1));
            hw[q] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                    (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
            lw[q] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                    (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
          }
          const uint32_t o = static_cast<uint32_t>((c8 >> 6) * a.cap * 128) +
                             sw128_offset(static_cast<uint32_t>(rr), static_cast<uint32_t>(c8 & 63));
          *reinterpret_cast<uint4*>(sC + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sC + static_cast<uint32_t>(NCB * a.cap * 128) + o) =
              make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->c_full);
    }
  } else {
    // ------------------------------------------------------ selection: one thread per row
    const int w = (warp - 4) >> 2;  // selection group
    const int row = tid - 128 - w * 128;
    const uint32_t tb = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                        static_cast<uint32_t>(w * 256);
    float* stage = reinterpret_cast<float*>(smem_gs + a.off_stage) + w * 32 * 128;  // [x][row]
    bool ok = true;
    uint32_t j = 0;  // scored tiles of this group
    for (uint32_t k = static_cast<uint32_t>(w);; k += 2) {
      const uint32_t sl = k % kGsRing;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->t_full[sl], (k / kGsRing) & 1,
                                                     abort_flag, err, kDevTimeoutAttn, TO));
      if (!ok) break;
      const GsTile e = bars->tiles[sl];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->t_empty[sl]);
      if (e.kind < 0) break;
      if (e.kind == 2) {
        // few causal blocks or topk == 1: every row of the run has the same fixed selection
        // (blocks 0..i, -1 padded; or just i), and the run's rows are contiguous in idx, so the
        // group writes them as one coalesced span
        int32_t* span = a.idx + (static_cast<size_t>(e.h) * a.T + e.t0) * a.topk;
        const int total = e.rows * a.topk;
        const int step = 128 % a.topk;
        int x = row % a.topk;
        for (int el = row; el < total; el += 128) {
          span[el] = (ksel == 0) ? e.i : (x <= e.i ? x : -1);
          x += step;
          if (x >= a.topk) x -= a.topk;
        }
        continue;
      }
      int32_t* out = a.idx + (static_cast<size_t>(e.h) * a.T + e.t0 + row) * a.topk;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->mma_done[w], j & 1, abort_flag, err,
                                                     kDevTimeoutAttn, TO));
      if (!ok) break;
      tc_fence_after();
      const int n = e.i;  // past blocks 0 .. i - 1
      // the first 32 columns, sorted: the row's initial top list
      uint32_t kk[KCAP];
      {
        uint32_t sr[32];
        tmem_ld32(tb, sr);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) reg_fence(sr[x]);
#pragma unroll
        for (int x = 0; x < 32; ++x) sr[x] = (x < n) ? gs_key(__uint_as_float(sr[x]), x) : 0u;
        if (KCAP <= 16) {
          // the 16 best of 32: both halves sorted, the larger of a[x] and b[15 - x] (a bitonic
          // sequence holding the 16 largest keys) sorted again; a row of at most 16 columns
          // only needs its first half sorted
          uint32_t ha[16], hb[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            ha[x] = sr[x];
            hb[x] = sr[16 + x];
          }
          bitonic_desc<16>(ha);
          if (n > 16) {
            bitonic_desc<16>(hb);
#pragma unroll
            for (int x = 0; x < 16; ++x) ha[x] = max(ha[x], hb[15 - x]);
            bitonic_clean_desc<16>(ha);
          }
#pragma unroll
          for (int x = 0; x < KCAP; ++x) kk[x] = ha[x];
        } else {
          bitonic32_desc(sr);
#pragma unroll
          for (int x = 0; x < KCAP; ++x) kk[x] = sr[x];
        }
      }
      for (int cc = 32; cc < n; cc += 32) {
        uint32_t sr[32];
        tmem_ld32(tb + static_cast<uint32_t>(cc), sr);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) reg_fence(sr[x]);
        // the list's ksel-th key (the list is sorted, so the least of its first ksel keys); a
        // column can beat it only with a score at least this
        uint32_t tk = 0xffffffffu;
#pragma unroll
        for (int x = 0; x < KCAP; ++x)
          if (x < ksel) tk = min(tk, kk[x]);
        const float thr = gs_ord2f(tk & ~0xffu);
        uint32_t mask = 0;
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (cc + x < n && __uint_as_float(sr[x]) >= thr) mask |= 1u << x;
        if (__any_sync(0xffffffffu, mask != 0)) {
#pragma unroll
          for (int x = 0; x < 32; ++x) stage[x * 128 + row] = __uint_as_float(sr[x]);
          while (__any_sync(0xffffffffu, mask != 0)) {
            if (mask) {
              const int x = __ffs(mask) - 1;
              mask &= mask - 1;
              const uint32_t key = gs_key(stage[x * 128 + row], cc + x);
#pragma unroll
              for (int y = KCAP - 1; y > 0; --y) kk[y] = max(kk[y], min(kk[y - 1], key));
              kk[0] = max(kk[0], key);
            }
          }
          __syncwarp();
        }
      }
      // this group's TMEM region is free for its next tile
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->tm_free[w]);
      ++j;
      if (row < e.rows) {
        int sel[KCAP];
#pragma unroll
        for (int x = 0; x < KCAP; ++x)
          sel[x] = (x < ksel) ? 255 - static_cast<int>(kk[x] & 0xffu) : 0x7fffffff;
        bitonic_asc<KCAP>(sel);
#pragma unroll
        for (int x = 0; x < KCAP; ++x)
          if (x < ksel) out[x] = sel[x];
        out[ksel] = e.i;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

namespace {

typedef CUresult (*EncodeTiledFnS)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_q_map_stream(CUtensorMap* map, const void* q, int T, int H, int D) {
  static EncodeTiledFnS fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFnS>(p);
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kTile)};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int KCAP>
cudaError_t launch_gs(const CUtensorMap& mq, const GsArgs& a, const GateSched& S, int smem,
                      cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(gate_stream_kernel<D, KCAP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gate_stream_kernel<D, KCAP><<<S.n_cta, 384, smem, stream>>>(mq, a, S);
  return cudaGetLastError();
}

}  // namespace

bool gate_stream_supported(int max_nb, int topk) {
  return max_nb - 1 <= kGsCapMax && topk >= 1 && topk - 1 <= 32;
}

int gate_stream_schedule(const int32_t* cu_host, int nseq, int H, int G, int d, int B, int topk,
                         int num_ctas, GateSched* S) {
  const int r = H / G, ksel = topk - 1;
  // estimated cost of a tile, in bytes of HBM traffic: every tile writes its rows' selections; a
  // scored tile also reads its query rows and selects over i past blocks. The first 32 scores
  // (one sorted chunk) hide under the query load; each further 64 cost about one more query
  // load's worth of issue slots (measured at 256 blocks).
  const double q_bytes = 128.0 * d * 2, out_bytes = 128.0 * topk * 4;
  auto tile_cost = [&](int i) -> double {
    return (ksel > 0 && i > ksel) ? q_bytes + out_bytes + q_bytes * std::max(0, i - 32) / 64.0
                                  : out_bytes;
  };
  double total = 0.0;
  long long n_tiles = 0;
  for (int s = 0; s < nseq; ++s) {
    const int L = cu_host[s + 1] - cu_host[s];
    const int nb = blocks_of(L, B);
    for (int i = 0; i < nb; ++i) {
      const int ntt = (std::min(B, L - i * B) + kTile - 1) / kTile;
      total += static_cast<double>(G) * r * ntt * tile_cost(i);
      n_tiles += static_cast<long long>(G) * r * ntt;
    }
  }
  if (n_tiles == 0) {
    S->n_cta = 0;
    return 0;
  }
  int grid = static_cast<int>(std::min<long long>(std::min(num_ctas, kGateMaxCtas), n_tiles));
  grid = std::max(grid, 1);
  long long start_lin[kGateMaxCtas + 1];
  int next = 0;
  double cum = 0.0;
  long long lin = 0;
  int base = 0;
  for (int s = 0; s < nseq && next < grid; ++s) {
    const int L = cu_host[s + 1] - cu_host[s];
    const int nb = blocks_of(L, B);
    for (int g = 0; g < G && next < grid; ++g) {
      for (int i = 0; i < nb && next < grid; ++i) {
        const int ntt = (std::min(B, L - i * B) + kTile - 1) / kTile;
        const int nt = r * ntt;
        const double ci = tile_cost(i);
        while (next < grid) {
          const double bound = total * next / grid;
          if (cum + nt * ci <= bound) break;
          const double need = (bound - cum) / ci;
          const int p = need <= 0.0 ? 0 : static_cast<int>(std::ceil(need - 1e-9));
          if (p >= nt) break;
          S->seg[next] = s * G + g;
          S->blk[next] = i;
          S->pos[next] = p;
          S->base[next] = base;
          start_lin[next] = lin + p;
          ++next;
        }
        cum += nt * ci;
        lin += nt;
      }
    }
    base += nb;
  }
  // CTAs whose share fell past the last tile get nothing
  for (int c = next; c < grid; ++c) {
    S->seg[c] = S->blk[c] = S->pos[c] = S->base[c] = 0;
    start_lin[c] = n_tiles;
  }
  start_lin[grid] = n_tiles;
  for (int c = 0; c < grid; ++c)
    S->count[c] = static_cast<int>(std::max<long long>(0, start_lin[c + 1] - start_lin[c]));
  // a CTA with no tiles must not start from an arbitrary cursor: point it at tile 0 of seq 0
  S->n_cta = grid;
  return grid;
}

cudaError_t launch_gate_stream(const void* q, const float* cents, const int32_t* cu_dev,
                               const int32_t* cu_host, int nseq, int max_nb, int T, int H, int G,
                               int d, int B, int topk, int32_t* idx, int* status, int num_sms,
                               cudaStream_t stream) {
  if (!gate_stream_supported(max_nb, topk)) return cudaErrorInvalidValue;
  static thread_local GateSched S;
  if (gate_stream_schedule(cu_host, nseq, H, G, d, B, topk, num_sms, &S) == 0) return cudaSuccess;
  CUtensorMap mq;
  if (!make_q_map_stream(&mq, q, T, H, d)) return cudaErrorInvalidValue;
  GsArgs a;
  a.cents = cents;
  a.cu = cu_dev;
  a.idx = idx;
  a.status = status;
  a.nseq = nseq;
  a.T = T;
  a.H = H;
  a.G = G;
  a.B = B;
  a.topk = topk;
  a.cap = std::max(16, ((max_nb - 1) + 15) & ~15);
  const uint32_t q_bytes = static_cast<uint32_t>(kTile * d * 2);
  const uint32_t c_bytes = static_cast<uint32_t>(2 * (d / 64) * a.cap * 128);
  const uint32_t st_bytes = (max_nb - 1 > 32) ? 2u * 32u * 128u * 4u : 0u;
  const uint32_t budget = 232448u;
  const uint32_t fixed = c_bytes + st_bytes + kGsBarsBytes;
  if (fixed + q_bytes > budget) return cudaErrorInvalidValue;
  a.nq = static_cast<int>(std::min<uint32_t>(kGsMaxQ, (budget - fixed) / q_bytes));
  a.off_c = static_cast<uint32_t>(a.nq) * q_bytes;
  a.off_stage = a.off_c + c_bytes;
  a.off_bars = a.off_stage + st_bytes;
  const int smem = static_cast<int>(a.off_bars + kGsBarsBytes);
  const int ksel = topk - 1;
  if (d == 64) {
    if (ksel <= 4) return launch_gs<64, 4>(mq, a, S, smem, stream);
    if (ksel <= 8) return launch_gs<64, 8>(mq, a, S, smem, stream);
    if (ksel <= 16) return launch_gs<64, 16>(mq, a, S, smem, stream);
    return launch_gs<64, 32>(mq, a, S, smem, stream);
  }
  if (ksel <= 4) return launch_gs<128, 4>(mq, a, S, smem, stream);
  if (ksel <= 8) return launch_gs<128, 8>(mq, a, S, smem, stream);
  if (ksel <= 16) return launch_gs<128, 16>(mq, a, S, smem, stream);
  return launch_gs<128, 32>(mq, a, S, smem, stream);
}

}  // namespace moba
