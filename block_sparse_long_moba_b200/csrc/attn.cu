// K4 — block-sparse attention on the tcgen05 tensor cores.
//
// Work items (256 query rows each, processed by persistent CTAs, one per SM):
//   routed item  : up to 256 (t, h) rows of one kv head g that routed to one past block b (a list
//                  built by the routing inversion), attending every key of b — the scattered query
//                  rows are gathered into one dense operand [FlashMoBA story, Gather-and-Densify];
//   diagonal item: 256 consecutive tokens of one query head inside their own block, attending the
//                  block's keys up to each query's position (causal inside the current block)
//                  [MoBA paper summary (atlas.scime.ai), "Approach"].
// Each row's result is a normalised partial O_s (bf16) plus its log-sum-exp (fp32), written to the
// row's slot; the merge kernel combines the slots.
//
// An item is two 128-row halves A and B that share every K/V sub-tile. For each 128-key sub-tile:
//   S_x = Q_x K^T        tcgen05.mma kind::f16, M=128 N=128, Q and K K-major (128-byte swizzle),
//                        fp32 accumulator in TMEM
//   P_x = exp2(S_x * scale * log2e - m)   one softmax warpgroup per half, thread = row = TMEM
//                                         lane; P written back over S in TMEM as packed bf16
//   O_x += P_x V         tcgen05.mma with A = P from TMEM and B = V (MN-major) from shared memory
// The MMA issue order S_A(j), PV_B(j-1), S_B(j), PV_A(j) lets one half's softmax overlap the other
// half's matrix products, so the tensor pipe waits on neither softmax alone. The reference max m of
// a row is raised only when the row max grows by more than 2^8 (O and l are then rescaled in
// TMEM); p <= 256 always, and O / l is exact either way. Because PV_x(j-1) is issued before
// S_x(j), the arrival of S_x(j) implies O_x is complete, so a rescale never waits.
//
// Warp roles (384 threads): warp 0 = TMA producer of K/V sub-tiles; warp 1 = TMEM owner and MMA
// issuer (both run converged and let elect.sync pick the issuing lane); warps 2-3 = query rows
// (d = 128: gathered by the TMA unit and by cp.async in parallel; d = 64: see its kernel);
// warps 4-7 = softmax and epilogue of half A; warps 8-11 = the same for half B. Every wait is
// bounded (2 s); on a timeout the kernel raises a CTA abort flag, records a status code, drains
// what it has in flight and returns.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace moba {

// Column pairs (of every 8) whose exp2 runs on the FMA pipe instead of MUFU.EX2, balancing the two.
constexpr int kPolyPairs = 0;
#ifndef MOBA_POLY_PAIRS_PVT
#define MOBA_POLY_PAIRS_PVT 1
#endif
constexpr int kPolyPairsPvt = MOBA_POLY_PAIRS_PVT;

// Partial outputs are written once and read once by the merge: with MOBA_PART_STREAM they are
// stored with the evict-first policy so that they do not push the gathered query rows out of L2.
#ifndef MOBA_PART_STREAM
#define MOBA_PART_STREAM 1
#endif
__device__ __forceinline__ void st_part(uint4* p, uint4 v) {
#if MOBA_PART_STREAM
  __stcs(p, v);
#else
  *p = v;
#endif
}

struct AttnArgs {
  const __nv_bfloat16* q;  // [T, H, D]
  const int4* tiles;       // routed items: {bucket, first entry, rows, -}
  const int* n_routed;     // device count of routed items
  const int* entries;      // partial row of every routed (t, h, slot)
  BlockTables tb;
  __nv_bfloat16* part_o;   // [rows, D]
  float* part_lse;         // [rows]
  int* status;
  int T, H, G, r, topk, NB;
  int b0, nblk, T0;        // chunk: global blocks [b0, b0 + nblk), first token T0
  int P2;                  // ceil(B / 256): diagonal items per (block, head)
  int n_diag;              // P2 * nblk * H diagonal items (some may be empty)
  float scale_log2;        // scale * log2(e)
  unsigned long long wait_ns;  // limit of one pipeline wait (abort drains use kDrainTimeoutNs)
  int diag_stall;              // diagnostics: the MMA issuer first waits on a barrier nobody arrives on
  long long ent_cap, rows_cap, q_rows;  // sizes of entries, partial outputs, q rows (checks)
};

struct __align__(16) Item {
  int kind;  // 0 empty, 1 routed, 2 diagonal, -1 end of the CTA's work
  int g, h, b;
  int key0, klen, nsub;
  int rows;     // valid rows of the item (<= 256)
  int start;    // routed: first entry of the item
  int qtok0;    // diagonal: first query token
  int qoff;     // diagonal: position of the first query inside its block
  int slot;     // diagonal: output slot of the current block
};

__device__ __forceinline__ Item decode_item(const AttnArgs& a, int w, int n_routed) {
  Item it;
  it.kind = 0;
  it.h = 0;
  it.start = 0;
  it.qtok0 = 0;
  it.qoff = 0;
  it.slot = 0;
  if (w < n_routed) {
    const int4 tl = a.tiles[w];
    if (!in_range(tl.x, static_cast<long long>(a.G) * a.NB, a.status) ||
        !in_range(static_cast<long long>(tl.y) + tl.z - 1, a.ent_cap, a.status))
      return it;  // (MOBA_CHECKS) a corrupt work item is skipped by every role alike
    it.kind = 1;
    it.g = tl.x / a.NB;
    it.b = tl.x % a.NB;
    it.start = tl.y;
    it.rows = tl.z;
    it.key0 = a.tb.blk_start[it.b];
    it.klen = a.tb.blk_len[it.b];
    it.nsub = (it.klen + kTile - 1) / kTile;
    return it;
  }
  const int wd = w - n_routed;
  it.h = wd % a.H;
  const int rest = wd / a.H;
  const int bl = rest % a.nblk;
  const int p2 = a.P2 - 1 - rest / a.nblk;  // longest diagonal items first
  it.b = a.b0 + bl;
  const int len = a.tb.blk_len[it.b];
  if (p2 * kItemRows >= len) return it;  // empty (short block)
  it.kind = 2;
  it.g = it.h / a.r;
  it.key0 = a.tb.blk_start[it.b];
  it.qoff = p2 * kItemRows;
  it.rows = min(kItemRows, len - it.qoff);
  it.klen = it.qoff + it.rows;  // keys up to the last query of the item
  it.nsub = (it.klen + kTile - 1) / kTile;
  it.qtok0 = it.key0 + it.qoff;
  const int i = it.b - a.tb.blk_off[a.tb.blk_seq[it.b]];
  it.slot = min(a.topk, i + 1) - 1;
  return it;
}

// ------------------------------------------------------------------------------------------
// Work-item ring. One scheduler warp decodes the CTA's work items 32 at a time (one per lane, so
// the global loads of the routing tiles and block tables of 32 items overlap) and publishes the
// non-empty ones, in order, into a small shared-memory ring, followed by an end marker. Every
// other role copies each item out of the ring and frees the slot at once, so no role waits on a
// global load to learn what to do next.
constexpr int kRing = 16;

struct ItemRing {
  Item items[kRing];
  uint64_t full[kRing], empty[kRing];
};

// Scheduler side: one whole, converged warp. Returns false after an abort.
__device__ __forceinline__ bool ring_produce(ItemRing* ring, const AttnArgs& a, int n_items,
                                             int n_routed, volatile int* abort_flag, int* err,
                                             uint64_t timeout_ns) {
  const int lane = threadIdx.x & 31;
  uint32_t n = 0;
  auto publish = [&](const Item& it, int src) -> bool {
    const uint32_t slot = n % kRing;
    const bool ok = __all_sync(0xffffffffu,
                               mbar_wait_bounded(&ring->empty[slot], ((n / kRing) & 1) ^ 1,
                                                 abort_flag, err, kDevTimeoutAttn, timeout_ns));
    if (!ok) return false;
    if (lane == src) {
      ring->items[slot] = it;
      mbar_arrive(&ring->full[slot]);
    }
    ++n;
    return true;
  };
  const int stride = static_cast<int>(gridDim.x);
  for (int w0 = blockIdx.x; w0 < n_items; w0 += 32 * stride) {
    const int w = w0 + lane * stride;
    Item it;
    it.kind = 0;
    if (w < n_items) it = decode_item(a, w, n_routed);
    uint32_t m = __ballot_sync(0xffffffffu, it.kind != 0);
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      if (!publish(it, src)) return false;
    }
  }
  Item end;
  end.kind = -1;
  end.g = end.h = end.b = end.key0 = end.klen = end.nsub = 0;
  end.rows = end.start = end.qtok0 = end.qoff = end.slot = 0;
  return publish(end, 0);
}

// True if item number `lt` has been published (does not wait).
__device__ __forceinline__ bool ring_ready(ItemRing* ring, uint32_t lt) {
  return mbar_try_wait(&ring->full[lt % kRing], (lt / kRing) & 1);
}

// Consumer side: copies item number `lt` of this CTA and frees its slot.
__device__ __forceinline__ bool ring_consume(ItemRing* ring, uint32_t lt, Item& it,
                                             volatile int* abort_flag, int* err,
                                             uint64_t timeout_ns) {
  const uint32_t slot = lt % kRing;
  if (!mbar_wait_bounded(&ring->full[slot], (lt / kRing) & 1, abort_flag, err, kDevTimeoutAttn,
                         timeout_ns))
    return false;
  it = ring->items[slot];
  mbar_arrive(&ring->empty[slot]);
  return true;
}

// ------------------------------------------------------------------------------------------
// d = 64 kernel.
//
// Roles (384 threads): warp 0 = TMA producer of K/V sub-tiles; warp 1 = TMEM owner and MMA issuer
// (the whole warp runs converged, elect.sync picks the issuing lane); warp 2 = query rows (TMA
// tile loads from the densified rows, or a tile::gather4 gather for diagonal items); warp 3 =
// item scheduler; warps 4-7 = softmax and epilogue of half A; warps 8-11 = half B.
//
// Small blocks make small items (a 128-key block is one sub-tile), so the per-item overheads are
// what this kernel is shaped around:
//   * a routed item's query rows were densified in list order beforehand, so they arrive as one
//     or two 128-row TMA tiles, QB items ahead;
//   * O accumulators are double-buffered in TMEM per half (item parity), and the epilogue of an
//     item runs after the next item's softmax, so it never delays the tensor pipe; each output
//     row leaves a per-warp staging area in shared memory as one 128-byte TMA store;
//   * an item of at most 128 rows (every diagonal item of a 128-key block, the tail item of a
//     routed list) runs on half A only: half B issues no MMA and its warps skip the item.
struct D64Cfg {
  static constexpr int D = 64;
  static constexpr int HALF_BYTES = kTile * D * 2;  // 16 KB: one 128 x 64 bf16 tile
  static constexpr int Q_BYTES = 2 * HALF_BYTES;    // one 256-row item
  static constexpr int QB = 3;                      // Q buffers (items loaded ahead)
  static constexpr int NK = 2, NV = 3;              // K and V ring depths (V is freed later)
  static constexpr int OFF_K = QB * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * HALF_BYTES;
  static constexpr int OFF_EP = OFF_V + NV * HALF_BYTES;  // 8 softmax warps x 32 rows x 128 B
  static constexpr int OFF_BARS = OFF_EP + 8 * 32 * 128;
  static constexpr int SMEM_BYTES = OFF_BARS + 8192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t REGS_CTRL = 72, REGS_SOFTMAX = 216;  // 128*72 + 256*216 = 384*168
  static constexpr uint32_t RING_CONSUMERS = 3 * 32 + 256;       // warps 0-2 and the softmax
  // TMEM columns: S/P of half x at 128 x; O of half x for item parity p at 256 + 64 (2 p + x)
  __host__ __device__ static constexpr uint32_t tm_s(int x) { return 128u * x; }
  __host__ __device__ static constexpr uint32_t tm_o(int x, uint32_t p) {
    return 256u + 64u * (2u * p + static_cast<uint32_t>(x));
  }
};
static_assert(D64Cfg::SMEM_BYTES <= 232448, "shared memory budget of one CTA");

struct D64Bars {
  uint64_t q_full[D64Cfg::QB], q_empty[D64Cfg::QB];
  uint64_t k_full[D64Cfg::NK], k_empty[D64Cfg::NK], v_full[D64Cfg::NV], v_empty[D64Cfg::NV];
  uint64_t s_full[2], p_full[2], o_full[2][2];
  uint64_t drain, never;
  uint32_t tmem_base;
  int abort_flag;
  ItemRing ring;
  // per softmax thread: the previous item's output row (-1 = none), 1 / l and log-sum-exp
  int ep_row[kItemRows];
  float ep_inv[kItemRows], ep_lse[kItemRows];
};
static_assert(sizeof(D64Bars) <= 8192, "barrier block");

__global__ void __launch_bounds__(384, 1)
    attn_kernel_d64(const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v,
                    const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_qd,
                    const __grid_constant__ CUtensorMap map_po, const AttnArgs a) {
  using C = D64Cfg;
  constexpr int D = C::D;
  extern __shared__ __align__(1024) uint8_t smem64[];
  uint8_t* sQ = smem64;
  uint8_t* sK = smem64 + C::OFF_K;
  uint8_t* sV = smem64 + C::OFF_V;
  D64Bars* bars = reinterpret_cast<D64Bars*>(smem64 + C::OFF_BARS);
  ItemRing* ring = &bars->ring;
  volatile int* abort_flag = &bars->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the swizzled layouts assume a 1024-byte aligned base: refuse to run otherwise
  if (smem_u32(smem64) & 1023u) {
    if (tid == 0) atomicCAS(a.status, 0, kDevSmemAlign);
    return;
  }
  if (tid == 0) {
    for (int x = 0; x < C::QB; ++x) {
      mbar_init(&bars->q_full[x], 1);
      mbar_init(&bars->q_empty[x], 1);
    }
    for (int x = 0; x < C::NK; ++x) {
      mbar_init(&bars->k_full[x], 1);
      mbar_init(&bars->k_empty[x], 1);
    }
    for (int x = 0; x < C::NV; ++x) {
      mbar_init(&bars->v_full[x], 1);
      mbar_init(&bars->v_empty[x], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_full[x], 128);
      mbar_init(&bars->o_full[x][0], 1);
      mbar_init(&bars->o_full[x][1], 1);
    }
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->never, 1);
    for (int x = 0; x < kRing; ++x) {
      mbar_init(&ring->full[x], 1);
      mbar_init(&ring->empty[x], C::RING_CONSUMERS);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_qd);
    prefetch_tensormap(&map_po);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_routed = *a.n_routed;
  const int n_items = n_routed + a.n_diag;
  const uint64_t TO = a.wait_ns;
  int* err = a.status;
  auto pop = [&](uint32_t lt, Item& it) -> bool {
    return ring_consume(ring, lt, it, abort_flag, err, TO);
  };

  if (warp < 4) {
    regs_dec<C::REGS_CTRL>();
    if (warp == 0) {
      // -------------------------------------------------------------- TMA producer (K, V)
      uint32_t J = 0, issued_k = 0, issued_v = 0;
      bool ok = true;
      for (uint32_t lt = 0;; ++lt) {
        Item it;
        ok = __all_sync(0xffffffffu, pop(lt, it));
        if (!ok || it.kind < 0) break;
        for (int j = 0; j < it.nsub; ++j, ++J) {
          const int sk = J % C::NK, sv = J % C::NV;
          const int tok = it.key0 + j * kTile;
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->k_empty[sk], ((J / C::NK) & 1) ^ 1,
                                                         abort_flag, err, kDevTimeoutAttn, TO));
          if (!ok) break;
          mbar_arrive_expect_tx_elect(&bars->k_full[sk], C::HALF_BYTES);
          tma_load_3d_elect(sK + sk * C::HALF_BYTES, &map_k, &bars->k_full[sk], 0, it.g, tok);
          ++issued_k;
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->v_empty[sv], ((J / C::NV) & 1) ^ 1,
                                                         abort_flag, err, kDevTimeoutAttn, TO));
          if (!ok) break;
          mbar_arrive_expect_tx_elect(&bars->v_full[sv], C::HALF_BYTES);
          tma_load_3d_elect(sV + sv * C::HALF_BYTES, &map_v, &bars->v_full[sv], 0, it.g, tok);
          ++issued_v;
        }
        if (!ok) break;
      }
      if (!ok) {
        // after an abort, let the loads still in flight land before the CTA exits (bounded)
        volatile int no_abort = 0;
        for (uint32_t x = 0; x < static_cast<uint32_t>(C::NK) && x < issued_k; ++x) {
          const uint32_t Jx = issued_k - 1 - x;
          mbar_wait_bounded(&bars->k_full[Jx % C::NK], (Jx / C::NK) & 1, &no_abort, err, kDevDrainTimeout,
                            kDrainTimeoutNs);
        }
        for (uint32_t x = 0; x < static_cast<uint32_t>(C::NV) && x < issued_v; ++x) {
          const uint32_t Jx = issued_v - 1 - x;
          mbar_wait_bounded(&bars->v_full[Jx % C::NV], (Jx / C::NV) & 1, &no_abort, err, kDevDrainTimeout,
                            kDrainTimeoutNs);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      uint32_t J = 0;                // K/V sub-tiles consumed
      uint32_t cs[2] = {0u, 0u};     // sub-tiles processed by each half (s_full / p_full phase)
      uint32_t ci[2] = {0u, 0u};     // items processed by each half (O buffer, o_full)
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu,
                          mbar_wait_bounded(bar, parity, abort_flag, err, kDevTimeoutAttn, TO));
      };
      auto issue_s = [&](int half, uint32_t qb, int sk) {
        const uint64_t ad = smem_desc_sw128(sQa + qb * C::Q_BYTES + half * C::HALF_BYTES, 16, 1024);
        const uint64_t bd = smem_desc_sw128(sKa + sk * C::HALF_BYTES, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ss_elect(tmem + C::tm_s(half), desc_advance(ad, ks * 32), desc_advance(bd, ks * 32),
                       IDESC_QK, ks > 0 ? 1u : 0u);
        mma_commit_elect(&bars->s_full[half]);
      };
      // O_x += P_x V_sv for the half's sub-tile number c of its item number item
      auto issue_pv = [&](int half, int sv, uint32_t c, uint32_t item, bool first, bool last,
                          bool free_v) -> bool {
        if (!wait(&bars->p_full[half], c & 1)) return false;
        tc_fence_after();
        const uint32_t t_o = tmem + C::tm_o(half, item & 1);
        const uint32_t t_p = tmem + C::tm_s(half);
        const uint64_t bd = smem_desc_sw128(sVa + sv * C::HALF_BYTES, 16384, 1024);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_ts_elect(t_o, t_p + ks * 8, desc_advance(bd, ks * 2048), IDESC_PV,
                       (first && ks == 0) ? 0u : 1u);
        if (free_v) mma_commit_elect(&bars->v_empty[sv]);
        if (last) mma_commit_elect(&bars->o_full[half][item & 1]);
        return true;
      };
      // PV of half B is issued one step late, after the next S of half A (ping-pong)
      bool pend = false, pend_first = false, pend_last = false;
      int pend_sv = 0;
      uint32_t pend_c = 0, pend_item = 0;
      if (a.diag_stall) ok = wait(&bars->never, 0);  // runs out: the whole CTA takes its abort path
      for (uint32_t lt = 0; ok; ++lt) {
        Item it;
        ok = __all_sync(0xffffffffu, pop(lt, it));
        if (!ok || it.kind < 0) break;
        const bool hasB = it.rows > kTile;
        const uint32_t qb = lt % C::QB;
        ok = wait(&bars->q_full[qb], (lt / C::QB) & 1);
        if (!ok) break;
        tc_fence_after();
        for (int j = 0; j < it.nsub; ++j, ++J) {
          const int sk = J % C::NK, sv = J % C::NV;
          ok = wait(&bars->k_full[sk], (J / C::NK) & 1);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, qb, sk);
          if (pend) {
            pend = false;
            ok = issue_pv(1, pend_sv, pend_c, pend_item, pend_first, pend_last, true);
            if (!ok) break;
          }
          if (hasB) issue_s(1, qb, sk);
          mma_commit_elect(&bars->k_empty[sk]);
          if (j == it.nsub - 1) mma_commit_elect(&bars->q_empty[qb]);
          ok = wait(&bars->v_full[sv], (J / C::NV) & 1);
          if (!ok) break;
          ok = issue_pv(0, sv, cs[0], ci[0], j == 0, j == it.nsub - 1, !hasB);
          if (!ok) break;
          ++cs[0];
          if (hasB) {
            pend = true;
            pend_sv = sv;
            pend_c = cs[1]++;
            pend_item = ci[1];
            pend_first = (j == 0);
            pend_last = (j == it.nsub - 1);
          }
        }
        if (!ok) break;
        ++ci[0];
        if (hasB) ++ci[1];
      }
      if (ok && pend) ok = issue_pv(1, pend_sv, pend_c, pend_item, pend_first, pend_last, true);
      if (!ok) {
        // after an abort, wait (bounded) until the MMAs already issued have finished with TMEM
        volatile int no_abort = 0;
        mma_commit_elect(&bars->drain);
        mbar_wait_bounded(&bars->drain, 0, &no_abort, err, kDevDrainTimeout, kDrainTimeoutNs);
      }
    } else if (warp == 2) {
      // ------------------------------------------------------------------ Q rows
      // A routed item's query rows were copied in entry order into one dense array (densify), so
      // they arrive as one or two 128-row tiles on the TMA unit. A
      // diagonal item's rows (consecutive tokens of one head, H rows apart) are gathered on the
      // TMA unit: each lane gathers rows 4 lane .. 4 lane + 3 with one tile::gather4 copy (four
      // 128-byte rows, swizzled into the layout the MMA reads). Lane 0 posts the item's bytes on
      // q_full first, so the warp never waits for the data.
      bool ok = true;
      uint32_t issued = 0;
      for (uint32_t lt = 0; ok; ++lt) {
        Item cur;
        ok = __all_sync(0xffffffffu, pop(lt, cur));
        if (!ok || cur.kind < 0) break;
        const uint32_t qb = lt % C::QB;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->q_empty[qb], ((lt / C::QB) & 1) ^ 1,
                                                       abort_flag, err, kDevTimeoutAttn, TO));
        if (!ok) break;
        const bool hasB = cur.rows > kTile;
        uint8_t* dst = sQ + qb * C::Q_BYTES;
        if (cur.kind == 1) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&bars->q_full[qb], (hasB ? 2 : 1) * C::HALF_BYTES);
            tma_load_2d(dst, &map_qd, &bars->q_full[qb], 0, cur.start);
            if (hasB)
              tma_load_2d(dst + C::HALF_BYTES, &map_qd, &bars->q_full[qb], 0, cur.start + kTile);
          }
        } else {
          // query row (t * H + h) of item row m; padding rows repeat a valid row (their results
          // are never written)
          int y[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const int m = (x >> 2) * kTile + 4 * lane + (x & 3);
            y[x] = (cur.qtok0 + (m < cur.rows ? m : 0)) * a.H + cur.h;
          }
          if (lane == 0)
            mbar_arrive_expect_tx(&bars->q_full[qb], (hasB ? 2 : 1) * C::HALF_BYTES);
          __syncwarp();
          tma_gather4(dst + lane * 512, &map_q, &bars->q_full[qb], 0, y[0], y[1], y[2], y[3]);
          if (hasB)
            tma_gather4(dst + C::HALF_BYTES + lane * 512, &map_q, &bars->q_full[qb], 0, y[4],
                        y[5], y[6], y[7]);
        }
        __syncwarp();
        ++issued;
      }
      if (!ok) {
        // after an abort, let the loads still in flight land before the CTA exits (bounded)
        volatile int no_abort = 0;
        for (uint32_t x = 0; x < static_cast<uint32_t>(C::QB) && x < issued; ++x) {
          const uint32_t l = issued - 1 - x;
          mbar_wait_bounded(&bars->q_full[l % C::QB], (l / C::QB) & 1, &no_abort, err, kDevDrainTimeout,
                            kDrainTimeoutNs);
        }
      }
    } else {
      // ------------------------------------------------------------------ item scheduler
      ring_produce(ring, a, n_items, n_routed, abort_flag, err, TO);
    }
  } else {
    regs_inc<C::REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax + epilogue
    const int half = (warp >= 8) ? 1 : 0;
    const int row = tid - 128 - half * 128;  // TMEM lane / row inside the half
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_off + C::tm_s(half);
    const float sl2 = a.scale_log2;
    const int q = half * kTile + row;        // row inside the 256-row item
    uint32_t cs = 0, ci = 0;  // sub-tiles and items processed by this half
    bool ok = true;
    // epilogue of this half's item number ci - 1 (its output row, 1 / l and log-sum-exp are
    // parked in shared memory meanwhile, to keep registers for the softmax)
    auto epilogue = [&]() -> bool {
      const uint32_t pci = ci - 1, ob = pci & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars->o_full[half][ob], (pci >> 1) & 1,
                                                     abort_flag, err, kDevTimeoutAttn, TO)))
        return false;
      tc_fence_after();
      const uint32_t t_o = tmem + lane_off + C::tm_o(half, ob);
      const int prev_prow = bars->ep_row[q];
      const float inv = bars->ep_inv[q];
      // each thread's output row goes through shared memory (its 16-byte chunk c at chunk
      // c ^ (r % 8) of the warp's staging row r: the 128-byte swizzle, conflict-free) and leaves
      // as one 128-byte TMA store, so the warp does not wait for its stores; the staging row is
      // reused one item later, once that store has read it
      uint8_t* ep = smem64 + C::OFF_EP + (warp - 4) * (32 * 128);
      bulk_wait_group_read<0>();
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t orr[32];
        tmem_ld32(t_o + c0, orr);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) reg_fence(orr[x]);
#pragma unroll
        for (int x = 0; x < 4; ++x)
          *reinterpret_cast<uint4*>(ep + lane * 128 + (((c0 / 8 + x) ^ (lane & 7)) * 16)) = make_uint4(
              pack_bf16x2(__uint_as_float(orr[8 * x + 0]) * inv, __uint_as_float(orr[8 * x + 1]) * inv),
              pack_bf16x2(__uint_as_float(orr[8 * x + 2]) * inv, __uint_as_float(orr[8 * x + 3]) * inv),
              pack_bf16x2(__uint_as_float(orr[8 * x + 4]) * inv, __uint_as_float(orr[8 * x + 5]) * inv),
              pack_bf16x2(__uint_as_float(orr[8 * x + 6]) * inv, __uint_as_float(orr[8 * x + 7]) * inv));
      }
      tc_fence_before();
      if (prev_prow >= 0 && in_range(prev_prow, a.rows_cap, a.status)) {
        fence_proxy_async_smem();  // the staging row is visible to the TMA unit
        tma_store_2d(&map_po, ep + lane * 128, 0, prev_prow);
        bulk_commit_group();
      }
      if (prev_prow >= 0 && in_range(prev_prow, a.rows_cap, a.status))
        a.part_lse[prev_prow] = bars->ep_lse[q];
      return true;
    };
    for (uint32_t lt = 0;; ++lt) {
      Item it;
      ok = __all_sync(0xffffffffu, pop(lt, it));
      if (!ok || it.kind < 0) break;
      if (half == 1 && it.rows <= kTile) continue;  // half B idle for this item
      const int r_item = q;
      const bool valid = r_item < it.rows;
      int prow = 0, limit;
      if (it.kind == 1) {
        if (valid) prow = __ldg(a.entries + it.start + r_item);
        limit = it.klen;
      } else {
        const int t = it.qtok0 + r_item;
        prow = ((t - a.T0) * a.H + it.h) * a.topk + it.slot;
        limit = valid ? it.qoff + r_item + 1 : 1;
      }
      const uint32_t t_o = tmem + lane_off + C::tm_o(half, ci & 1);
      float m_ref = -INFINITY, l_sum = 0.f;
      for (int j = 0; j < it.nsub; ++j, ++cs) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->s_full[half], cs & 1, abort_flag,
                                                       err, kDevTimeoutAttn, TO));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128];
        const int lim = limit - j * kTile;  // valid columns: c < lim
        // load S in two halves so the second TMEM load overlaps the first half's max
        tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 64; ++c) reg_fence(sr[c]);
        tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        if (lim < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) mx8[x] = __uint_as_float(sr[x]);
#pragma unroll
        for (int c = 8; c < 64; c += 8) {
#pragma unroll
          for (int x = 0; x < 8; ++x) mx8[x] = fmaxf(mx8[x], __uint_as_float(sr[c + x]));
        }
        tmem_wait_ld();
#pragma unroll
        for (int c = 64; c < 128; ++c) reg_fence(sr[c]);
        if (lim < kTile) {
#pragma unroll
          for (int c = 64; c < 128; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int c = 64; c < 128; c += 8) {
#pragma unroll
          for (int x = 0; x < 8; ++x) mx8[x] = fmaxf(mx8[x], __uint_as_float(sr[c + x]));
        }
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float mxs = mx * sl2;
        // raise the reference max only when it grew by more than 2^8 (rare); tcgen05.ld/st are
        // warp-collective, so the O rescale runs for the whole warp (alpha = 1 where not needed)
        const bool need = mxs > m_ref + 8.f;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_ref - mxs);  // 0 on the first sub-tile
          l_sum *= alpha;
          m_ref = mxs;
        }
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O_x holds sub-tiles < j and is complete (its last PV was issued before this S)
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t orr[32];
            tmem_ld32(t_o + c0, orr);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) reg_fence(orr[x]);
#pragma unroll
            for (int x = 0; x < 32; ++x) orr[x] = __float_as_uint(__uint_as_float(orr[x]) * alpha);
            tmem_st32(t_o + c0, orr);
          }
          tmem_wait_st();
        }
        const float neg = -m_ref;
        float ps8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) ps8[x] = 0.f;
#pragma unroll
        for (int c = 0; c < 128; c += 16) {
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float t0 = fmaf(__uint_as_float(sr[c + 2 * x]), sl2, neg);
            const float t1 = fmaf(__uint_as_float(sr[c + 2 * x + 1]), sl2, neg);
            const bool poly = x >= 8 - kPolyPairs;
            const float p0 = poly ? exp2_poly(t0) : ex2_approx(t0);
            const float p1 = poly ? exp2_poly(t1) : ex2_approx(t1);
            ps8[x] += p0 + p1;
            sr[(c >> 1) + x] = pack_bf16x2(p0, p1);  // packed in place: index <= c + 2x
          }
        }
        l_sum += ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
        tmem_st32(t_s + 0, *reinterpret_cast<const uint32_t(*)[32]>(&sr[0]));
        tmem_st32(t_s + 32, *reinterpret_cast<const uint32_t(*)[32]>(&sr[32]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[half]);
      }
      if (!ok) break;
      // the previous item's O is complete by now (its last PV preceded this item's S)
      if (ci > 0) {
        ok = epilogue();
        if (!ok) break;
      }
      bars->ep_row[q] = valid ? prow : -1;
      bars->ep_inv[q] = 1.f / l_sum;
      bars->ep_lse[q] = (m_ref + __log2f(l_sum)) * 0.69314718055994531f;
      ++ci;
    }
    if (ok && ci > 0) ok = epilogue();
    bulk_wait_all();  // this thread's output stores are complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------
// d = 128: P staged in shared memory, PV computed transposed for both halves at once.
//
// On B200 a 128 x N x 16 tcgen05.mma issued back to back costs ~100 cycles for any N <= 128
// (measured) but reaches the nominal 128 cycles at N = 256. Here the two 128-row halves A and B
// keep their own S = Q K^T (M = 128, N = 128 keys), but P = exp(...) goes to shared memory and
// the value product is computed as O^T = V^T P^T: M = d = 128, N = 256 queries (both halves),
// K = 128 keys — eight full-rate instructions per sub-tile instead of sixteen half-rate ones.
// Since P no longer aliases S in tensor memory, S_x(j+1) is issued as soon as the softmax has
// read S_x(j), so QK^T of the next sub-tile overlaps this sub-tile's softmax.
// Tensor memory: S_A [0,128), S_B [128,256), O^T [256,512) (lanes = d, columns = the 256 rows).
// O^T columns are rescaled (rarely) by the warpgroup that owns those rows, between PV(j-1) and
// PV(j); the epilogue normalises O^T by l, transposes it through shared memory and writes rows.
struct PvtCfg {
  static constexpr int D = 128;
  static constexpr int HALF_BYTES = kTile * D * 2;  // 32 KB
  static constexpr int Q_BYTES = 2 * HALF_BYTES;     // 64 KB (one buffer)
  static constexpr int NSTK = 2;                     // K ring
  static constexpr int P_BYTES = 2 * HALF_BYTES;     // 256 rows x 128 keys bf16
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + NSTK * HALF_BYTES;
  static constexpr int OFF_P = OFF_V + HALF_BYTES;   // single V stage
  static constexpr int OFF_ALPHA = OFF_P + P_BYTES;  // float[256]
  static constexpr int OFF_INVL = OFF_ALPHA + 1024;  // float[256]
  static constexpr int OFF_BARS = OFF_INVL + 1024;
  static constexpr int SMEM_BYTES = OFF_BARS + 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_OT = 256;
  // the MMA issuer needs ~100 registers; 128*104 + 256*200 = 384*168 leaves nothing spilled
  static constexpr uint32_t REGS_CTRL = 104, REGS_SOFTMAX = 200;
  __host__ __device__ static constexpr uint32_t tm_s(int x) { return 128u * x; }
};
static_assert(PvtCfg::SMEM_BYTES <= 232448, "shared memory budget of one CTA");

struct PvtBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[2], k_empty[2], v_full, v_empty;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, pv_done;
  uint64_t drain, never;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(PvtBars) <= 256, "barrier block");

// Walks the 128-key sub-tiles of this CTA's work items in order (empty items skipped).
struct SubTileCursor {
  int w = -1, j = 0;
  Item it;
  __device__ __forceinline__ bool next(const AttnArgs& a, int n_items, int n_routed) {
    if (w >= 0 && ++j < it.nsub) return true;
    for (w = (w < 0) ? static_cast<int>(blockIdx.x) : w + static_cast<int>(gridDim.x); w < n_items;
         w += gridDim.x) {
      it = decode_item(a, w, n_routed);
      if (it.kind != 0) {
        j = 0;
        return true;
      }
    }
    return false;
  }
};

// Byte offset of element (row, col) in a 256-row operand stored as two 64-column blocks of
// 256 x 128 bytes with the 128-byte swizzle (the P layout, also used to stage O rows).
__device__ __forceinline__ uint32_t p_offset(uint32_t row, uint32_t col) {
  return (col >> 6) * 32768u + sw128_offset(row, col & 63u);
}

__global__ void __launch_bounds__(384, 1)
    attn_kernel_pvt(const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v,
                    const __grid_constant__ CUtensorMap map_q, const AttnArgs a) {
  using C = PvtCfg;
  constexpr int D = C::D;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sP = smem + C::OFF_P;
  float* s_alpha = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
  float* s_invl = reinterpret_cast<float*>(smem + C::OFF_INVL);
  PvtBars* bars = reinterpret_cast<PvtBars*>(smem + C::OFF_BARS);
  volatile int* abort_flag = &bars->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the swizzled layouts assume a 1024-byte aligned base: refuse to run otherwise
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicCAS(a.status, 0, kDevSmemAlign);
    return;
  }
  if (tid == 0) {
    mbar_init(&bars->q_full, 33);  // warp 2 lane 0 (TMA bytes) + the 32 lanes of warp 3
    mbar_init(&bars->q_empty, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->k_full[x], 1);
      mbar_init(&bars->k_empty[x], 1);
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->s_free[x], 128);
    }
    mbar_init(&bars->v_full, 1);
    mbar_init(&bars->v_empty, 1);
    mbar_init(&bars->p_full, 256);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->never, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
    prefetch_tensormap(&map_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_routed = *a.n_routed;
  const int n_items = n_routed + a.n_diag;
  const uint64_t TO = a.wait_ns;
  int* err = a.status;

  if (warp < 4) {
    regs_dec<C::REGS_CTRL>();
    if (warp == 0) {
      // -------------------------------------------------------------- TMA producer (K, V)
      // K runs up to two sub-tiles ahead of V: the next QK^T is issued before this PV, and the
      // single V stage only frees up when the previous PV has completed.
      SubTileCursor ck, cv;
      bool hk = ck.next(a, n_items, n_routed), hv = cv.next(a, n_items, n_routed);
      uint32_t JK = 0, JV = 0;
      bool ok = true;
      while (ok && (hk || hv)) {
        if (hk && (JK < JV + 2 || !hv)) {
          const int st = JK & 1;
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->k_empty[st], ((JK >> 1) & 1) ^ 1,
                                                         abort_flag, err, kDevTimeoutAttn, TO));
          if (!ok) break;
          const int tok = ck.it.key0 + ck.j * kTile;
          mbar_arrive_expect_tx_elect(&bars->k_full[st], C::HALF_BYTES);
          tma_load_3d_elect(sK + st * C::HALF_BYTES, &map_k, &bars->k_full[st], 0, ck.it.g, tok);
          tma_load_3d_elect(sK + st * C::HALF_BYTES + 16384, &map_k, &bars->k_full[st], 64,
                            ck.it.g, tok);
          ++JK;
          hk = ck.next(a, n_items, n_routed);
        } else {
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->v_empty, (JV & 1) ^ 1, abort_flag,
                                                         err, kDevTimeoutAttn, TO));
          if (!ok) break;
          const int tok = cv.it.key0 + cv.j * kTile;
          mbar_arrive_expect_tx_elect(&bars->v_full, C::HALF_BYTES);
          tma_load_3d_elect(sV, &map_v, &bars->v_full, 0, cv.it.g, tok);
          tma_load_3d_elect(sV + 16384, &map_v, &bars->v_full, 64, cv.it.g, tok);
          ++JV;
          hv = cv.next(a, n_items, n_routed);
        }
      }
      if (!ok) {
        volatile int no_abort = 0;
        for (uint32_t x = 0; x < 2; ++x) {
          if (JK > x) {
            const uint32_t Jx = JK - 1 - x;
            mbar_wait_bounded(&bars->k_full[Jx & 1], (Jx >> 1) & 1, &no_abort, err,
                              kDevDrainTimeout, kDrainTimeoutNs);
          }
        }
        if (JV > 0)
          mbar_wait_bounded(&bars->v_full, (JV - 1) & 1, &no_abort, err, kDevDrainTimeout,
                            kDrainTimeoutNs);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_PVT = idesc_bf16_f32(128, 256, 1, 0);  // A = V^T (MN-major)
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV), sPa = smem_u32(sP);
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu,
                          mbar_wait_bounded(bar, parity, abort_flag, err, kDevTimeoutAttn, TO));
      };
      // S_x(J) = Q_x K_J^T; the S_x buffer must have been read by the softmax of sub-tile J-1
      auto issue_s = [&](int x, uint32_t J) -> bool {
        if (J > 0 && !wait(&bars->s_free[x], (J - 1) & 1)) return false;
        tc_fence_after();
        const int st = J & 1;
        const uint64_t ad = smem_desc_sw128(sQa + x * C::HALF_BYTES, 16, 1024);
        const uint64_t bd = smem_desc_sw128(sKa + st * C::HALF_BYTES, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_ss_elect(tmem + C::tm_s(x), desc_advance(ad, off), desc_advance(bd, off), IDESC_QK,
                       ks > 0 ? 1u : 0u);
        }
        mma_commit_elect(&bars->s_full[x]);
        return true;
      };
      auto issue_s_pair = [&](uint32_t J, bool last_of_item) -> bool {
        if (!wait(&bars->k_full[J & 1], (J >> 1) & 1)) return false;
        tc_fence_after();
        if (!issue_s(0, J) || !issue_s(1, J)) return false;
        mma_commit_elect(&bars->k_empty[J & 1]);
        if (last_of_item) mma_commit_elect(&bars->q_empty);
        return true;
      };
      // O^T (+)= V_J^T P_J^T for both halves
      auto issue_pvt = [&](uint32_t J, bool first) -> bool {
        if (!wait(&bars->v_full, J & 1)) return false;
        if (!wait(&bars->p_full, J & 1)) return false;
        tc_fence_after();
        const uint64_t ad = smem_desc_sw128(sVa, 16384, 1024);
        const uint64_t bd = smem_desc_sw128(sPa, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_ss_elect(tmem + C::TM_OT, desc_advance(ad, ks * 2048),
                       desc_advance(bd, (ks >> 2) * 32768 + (ks & 3) * 32), IDESC_PVT,
                       (first && ks == 0) ? 0u : 1u);
        mma_commit_elect(&bars->v_empty);
        mma_commit_elect(&bars->pv_done);
        return true;
      };
      uint32_t J = 0, lt = 0;
      if (a.diag_stall) ok = wait(&bars->never, 0);  // runs out: the whole CTA takes its abort path
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        const Item it = decode_item(a, w, n_routed);
        if (it.kind == 0) continue;
        ok = wait(&bars->q_full, lt & 1);
        if (!ok) break;
        tc_fence_after();
        ok = issue_s_pair(J, it.nsub == 1);
        for (int j = 0; j < it.nsub && ok; ++j) {
          if (j + 1 < it.nsub) {
            ok = issue_s_pair(J + j + 1, j + 1 == it.nsub - 1);
            if (!ok) break;
          }
          ok = issue_pvt(J + j, j == 0);
        }
        J += it.nsub;
        ++lt;
      }
      if (!ok) {
        volatile int no_abort = 0;
        mma_commit_elect(&bars->drain);
        mbar_wait_bounded(&bars->drain, 0, &no_abort, err, kDevDrainTimeout, kDrainTimeoutNs);
      }
    } else {
      // ------------------------------------------------------------------ Q row gather
      // Two warps, two copy engines in parallel. Warp 2 gathers half A (rows 0..127) on the TMA
      // unit with tile::gather4 (four rows x one 64-column box per copy, two boxes per row; lane 0
      // posts the bytes on q_full first). Warp 3 copies half B (rows 128..255) with 16-byte
      // cp.async, two 256-byte rows per warp instruction, and arrives once its copies have landed.
      // Each lane reads the routing entries of four consecutive rows (coalesced over the warp);
      // warp 3 hands the query-row index of a row to the 16 lanes that copy it by shuffles.
      const int half = warp - 2;  // 0: rows 0..127 (TMA), 1: rows 128..255 (cp.async)
      uint32_t lt = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        const Item it = decode_item(a, w, n_routed);
        if (it.kind == 0) continue;
        int qr4[4];  // query rows (t * H + h) of item rows half * 128 + 4 lane + r, -1 = padding
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int m = half * kTile + 4 * lane + r;
          qr4[r] = (it.kind == 1 && m < it.rows) ? __ldg(a.entries + it.start + m) : 0;
        }
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->q_empty, (lt & 1) ^ 1, abort_flag,
                                                       err, kDevTimeoutAttn, TO));
        if (!ok) break;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int m = half * kTile + 4 * lane + r;
          // half A padding repeats a valid row for the TMA (never written back); half B padding
          // is zero-filled by cp.async
          qr4[r] = (m >= it.rows && half == 1) ? -1
                   : (it.kind == 1) ? (m < it.rows ? a.T0 * a.H + qr4[r] / a.topk : a.T0 * a.H)
                                    : (it.qtok0 + (m < it.rows ? m : 0)) * a.H + it.h;
        }
        if (half == 0) {
          if (lane == 0) mbar_arrive_expect_tx(&bars->q_full, C::HALF_BYTES);
          __syncwarp();
          uint8_t* dst = sQ + lane * 512;
          tma_gather4(dst, &map_q, &bars->q_full, 0, qr4[0], qr4[1], qr4[2], qr4[3]);
          tma_gather4(dst + 16384, &map_q, &bars->q_full, 64, qr4[0], qr4[1], qr4[2], qr4[3]);
        } else {
          const uint32_t dst0 = smem_u32(sQ) + C::HALF_BYTES;
          const int c = lane & 15, r0 = lane >> 4;
          // instruction i copies rows 2 i and 2 i + 1 of half B, held by lane i / 2 in its
          // registers 2 (i % 2) and 2 (i % 2) + 1
#pragma unroll 8
          for (int i = 0; i < kTile / 2; ++i) {
            const int va = __shfl_sync(0xffffffffu, qr4[2 * (i & 1)], i >> 1);
            const int vb = __shfl_sync(0xffffffffu, qr4[2 * (i & 1) + 1], i >> 1);
            const int qr = r0 ? vb : va;
            const int m = 2 * i + r0;
            const bool take = qr >= 0 && in_range(qr, a.q_rows, a.status);
            const __nv_bfloat16* src = take ? a.q + static_cast<size_t>(qr) * D + c * 8 : a.q;
            cp_async_16(dst0 + (c >> 3) * 16384 + sw128_offset(m, (c & 7) * 8), src,
                        take ? 16u : 0u);
          }
          cp_async_wait_all();
          fence_proxy_async_smem();
          mbar_arrive(&bars->q_full);
        }
        ++lt;
      }
      if (half == 1) cp_async_wait_all();
      if (!ok && half == 0 && lt > 0) {
        // after an abort, let the gathers still in flight land before the CTA exits (bounded)
        volatile int no_abort = 0;
        mbar_wait_bounded(&bars->q_full, (lt - 1) & 1, &no_abort, err, kDevDrainTimeout,
                          kDrainTimeoutNs);
      }
    }
  } else {
    regs_inc<C::REGS_SOFTMAX>();
    // -------------------------------------------------------------- softmax + epilogue
    const int half = (warp >= 8) ? 1 : 0;
    const int row = tid - 128 - half * 128;          // TMEM lane; row of this half
    const int q = half * kTile + row;                 // row of the 256-row item
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_off + C::tm_s(half);
    const uint32_t t_ot = tmem + lane_off + C::TM_OT + half * kTile;  // this half's O^T columns
    const uint32_t bar_id = 1 + half;                 // named barrier of this warpgroup
    const float sl2 = a.scale_log2;
    uint32_t J = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const Item it = decode_item(a, w, n_routed);
      if (it.kind == 0) continue;
      const bool valid = q < it.rows;
      int prow = 0, limit;
      if (it.kind == 1) {
        if (valid) prow = __ldg(a.entries + it.start + q);
        limit = it.klen;
      } else {
        const int t = it.qtok0 + q;
        prow = ((t - a.T0) * a.H + it.h) * a.topk + it.slot;
        limit = valid ? it.qoff + q + 1 : 1;
      }
      float m_ref = -INFINITY, l_sum = 0.f;
      for (int j = 0; j < it.nsub; ++j, ++J) {
        // A warp whose wait gives up does not leave on its own: the four warps of this half meet
        // at named barriers, so the decision to leave is taken by all of them together at the
        // next barrier (a warp that left alone would strand the other three there). Until then
        // a warp that gave up computes on whatever S holds; its results are never used.
        bool wok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->s_full[half], J & 1,
                                                             abort_flag, err, kDevTimeoutAttn, TO));
        tc_fence_after();
        uint32_t sr[128];
        const int lim = limit - j * kTile;
        tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 128; ++c) reg_fence(sr[c]);
        tc_fence_before();
        mbar_arrive(&bars->s_free[half]);  // S_x may now be overwritten by the next QK^T
        if (lim < kTile) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        // row max with three-input max: 8 running maxima over 16 columns per step
        float mx8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x)
          mx8[x] = fmax3(__uint_as_float(sr[x]), __uint_as_float(sr[8 + x]),
                         __uint_as_float(sr[16 + x]));
#pragma unroll
        for (int c = 24; c < 120; c += 16) {
#pragma unroll
          for (int x = 0; x < 8; ++x)
            mx8[x] = fmax3(mx8[x], __uint_as_float(sr[c + x]), __uint_as_float(sr[c + 8 + x]));
        }
#pragma unroll
        for (int x = 0; x < 8; ++x) mx8[x] = fmaxf(mx8[x], __uint_as_float(sr[120 + x]));
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const float mxs = mx * sl2;
        const bool need = mxs > m_ref + 8.f;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_ref - mxs);
          l_sum *= alpha;
          m_ref = mxs;
        }
        const float neg = -m_ref;
        // p = exp2(s * scale * log2e - m) for a column pair, packed to bf16x2; pair sums in f32x2
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        auto exp_pair = [&](int c) -> uint32_t {
          float t0, t1;
          fma2(t0, t1, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]), sl2, sl2, neg, neg);
          // kPolyPairsPvt of every 8 column pairs run on the FMA pipe, the rest on MUFU.EX2
          float p0, p1;
          if (((c >> 1) & 7) >= 8 - kPolyPairsPvt) {
            exp2_poly2(t0, t1, p0, p1);
          } else {
            p0 = ex2_approx(t0);
            p1 = ex2_approx(t1);
          }
          const int x = (c >> 1) & 3;
          add2(sa[x], sb[x], sa[x], sb[x], p0, p1);
          return pack_bf16x2(p0, p1);
        };
        // columns 0..63 first, held packed in sr[0..31]
#pragma unroll
        for (int c = 0; c < 64; c += 2) sr[c >> 1] = exp_pair(c);
        // P(J) reuses the shared P tile: PV(J-1) must be complete (it also fixes O^T for a rescale)
        if (J > 0 && wok)
          wok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->pv_done, (J - 1) & 1,
                                                          abort_flag, err, kDevTimeoutAttn, TO));
        s_alpha[q] = alpha;
        // one barrier answers both questions in the common case: nothing to rescale, no abort
        if (named_bar_or(bar_id, 128, !wok || (need && j > 0))) {
          ok = named_bar_and(bar_id, 128, wok);  // the same answer for every warp of the half
          if (!ok) break;
          // some row of this half raised its max: scale this half's O^T columns (lane = d)
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < kTile; c0 += 32) {
            uint32_t orr[32];
            tmem_ld32(t_ot + c0, orr);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) reg_fence(orr[x]);
#pragma unroll
            for (int x = 0; x < 32; ++x)
              orr[x] = __float_as_uint(__uint_as_float(orr[x]) * s_alpha[half * kTile + c0 + x]);
            tmem_st32(t_ot + c0, orr);
          }
          tmem_wait_st();
        }
        // P row q -> shared memory (K-major, 128-byte swizzle); the second half of the row is
        // computed and stored chunk by chunk so the stores overlap the exponentials
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(sP + p_offset(q, c * 8)) =
              make_uint4(sr[4 * c], sr[4 * c + 1], sr[4 * c + 2], sr[4 * c + 3]);
#pragma unroll
        for (int c = 64; c < 128; c += 8) {
          const uint32_t w0 = exp_pair(c), w1 = exp_pair(c + 2), w2 = exp_pair(c + 4),
                         w3 = exp_pair(c + 6);
          *reinterpret_cast<uint4*>(sP + p_offset(q, c)) = make_uint4(w0, w1, w2, w3);
        }
        l_sum += ((sa[0] + sb[0]) + (sa[1] + sb[1])) + ((sa[2] + sb[2]) + (sa[3] + sb[3]));
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->p_full);
      }
      if (!ok) break;
      // ---- epilogue: O = O^T / l, transposed through the (now idle) P tile
      const bool eok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->pv_done, (J - 1) & 1,
                                                                 abort_flag, err, kDevTimeoutAttn,
                                                                 TO));
      tc_fence_after();
      s_invl[q] = (valid && l_sum > 0.f) ? 1.f / l_sum : 0.f;
      ok = named_bar_and(bar_id, 128, eok);  // leave together or not at all
      if (!ok) break;
      // thread `row` holds O^T lane d = row: columns are this half's 128 query rows
#pragma unroll 1
      for (int c0 = 0; c0 < kTile; c0 += 32) {
        uint32_t orr[32];
        tmem_ld32(t_ot + c0, orr);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) reg_fence(orr[x]);
#pragma unroll
        for (int x4 = 0; x4 < 32; x4 += 4) {
          const int qq = half * kTile + c0 + x4;
          const float4 il = *reinterpret_cast<const float4*>(s_invl + qq);
          const float ilv[4] = {il.x, il.y, il.z, il.w};
#pragma unroll
          for (int x = 0; x < 4; ++x)
            *reinterpret_cast<__nv_bfloat16*>(sP + p_offset(qq + x, row)) =
                __float2bfloat16_rn(__uint_as_float(orr[x4 + x]) * ilv[x]);
        }
      }
      named_bar_sync(bar_id, 128);
      // each warp writes its own 32 rows, two whole 256-byte rows per instruction (16 lanes each)
      {
        const int wrow0 = half * kTile + (warp & 3) * 32;
        const int my_prow = valid ? prow : -1;
        const int c = lane & 15;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int rr = 2 * i + (lane >> 4);
          const int pr = __shfl_sync(0xffffffffu, my_prow, rr);
          const uint4 v = *reinterpret_cast<const uint4*>(sP + p_offset(wrow0 + rr, c * 8));
          if (pr >= 0 && in_range(pr, a.rows_cap, a.status))
            st_part(reinterpret_cast<uint4*>(a.part_o + static_cast<size_t>(pr) * D) + c, v);
        }
      }
      if (valid && in_range(prow, a.rows_cap, a.status))
        a.part_lse[prow] = (m_ref + __log2f(l_sum)) * 0.69314718055994531f;
      // the P tile rows of this half are rewritten only by this warpgroup, after this point
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------- host side

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [T, G, D] bf16 -> 3-D map (D, G, T), box (64, 1, 128), 128-byte swizzle, zero fill out of range.
bool make_kv_map(CUtensorMap* map, const void* base, int T, int G, int D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(G),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(G) * D * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kTile)};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [T * H, D] bf16 query rows -> 2-D map (D, T * H), box (64, 1): one row per box, as the row
// gather (tile::gather4) requires; 128-byte swizzle.
bool make_q_rows_map(CUtensorMap* map, const void* base, long long rows, int D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, 64] bf16 dense query rows -> 2-D map (64, rows), box (64, 128), 128-byte swizzle, zero
// fill past the last row.
static bool make_q_dense_map(CUtensorMap* map, const void* base, long long rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kTile)};
  cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_attention(const AttnLaunch& L, cudaStream_t stream) {
  CUtensorMap mk, mv, mq, mqd, mpo;
  if (!make_kv_map(&mk, L.k, L.T, L.G, L.d) || !make_kv_map(&mv, L.v, L.T, L.G, L.d))
    return cudaErrorInvalidValue;
  if (!make_q_rows_map(&mq, L.q, static_cast<long long>(L.T) * L.H, L.d))
    return cudaErrorInvalidValue;
  if (L.d == 64 && (!L.qdense || !make_q_dense_map(&mqd, L.qdense, L.qdense_rows) ||
                    !make_q_rows_map(&mpo, L.part_o, L.rows_cap, 64)))
    return cudaErrorInvalidValue;
  AttnArgs a;
  a.q = static_cast<const __nv_bfloat16*>(L.q);
  a.tiles = L.tiles;
  a.n_routed = L.n_routed;
  a.entries = L.entries;
  a.tb = L.tb;
  a.part_o = static_cast<__nv_bfloat16*>(L.part_o);
  a.part_lse = L.part_lse;
  a.status = L.status;
  a.T = L.T;
  a.H = L.H;
  a.G = L.G;
  a.r = L.H / L.G;
  a.topk = L.topk;
  a.NB = L.NB;
  a.b0 = L.b0;
  a.nblk = L.nblk;
  a.T0 = L.T0;
  a.P2 = (L.B + kItemRows - 1) / kItemRows;
  a.n_diag = a.P2 * L.nblk * L.H;
  a.scale_log2 = L.scale * 1.4426950408889634f;
  a.wait_ns = L.wait_ns > 0 ? L.wait_ns : kWaitTimeoutNs;
  a.diag_stall = L.diag_stall;
  a.ent_cap = L.qdense_rows;
  a.rows_cap = L.rows_cap;
  a.q_rows = static_cast<long long>(L.T) * L.H;
  const int grid = L.grid > 0 ? L.grid : 1;
  // setmaxnreg.inc would wait forever if the launch had fewer registers than the split assumes
  {
    cudaFuncAttributes fa;
    cudaError_t e = (L.d == 64) ? cudaFuncGetAttributes(&fa, attn_kernel_d64)
                                : cudaFuncGetAttributes(&fa, attn_kernel_pvt);
    if (e != cudaSuccess) return e;
    const int need = (L.d == 64) ? 128 * D64Cfg::REGS_CTRL + 256 * D64Cfg::REGS_SOFTMAX
                                 : 128 * PvtCfg::REGS_CTRL + 256 * PvtCfg::REGS_SOFTMAX;
    if (fa.numRegs * 384 < need) return cudaErrorInvalidConfiguration;
  }
  if (L.d == 64) {
    const int smem = D64Cfg::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(attn_kernel_d64, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_kernel_d64<<<grid, 384, smem, stream>>>(mk, mv, mq, mqd, mpo, a);
  } else {
    const int smem = PvtCfg::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(attn_kernel_pvt, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_kernel_pvt<<<grid, 384, smem, stream>>>(mk, mv, mq, a);
  }
  return cudaGetLastError();
}

}  // namespace moba
