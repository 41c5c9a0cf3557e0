// K2 on the tensor cores, long-sequence form — parameter-less causal top-k gate [MoBA paper
// summary (atlas.scime.ai), "Approach"; MoBA README, "Parameter-less Gating Mechanism"] for
// sequences of more than 257 blocks (the small-block shapes: 512 to 1792 blocks of 128 keys).
//
// Scores of one tile of 128 query rows (128 consecutive tokens of one query head) against the past
// blocks of their sequence are one matrix product on tcgen05:
//   S[128, n] = Q[128, d] . C[n, d]^T,  C = c_hi + c_lo  (two bf16 terms of the fp32 centroids)
// so each fp32 centroid enters with ~2^-17 relative error and every product q * c_part is exact
// in the fp32 accumulator. The T x NB score matrix never exists in memory [FlashMoBA story,
// FlashTopK]: at most 256 scores per row at a time live in tensor memory, and the products are
// recomputed for each pass below (the tensor pipe is otherwise idle here).
//
// Selection, one thread per row (= TMEM lane), in two passes over the row's n scores:
//   1. group maxima over M strided groups (column j in group j mod M, M = 32 or 64); the ksel-th
//      largest group maximum tau is a lower bound of the ksel-th best score, since ksel distinct
//      groups each hold a score >= tau;
//   2. every score >= tau is a candidate (typically ksel + a few) and is appended, with its block,
//      to the row's candidate buffer in shared memory (one predicated 8-byte store per score, no
//      branch; ascending block order); a bitonic sort of the candidate scores gives the exact
//      ksel-th best score tau* and how many selected scores tie with it, the selection (the blocks
//      with score > tau* and the lowest-numbered ones equal to tau*: ties go to the lower block)
//      is marked in a bit mask, and the row is written ascending in 16-byte pieces.
// Each pass costs a compare per score and no per-score list insertion. A row whose candidates
// overflow the buffer (many exactly equal scores) runs a third pass with a running top list.
//
// A CTA holds two warpgroups (one query tile each) and works on one (query blocks, kv head) unit
// at a time: the hi / lo centroids of the unit's past blocks are placed in shared memory once and
// reused by all tiles and passes of the unit when they fit. Inside the forward pass they come
// pre-split from global memory (bulk copies in the swizzled row layout the MMA reads); when they
// do not fit, they stream through a ring of slots, thread 0 issuing the load of a slot's next
// piece as soon as both warpgroups' products have read it. The standalone gate converts the fp32
// centroids itself, chunk by chunk.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace moba {

namespace {

constexpr int kTilesPerUnit = 16;  // query tiles that share one conversion of the centroids

template <int D, int KCAP>
struct GateCfg {
  static constexpr int NCB = D / 64;
  static constexpr int M = (KCAP <= 16) ? 32 : 64;           // groups of pass 1
  static constexpr int CB = (KCAP <= 16) ? 32 : 64;          // candidate slots per row
  static constexpr int Q_BYTES = kTile * D * 2;             // one 128-row query tile
  static constexpr int CAND_BYTES = 2 * CB * 128 * 8;        // [2][CB][128] (fp32 score, int block)
  // centroid rows resident at once (a multiple of 16): what is left of the CTA's shared memory
  static constexpr int CAP = (D == 128) ? (KCAP <= 16 ? 192 : 64) : (KCAP <= 16 ? 512 : 256);
  static constexpr int B_BYTES = 2 * NCB * CAP * 128;        // hi + lo, 128 B per row per block
  static constexpr int OFF_B = 2 * Q_BYTES;                  // one Q buffer per warpgroup
  static constexpr int OFF_STAGE = OFF_B + B_BYTES;          // candidate buffer / staging
  static constexpr int OFF_BARS = OFF_STAGE + CAND_BYTES;
  static constexpr int SMEM_BYTES = OFF_BARS + 384;
  static constexpr int PIECE = 128;                          // MMA N (scores per TMEM buffer)
  // ring mode (past blocks beyond CAP): RS slots of PR centroid rows each, PR a multiple of 16
  static constexpr int PR = CAP >= 256 ? 128 : CAP / 2;
  static constexpr int RS = CAP / PR;
};
static_assert(GateCfg<64, 16>::RS <= 4 && GateCfg<64, 32>::RS <= 4 && GateCfg<128, 16>::RS <= 4 &&
                  GateCfg<128, 32>::RS <= 4 && GateCfg<128, 16>::CAP % GateCfg<128, 16>::PR == 0 &&
                  GateCfg<128, 16>::PR % 16 == 0 && GateCfg<128, 32>::PR % 16 == 0,
              "ring slots");
static_assert(GateCfg<128, 16>::SMEM_BYTES <= 232448 && GateCfg<64, 16>::SMEM_BYTES <= 232448 &&
                  GateCfg<128, 32>::SMEM_BYTES <= 232448 && GateCfg<64, 32>::SMEM_BYTES <= 232448,
              "shared memory budget of one CTA");

struct GateBars {
  uint64_t q_full[2], mma_done[2][2], chunk_full;
  uint64_t slot_full[4], slot_free[4];  // ring mode
  uint32_t tmem_base;
  int abort_flag;
  int red[32];
};

template <int D, int KCAP>
__device__ __forceinline__ uint32_t c_offset(int s, int row, int col) {
  using C = GateCfg<D, KCAP>;
  return static_cast<uint32_t>(s * C::NCB * C::CAP * 128 + (col >> 6) * C::CAP * 128) +
         sw128_offset(row, col & 63);
}

// Running top list of one row (the single-pass selection that rows with overflowing candidate
// buffers fall back to), best first. The first KCAP - ksel places hold sentinels that no score
// displaces, so the last place is always the ksel-th best so far. Equal scores keep the earlier
// (lower) block.
template <int KCAP>
struct TopList {
  float v[KCAP];
  int id[KCAP];
  __device__ __forceinline__ void init(int ksel) {
#pragma unroll
    for (int x = 0; x < KCAP; ++x) {
      v[x] = (x < KCAP - ksel) ? INFINITY : -INFINITY;
      id[x] = 0x7fffffff;
    }
  }
  __device__ __forceinline__ float thr() const { return v[KCAP - 1]; }
  // Inserts (s, j) if it beats the last place. gt[] is monotone (the list is sorted), so position
  // x takes the entry above it when s beats that one, s when s beats only the entry at x, and
  // keeps its entry otherwise: every position is computed independently.
  __device__ __forceinline__ void offer(float s, int j) {
    if (!(s > v[KCAP - 1])) return;
    bool gt[KCAP];
#pragma unroll
    for (int x = 0; x < KCAP; ++x) gt[x] = s > v[x];
#pragma unroll
    for (int x = KCAP - 1; x > 0; --x) {
      v[x] = gt[x - 1] ? v[x - 1] : (gt[x] ? s : v[x]);
      id[x] = gt[x - 1] ? id[x - 1] : (gt[x] ? j : id[x]);
    }
    v[0] = gt[0] ? s : v[0];
    id[0] = gt[0] ? j : id[0];
  }
};

// Bitonic sorting network over N (a power of two) fp32 registers, descending.
template <int N>
__device__ __forceinline__ void bitonic_desc_f(float (&k)[N]) {
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int a = 0; a < N; ++a) {
        const int b = a ^ stride;
        if (b > a) {
          const float hi = fmaxf(k[a], k[b]), lo = fminf(k[a], k[b]);
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

// The smallest of the first ksel entries of a descending list: its ksel-th largest value.
template <int N>
__device__ __forceinline__ float kth_of_sorted(const float (&k)[N], int ksel) {
  float t = INFINITY;
#pragma unroll
  for (int x = 0; x < N; ++x)
    if (x < ksel) t = fminf(t, k[x]);
  return t;
}

}  // namespace

template <int D, int KCAP>
__global__ void __launch_bounds__(256, 1)
    gate_tc_kernel(const __grid_constant__ CUtensorMap map_q, const float* __restrict__ cents,
                   const int32_t* __restrict__ cu, int nseq, int max_nb, int T, int H, int G,
                   int B, int topk, int32_t* __restrict__ idx, int* __restrict__ status,
                   const uint8_t* __restrict__ split, int nb_pad) {
  using C = GateCfg<D, KCAP>;
  constexpr int M = C::M, CB = C::CB;
  constexpr int STEP = (M == 32) ? 64 : 32;
  extern __shared__ __align__(1024) uint8_t smem[];
  GateBars* bars = reinterpret_cast<GateBars*>(smem + C::OFF_BARS);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int wg = tid >> 7, row = tid & 127;
  if (smem_u32(smem) & 1023u) {  // swizzled layouts need a 1024-byte aligned base
    if (tid == 0 && status) atomicCAS(status, 0, kDevTimeoutAttn);
    return;
  }
  volatile int* abort_flag = &bars->abort_flag;
  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->q_full[x], 1);
      mbar_init(&bars->mma_done[x][0], 1);
      mbar_init(&bars->mma_done[x][1], 1);
    }
    mbar_init(&bars->chunk_full, 1);
    for (int x = 0; x < C::RS; ++x) {
      mbar_init(&bars->slot_full[x], 1);
      mbar_init(&bars->slot_free[x], 2);  // one arrival per warpgroup
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == 0) prefetch_tensormap(&map_q);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t t_s = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + wg * 2 * C::PIECE;
  uint8_t* sQ = smem + wg * C::Q_BYTES;
  // this warpgroup's candidate buffer [CB][128] of (score bits, block) pairs (pass 2), the score
  // words reused as staging [32][128] (pass 3), the block words as the selected list's staging
  uint2* cand = reinterpret_cast<uint2*>(smem + C::OFF_STAGE) + wg * CB * 128;
  const uint32_t cand_base = smem_u32(cand + row);  // this row's slot 0 (slots 1024 bytes apart)
  // predicated append, no branch: if s >= t, store (s, j) in the slot at address a, advance a
  auto append_if_ge = [](uint32_t& a, float sv, float t, int j) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ge.f32 p, %1, %2;\n @p st.shared.v2.b32 [%0], {%1, %3};\n"
        " @p add.u32 %0, %0, 1024;\n}\n"
        : "+r"(a)
        : "f"(sv), "f"(t), "r"(j)
        : "memory");
  };
  uint32_t chunk_phase = 0;   // chunk_full phase (pre-split centroids)
  uint32_t ring_l = 0;        // ring loads so far (CTA-uniform count)
  uint32_t ring_issued = 0;   // ring loads issued by thread 0
  bool chunk_pending = false; // a chunk copy issued by thread 0 that no wait has seen land
  const uint32_t sBa = smem_u32(smem + C::OFF_B);
  const int r = H / G;
  const int ksel = topk - 1;
  // rows of the routing are written as 16-byte pieces when each row starts on a 16-byte boundary
  const bool vec_out = (topk & 3) == 0 && (reinterpret_cast<uintptr_t>(idx) & 15) == 0;
  const uint64_t TO = kWaitTimeoutNs;
  uint32_t qphase = 0;  // q_full phase of this warpgroup
  uint32_t npiece = 0;  // score pieces issued by this warpgroup (TMEM buffer npiece & 1)
  bool ok = true;

  // Work units: (sequence, kv head g, group of QG consecutive query blocks, sub-range of at most
  // kTilesPerUnit tiles). Tiles of a unit share the centroid prefix [0, i_max) of its last query
  // block; each tile only considers its own past blocks j < i. Every wait is bounded; `ok` is made
  // uniform at each barrier (CTA-wide __syncthreads_and, warpgroup-wide bar.red.and) so that a
  // timeout never leaves a barrier half-attended.
  const int ttiles_max = (B + kTile - 1) / kTile;
  const int tiles_per_block = r * ttiles_max;
  const int QG = max(1, kTilesPerUnit / tiles_per_block);      // query blocks per unit
  const int n_sub = (QG * tiles_per_block + kTilesPerUnit - 1) / kTilesPerUnit;
  const int n_groups = (max_nb + QG - 1) / QG;
  // Units are numbered heaviest first (query-block group ig descending: a later group scores
  // more past blocks) and dealt to the CTAs in a snake order (0..grid-1, then grid-1..0, ...), so
  // every CTA gets a similar mix of heavy and light units.
  const long long per_ig = static_cast<long long>(nseq) * G * n_sub;
  const long long n_units = per_ig * n_groups;
  const long long grid = gridDim.x;
  for (long long kr = 0;; ++kr) {
    const long long u = kr * grid + ((kr & 1) ? grid - 1 - blockIdx.x : blockIdx.x);
    if (u >= n_units) break;
    const int ig = n_groups - 1 - static_cast<int>(u / per_ig);
    long long rest = u % per_ig;
    const int sub = static_cast<int>(rest % n_sub);
    rest /= n_sub;
    const int g = static_cast<int>(rest % G);
    const int s = static_cast<int>(rest / G);
    const int seq0 = cu[s], L = cu[s + 1] - seq0;
    const int nb = blocks_of(L, B);
    const int i_first = ig * QG;
    if (i_first >= nb) continue;  // uniform over the CTA
    const int i_last = min(nb, i_first + QG) - 1;
    // tiles of the unit: query blocks i_first..i_last, r heads, 128-token tiles of each block
    const int nt_all = (i_last - i_first + 1) * tiles_per_block;
    const int tile_lo = sub * kTilesPerUnit;
    if (tile_lo >= nt_all) continue;
    const int ntiles = min(kTilesPerUnit, nt_all - tile_lo);
    auto tile_info = [&](int tile, int& i_t, int& h_t, int& t0_t, int& rows_t) {
      const int tg = tile_lo + tile;
      const int ib = tg / tiles_per_block, w = tg % tiles_per_block;
      i_t = i_first + ib;
      h_t = g * r + w / ttiles_max;
      const int tt = w % ttiles_max;
      const int blen = min(B, L - i_t * B);
      t0_t = seq0 + i_t * B + tt * kTile;
      rows_t = max(0, min(kTile, blen - tt * kTile));
    };
    // past blocks needed by the unit: [0, i_max) with i_max the largest scored query block
    const int i_max = i_last > ksel && ksel > 0 ? i_last : 0;
    const int base = seq_block_base(cu, s, B, bars->red);
    const int nchunks = (i_max + C::CAP - 1) / C::CAP;
    // past blocks beyond the resident capacity stream through a ring of slots (pre-split only)
    const bool ring = split != nullptr && nchunks > 1;
    auto load_q = [&](int tile) {  // TMA of a query tile into this warpgroup's buffer
      int i_t, h_t, t0_t, rows_t;
      tile_info(tile, i_t, h_t, t0_t, rows_t);
      mbar_arrive_expect_tx(&bars->q_full[wg], C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::NCB; ++c)
        tma_load_3d(sQ + c * 16384, &map_q, &bars->q_full[wg], c * 64, h_t, t0_t);
    };
    // the first tile of each warpgroup that needs scores
    auto next_scored = [&](int from) {
      for (int t = from; t < ntiles; t += 2) {
        int i_t, h_t, t0_t, rows_t;
        tile_info(t, i_t, h_t, t0_t, rows_t);
        if (rows_t > 0 && i_t > ksel && ksel > 0) return t;
      }
      return ntiles;
    };
    if (row == 0 && ok) {
      const int t = next_scored(wg);
      if (t < ntiles) load_q(t);
    }
    // tiles are processed in pairs (one per warpgroup); every chunk of centroids is shared
    for (int p = 0; p < (ntiles + 1) / 2; ++p) {
      const int tile = 2 * p + wg;
      int i_t = 0, h = 0, t0 = 0, rows = 0;
      if (tile < ntiles) tile_info(tile, i_t, h, t0, rows);
      const bool scored = tile < ntiles && rows > 0 && i_t > ksel && ksel > 0;
      // past blocks this warpgroup scores, and the pair's (both warpgroups') number of ring pieces
      const int n_self = scored ? i_t : 0;
      int n_pair = n_self;
      {
        const int other = 2 * p + 1 - wg;
        int i_o = 0, h_o = 0, t0_o = 0, rows_o = 0;
        if (other < ntiles) tile_info(other, i_o, h_o, t0_o, rows_o);
        if (other < ntiles && rows_o > 0 && i_o > ksel && ksel > 0) n_pair = max(n_pair, i_o);
      }
      const int K_pair = (n_pair + C::PR - 1) / C::PR;
      // (thread 0) ring load Lm: centroid rows of piece k into slot Lm % RS, once both warpgroups
      // have released the slot's previous load. A wait that runs out raises the CTA's abort flag
      // (every later wait then fails, and `ok` turns false at the next warpgroup barrier), so
      // `ok` itself is left alone here: it must stay uniform inside the issuing warp.
      auto ring_load = [&](uint32_t Lm, int k) {
        if (!ok) return;
        const uint32_t sl = Lm % C::RS;
        if (Lm >= static_cast<uint32_t>(C::RS) &&
            !mbar_wait_bounded(&bars->slot_free[sl], ((Lm / C::RS) - 1) & 1, abort_flag, status,
                               kDevTimeoutAttn, TO))
          return;
        const int c0r = k * C::PR;
        const int rows_pad = (min(C::PR, n_pair - c0r) + 15) & ~15;
        mbar_arrive_expect_tx(&bars->slot_full[sl], 2 * C::NCB * rows_pad * 128);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int at = 0; at < C::NCB; ++at)
            bulk_load(smem + C::OFF_B + c_offset<D, KCAP>(part, static_cast<int>(sl) * C::PR, 64 * at),
                      split + ((static_cast<size_t>(g * 2 + part) * C::NCB + at) * nb_pad + base +
                               c0r) * 128,
                      rows_pad * 128, &bars->slot_full[sl]);
        ++ring_issued;
      };
      int32_t* out = idx + (static_cast<size_t>(h) * T + t0 + row) * topk;
      if (tile < ntiles && rows > 0 && !scored && row < rows) {
        // few causal blocks or topk == 1: the selection is fixed, no scores needed
        if (ksel == 0) out[0] = i_t;
        else
          for (int x = 0; x < topk; ++x) out[x] = (x <= i_t) ? x : -1;
      }
      // per-row selection state across the three passes
      float gmax[M];
#pragma unroll
      for (int x = 0; x < M; ++x) gmax[x] = -INFINITY;
      float tau = -INFINITY, tau_star = INFINITY;
      int cnt = 0, tie_budget = 0;
      unsigned long long sel_mask = 0;  // selected candidate slots (ksel bits)
      bool overflow = false;
      TopList<KCAP> top;  // the third pass's running list (initialised there)
      bool q_ready = false;
      // scores of 128 rows x np past blocks (from centroid rows row_off.. of the B region) into
      // TMEM buffer `buf`; one converged warp of the warpgroup issues
      const uint32_t qa = smem_u32(sQ);
      auto issue_rows = [&](int row_off, int np, uint32_t buf) {
        const int nmma = (np + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(128, nmma, 0, 0);
        tc_fence_after();
#pragma unroll
        for (int sp = 0; sp < 2; ++sp) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t aoff = (ks >> 2) * 16384 + (ks & 3) * 32;
            const uint32_t boff = static_cast<uint32_t>(sp * C::NCB * C::CAP * 128 +
                                                        (ks >> 2) * C::CAP * 128 + row_off * 128 +
                                                        (ks & 3) * 32);
            mma_ss_elect(tmem + wg * 2 * C::PIECE + buf * C::PIECE,
                         smem_desc_sw128(qa + aoff, 16, 1024),
                         smem_desc_sw128(sBa + boff, 16, 1024), idesc, (sp > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit_elect(&bars->mma_done[wg][buf]);
      };
      // the pass's work on one piece of scores (TMEM buffer of piece number pc; its columns are
      // past blocks gb .. gb + np - 1)
      auto select_piece = [&](int pass, uint32_t pc, int gb, int np) {
          tc_fence_after();
          const uint32_t tb = t_s + (pc & 1) * C::PIECE;
          // STEP columns per TMEM wait (64 with 32 groups, where both halves feed the same
          // group maxima; 32 with 64 groups, for registers); columns past the tile's last past
          // block read as -inf, so the per-score work below needs no bounds test
          for (int cc = 0; cc < np; cc += STEP) {
            uint32_t sa[32], sb[32];
            const bool two = STEP == 64 && cc + 32 < np;  // warpgroup-uniform
            tmem_ld32(tb + cc, sa);
            if (two) tmem_ld32(tb + cc + 32, sb);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              reg_fence(sa[x]);
              if (STEP == 64) reg_fence(sb[x]);
            }
            const int lim = np - cc;  // valid columns of the 64: c < lim
            if (lim < STEP) {
#pragma unroll
              for (int x = 0; x < 32; ++x) {
                if (x >= lim) sa[x] = __float_as_uint(-INFINITY);
                if (STEP == 64 && 32 + x >= lim) sb[x] = __float_as_uint(-INFINITY);
              }
            }
            const int jb = gb + cc;  // block of sa[x] is jb + x, of sb[x] jb + 32 + x
            if (pass == 0) {
              // group maxima, column j in group j mod M
              if (M == 32) {
#pragma unroll
                for (int x = 0; x < 32; ++x)
                  gmax[x] = fmax3(gmax[x], __uint_as_float(sa[x]), __uint_as_float(sb[x]));
              } else if ((jb & 32) == 0) {
#pragma unroll
                for (int x = 0; x < 32; ++x) gmax[x] = fmaxf(gmax[x], __uint_as_float(sa[x]));
              } else {
#pragma unroll
                for (int x = 0; x < 32; ++x)
                  gmax[(32 + x) % M] = fmaxf(gmax[(32 + x) % M], __uint_as_float(sa[x]));
              }
            } else if (pass == 1) {
              // every score >= tau is a candidate, kept with its block (ascending). While at
              // least eight slots are free, eight columns at a time append without a capacity
              // test ((score, block) pairs to cand[slot][row]).
              auto append = [&](const uint32_t (&v)[32], int jb0) {
#pragma unroll
                for (int x0 = 0; x0 < 32; x0 += 8) {
                  if (cnt <= CB - 8) {
                    uint32_t cp = cand_base + static_cast<uint32_t>(cnt) * 1024u;
#pragma unroll
                    for (int x = x0; x < x0 + 8; ++x)
                      append_if_ge(cp, __uint_as_float(v[x]), tau, jb0 + x);
                    cnt = static_cast<int>((cp - cand_base) >> 10);
                  } else {
#pragma unroll
                    for (int x = x0; x < x0 + 8; ++x) {
                      const float sv = __uint_as_float(v[x]);
                      if (sv >= tau) {
                        if (cnt < CB) {
                          cand[cnt * 128 + row] = make_uint2(__float_as_uint(sv), jb0 + x);
                        }
                        ++cnt;
                      }
                    }
                  }
                }
              };
              append(sa, jb);
              if (two) append(sb, jb + 32);
            } else {
              // rows whose candidates overflowed keep a running top list instead
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                if (hh == 1 && !two) break;
                const uint32_t(&sr)[32] = hh ? sb : sa;
                const int jh = jb + 32 * hh;
                const float thr0 = top.thr();
                uint32_t mask = 0;
                if (overflow) {
#pragma unroll
                  for (int x = 0; x < 32; ++x)
                    if (__uint_as_float(sr[x]) > thr0) mask |= 1u << x;
                }
                if (__any_sync(0xffffffffu, mask != 0)) {
                  if (overflow) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) cand[x * 128 + row].x = sr[x];
                  }
                  while (__any_sync(0xffffffffu, mask != 0)) {
                    if (mask) {
                      const int x = __ffs(mask) - 1;
                      mask &= mask - 1;
                      top.offer(__uint_as_float(cand[x * 128 + row].x), jh + x);
                    }
                  }
                  __syncwarp();
                }
              }
            }
          }
          tc_fence_before();
      };
      auto wait_q = [&]() {
        if (!q_ready) {
          const bool w = ok && mbar_wait_bounded(&bars->q_full[wg], qphase, abort_flag, status,
                                                 kDevTimeoutAttn, TO);
          qphase ^= 1;
          q_ready = true;
          ok = named_bar_and(1 + wg, 128, w);
        }
      };
      for (int pass = 0; pass < 3; ++pass) {
        // the third pass only runs for rows whose candidates overflowed (CTA-uniform decision)
        if (pass == 2 && !__syncthreads_or(overflow && scored && row < rows)) break;
        if (pass == 2) top.init(ksel);
        if (ring) {
          // Ring mode: piece k of the pass (past blocks k PR .. k PR + PR - 1) is ring load
          // L0 + k, in slot (L0 + k) % RS. Thread 0 keeps RS loads in flight: load m + RS is
          // issued once both warpgroups' products have finished reading load m (slot_free).
          const int K_w = (n_self + C::PR - 1) / C::PR;  // pieces this warpgroup scores
          const uint32_t L0 = ring_l;
          if (tid == 0)
            for (int k = 0; k < min(C::RS, K_pair); ++k) ring_load(L0 + k, k);
          if (K_w > 0) wait_q();
          auto issue_k = [&](int k) {
            const uint32_t Lk = L0 + k;
            const bool w = __all_sync(0xffffffffu,
                                      ok && mbar_wait_bounded(&bars->slot_full[Lk % C::RS],
                                                              (Lk / C::RS) & 1, abort_flag, status,
                                                              kDevTimeoutAttn, TO));
            if (w) issue_rows(static_cast<int>(Lk % C::RS) * C::PR,
                              min(C::PR, n_self - k * C::PR), npiece & 1);
          };
          if (K_w > 0) {
            if (ok && warp == wg * 4) issue_k(0);
            ++npiece;
          }
          for (int k = 0; k < K_pair; ++k) {
            const bool need = k < K_w;  // warpgroup-uniform
            const uint32_t pc = npiece - 1;
            if (need && k + 1 < K_w) {
              if (ok && warp == wg * 4) issue_k(k + 1);
              ++npiece;
            }
            bool w = ok;
            if (need)
              w = ok && mbar_wait_bounded(&bars->mma_done[wg][pc & 1], (pc >> 1) & 1, abort_flag,
                                          status, kDevTimeoutAttn, TO);
            // this warpgroup's products no longer read the slot (or never did). A warpgroup that
            // does not score piece k still waits for its load first, so that its release counts
            // toward this load and not an earlier one of the slot.
            if (row == 0) {
              const uint32_t Lk = L0 + k;
              if (!need && ok)  // a timeout raises the abort flag; the release happens regardless
                mbar_wait_bounded(&bars->slot_full[Lk % C::RS], (Lk / C::RS) & 1, abort_flag,
                                  status, kDevTimeoutAttn, TO);
              mbar_arrive(&bars->slot_free[Lk % C::RS]);
            }
            if (tid == 0 && k + C::RS < K_pair) ring_load(L0 + k + C::RS, k + C::RS);
            if (need) {
              if (__all_sync(0xffffffffu, w))
                select_piece(pass, pc, k * C::PR, min(C::PR, n_self - k * C::PR));
              // every thread of the warpgroup has read this buffer before piece k + 2 overwrites it
              ok = named_bar_and(1 + wg, 128, w);
            }
          }
          ring_l += K_pair;
        } else {
        for (int ch = 0; ch < nchunks; ++ch) {
          const int c0 = ch * C::CAP;
          const int n = min(C::CAP, i_max - c0);
          if ((nchunks > 1 || (p == 0 && pass == 0)) && split) {
            // pre-split hi / lo rows of blocks [c0, c0 + n) (16-row padded): one bulk copy per
            // part and 64-column atom; rows were swizzled by their block's index in its sequence,
            // and c0 % 8 == 0, so they land in the layout the MMA reads
            ok = __syncthreads_and(ok);
            const int rows_pad = (n + 15) & ~15;
            if (tid == 0 && ok) {
              mbar_arrive_expect_tx(&bars->chunk_full, 2 * C::NCB * rows_pad * 128);
#pragma unroll
              for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int at = 0; at < C::NCB; ++at)
                  bulk_load(smem + C::OFF_B + c_offset<D, KCAP>(part, 0, 64 * at),
                            split + ((static_cast<size_t>(g * 2 + part) * C::NCB + at) * nb_pad +
                                     base + c0) * 128,
                            rows_pad * 128, &bars->chunk_full);
              chunk_pending = true;
            }
            const bool w = ok && mbar_wait_bounded(&bars->chunk_full, chunk_phase, abort_flag,
                                                   status, kDevTimeoutAttn, TO);
            chunk_phase ^= 1;
            if (tid == 0 && w) chunk_pending = false;
            ok = __syncthreads_and(w);
          } else if (nchunks > 1 || (p == 0 && pass == 0)) {
            // split the fp32 centroids of blocks [c0, c0 + n) into hi / lo bf16 tiles; each thread
            // issues the loads of eight 8-column groups before converting any
            ok = __syncthreads_and(ok);
            const int nrows = (n + 15) & ~15;
            const int ngroups = nrows * (D / 8);
            for (int e0 = tid; ok && e0 < ngroups; e0 += 8 * static_cast<int>(blockDim.x)) {
              float4 va[8], vb[8];
#pragma unroll
              for (int uu = 0; uu < 8; ++uu) {
                const int e = e0 + uu * static_cast<int>(blockDim.x);
                const int rr = e / (D / 8), c8 = (e % (D / 8)) * 8;
                va[uu] = make_float4(0.f, 0.f, 0.f, 0.f);
                vb[uu] = va[uu];
                if (e < ngroups && rr < n) {
                  const float4* src = reinterpret_cast<const float4*>(
                      cents + (static_cast<size_t>(base + c0 + rr) * G + g) * D + c8);
                  va[uu] = __ldg(src);
                  vb[uu] = __ldg(src + 1);
                }
              }
#pragma unroll
              for (int uu = 0; uu < 8; ++uu) {
                const int e = e0 + uu * static_cast<int>(blockDim.x);
                if (e >= ngroups) break;
                const int rr = e / (D / 8), c8 = (e % (D / 8)) * 8;
                const float x[8] = {va[uu].x, va[uu].y, va[uu].z, va[uu].w,
                                    vb[uu].x, vb[uu].y, vb[uu].z, vb[uu].w};
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * k]);
                  const __nv_bfloat16 h1 = __float2bfloat16_rn(x[2 * k + 1]);
                  const __nv_bfloat16 l0 = __float2bfloat16_rn(x[2 * k] - __bfloat162float(h0));
                  const __nv_bfloat16 l1 =
                      __float2bfloat16_rn(x[2 * k + 1] - __bfloat162float(h1));
                  hw[k] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                          (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
                  lw[k] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                          (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
                }
                *reinterpret_cast<uint4*>(smem + C::OFF_B + c_offset<D, KCAP>(0, rr, c8)) =
                    make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(smem + C::OFF_B + c_offset<D, KCAP>(1, rr, c8)) =
                    make_uint4(lw[0], lw[1], lw[2], lw[3]);
              }
            }
            fence_proxy_async_smem();
            __syncthreads();
          }
          if (!scored || c0 >= i_t) continue;  // warpgroup-uniform
          const int n_t = min(n, i_t - c0);       // this tile's past blocks in the chunk
          wait_q();
          // scores of this chunk, 128 past blocks per TMEM buffer; the products of piece p + 1 are
          // issued before piece p is selected (its buffer was freed by the barrier ending p - 1)
          if (ok && warp == wg * 4) issue_rows(0, min(C::PIECE, n_t), npiece & 1);
          ++npiece;
          for (int p0 = 0; p0 < n_t; p0 += C::PIECE) {
            const int np = min(C::PIECE, n_t - p0);
            const uint32_t pc = npiece - 1;  // this piece's number
            if (p0 + C::PIECE < n_t) {
              if (ok && warp == wg * 4)
                issue_rows(p0 + C::PIECE, min(C::PIECE, n_t - p0 - C::PIECE), npiece & 1);
              ++npiece;
            }
            const bool w = ok && mbar_wait_bounded(&bars->mma_done[wg][pc & 1], (pc >> 1) & 1,
                                                   abort_flag, status, kDevTimeoutAttn, TO);
            if (__all_sync(0xffffffffu, w)) select_piece(pass, pc, c0 + p0, np);
            // every thread of the warpgroup has read this buffer before piece p + 2 overwrites it
            ok = named_bar_and(1 + wg, 128, w);
          }
        }
        }
        if (!scored) continue;
        if (pass == 0) {
          // tau: the ksel-th largest group maximum (ksel <= M groups hold a score >= tau)
          bitonic_desc_f<M>(gmax);
          tau = kth_of_sorted<M>(gmax, ksel);
        } else if (pass == 1) {
          overflow = cnt > CB;
          if (!overflow) {
            // the exact ksel-th best score tau* among the candidates (a sort of 32 values when
            // they fit, the buffer's CB otherwise), and how many of the selected tie with it
            float cv[CB];
#pragma unroll
            for (int x = 0; x < CB; ++x)
              cv[x] = (x < cnt) ? __uint_as_float(cand[x * 128 + row].x) : -INFINITY;
            int above = 0;
            if (CB > 32 && cnt <= 32) {
              float c32[32];
#pragma unroll
              for (int x = 0; x < 32; ++x) c32[x] = cv[x];
              bitonic_desc_f<32>(c32);
              tau_star = kth_of_sorted<32>(c32, ksel);
#pragma unroll
              for (int x = 0; x < 32; ++x) above += (c32[x] > tau_star) ? 1 : 0;
            } else {
              bitonic_desc_f<CB>(cv);
              tau_star = kth_of_sorted<CB>(cv, ksel);
#pragma unroll
              for (int x = 0; x < CB; ++x) above += (cv[x] > tau_star) ? 1 : 0;
            }
            tie_budget = ksel - above;
            // the buffer is in ascending block order: the selection is the blocks above tau* and
            // the lowest ties, marked in a bit mask (loads independent of the running tie count)
            int ties = 0;
#pragma unroll
            for (int x = 0; x < CB; ++x) {
              if (x < cnt) {
                const float sv = __uint_as_float(cand[x * 128 + row].x);
                const bool tie = sv == tau_star && ties < tie_budget;
                ties += tie ? 1 : 0;
                if (sv > tau_star || tie) sel_mask |= 1ull << x;
              }
            }
          }
        }
      }
      // the Q buffer is free: every product of this tile is done; load the next scored tile
      if (scored && row == 0 && ok) {
        const int t = next_scored(tile + 2);
        if (t < ntiles) load_q(t);
      }
      if (!scored || row >= rows || !ok) continue;
      if (!overflow) {
        // the ksel selected blocks (the set bits of sel_mask, ascending) and the current block,
        // as 16-byte pieces of the row when its length and address allow
        unsigned long long m = sel_mask;
        auto sel = [&](int x) {
          if (x >= ksel) return i_t;
          const int slot = __ffsll(static_cast<long long>(m)) - 1;
          m &= m - 1;
          return static_cast<int>(cand[slot * 128 + row].y);
        };
        if (vec_out) {
          for (int x = 0; x < topk; x += 4) {
            const int a0 = sel(x), a1 = sel(x + 1), a2 = sel(x + 2), a3 = sel(x + 3);
            *reinterpret_cast<int4*>(out + x) = make_int4(a0, a1, a2, a3);
          }
        } else {
          for (int x = 0; x < topk; ++x) out[x] = sel(x);
        }
        continue;
      }
      {
        // the ksel real entries of the running list (sentinels map to INT_MAX), ascending
        int sel[KCAP];
#pragma unroll
        for (int x = 0; x < KCAP; ++x) sel[x] = top.id[x];
#pragma unroll
        for (int a0 = 0; a0 < KCAP - 1; ++a0) {
#pragma unroll
          for (int b0 = 0; b0 < KCAP - 1 - a0; ++b0) {
            const int lo_ = min(sel[b0], sel[b0 + 1]), hi_ = max(sel[b0], sel[b0 + 1]);
            sel[b0] = lo_;
            sel[b0 + 1] = hi_;
          }
        }
#pragma unroll
        for (int x = 0; x < KCAP; ++x)
          if (x < ksel) out[x] = sel[x];
      }
      out[ksel] = i_t;
    }
    ok = __syncthreads_and(ok);
    if (!ok) break;
  }
  if (tid == 0 && ring_issued > 0) {
    // ring loads whose landing no wait may have seen: let them land before the CTA exits
    volatile int no_abort = 0;
    for (uint32_t x = 0; x < static_cast<uint32_t>(C::RS) && x < ring_issued; ++x) {
      const uint32_t Lm = ring_issued - 1 - x;
      mbar_wait_bounded(&bars->slot_full[Lm % C::RS], (Lm / C::RS) & 1, &no_abort, status,
                        kDevDrainTimeout, kDrainTimeoutNs);
    }
  }
  if (tid == 0 && chunk_pending) {
    // a chunk copy whose landing no wait saw: let it land before the CTA exits (bounded)
    volatile int no_abort = 0;
    mbar_wait_bounded(&bars->chunk_full, chunk_phase ^ 1, &no_abort, status, kDevDrainTimeout,
                      kDrainTimeoutNs);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Pre-split centroids for the gate: for kv head g, part (0 = hi, 1 = lo bf16 of the fp32
// centroid), 64-column atom a and global block b, one 128-byte row at
// (((g * 2 + part) * NCB + a) * nb_pad + b) * 128 with its 16-byte pieces swizzled by the
// block's index inside its sequence (mod 8) — the rows of a chunk that starts at a multiple of 8
// then land in shared memory in the MMA's 128-byte-swizzle layout. Rows b >= NB are zero.
template <int D>
__global__ void __launch_bounds__(256) split_cents_kernel(const float* __restrict__ cents,
                                                          BlockTables tb, int NB, int nb_pad,
                                                          int G, uint8_t* __restrict__ split) {
  constexpr int NCB = D / 64;
  const long long n = static_cast<long long>(nb_pad) * G * NCB * 8;  // 16-byte pieces per part
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < n;
       x += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(x % 8);
    long long rest = x / 8;
    const int at = static_cast<int>(rest % NCB);
    rest /= NCB;
    const int b = static_cast<int>(rest % nb_pad);
    const int g = static_cast<int>(rest / nb_pad);
    uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi;
    int j = 0;
    if (b < NB) {
      j = b - tb.blk_off[tb.blk_seq[b]];
      const float4* src =
          reinterpret_cast<const float4*>(cents + (static_cast<size_t>(b) * G + g) * D + at * 64 + c * 8);
      const float4 va = __ldg(src), vb = __ldg(src + 1);
      const float v[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * k]);
        const __nv_bfloat16 h1 = __float2bfloat16_rn(v[2 * k + 1]);
        const __nv_bfloat16 l0 = __float2bfloat16_rn(v[2 * k] - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(v[2 * k + 1] - __bfloat162float(h1));
        hw[k] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        lw[k] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
      }
      hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    const size_t piece = static_cast<size_t>((c ^ (j & 7)) & 7) * 16;
    *reinterpret_cast<uint4*>(split + ((static_cast<size_t>(g * 2) * NCB + at) * nb_pad + b) * 128 +
                              piece) = hi;
    *reinterpret_cast<uint4*>(split + ((static_cast<size_t>(g * 2 + 1) * NCB + at) * nb_pad + b) *
                                          128 +
                              piece) = lo;
  }
}

namespace {

typedef CUresult (*EncodeTiledFnG)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_q_map(CUtensorMap* map, const void* q, int T, int H, int D) {
  static EncodeTiledFnG fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFnG>(p);
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
cudaError_t launch_t(const CUtensorMap& mq, const float* cents, const int32_t* cu, int nseq,
                     int max_nb, int T, int H, int G, int B, int topk, int32_t* idx, int* status,
                     int grid, cudaStream_t stream, const uint8_t* split, int nb_pad) {
  const int smem = GateCfg<D, KCAP>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(gate_tc_kernel<D, KCAP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gate_tc_kernel<D, KCAP><<<grid, 256, smem, stream>>>(mq, cents, cu, nseq, max_nb, T, H, G, B,
                                                       topk, idx, status, split, nb_pad);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const CUtensorMap& mq, const float* cents, const int32_t* cu, int nseq,
                     int max_nb, int T, int H, int G, int B, int topk, int32_t* idx, int* status,
                     int grid, cudaStream_t stream, const uint8_t* split, int nb_pad) {
  const int ksel = topk - 1;
  if (ksel <= 4)
    return launch_t<D, 4>(mq, cents, cu, nseq, max_nb, T, H, G, B, topk, idx, status, grid,
                          stream, split, nb_pad);
  if (ksel <= 8)
    return launch_t<D, 8>(mq, cents, cu, nseq, max_nb, T, H, G, B, topk, idx, status, grid,
                          stream, split, nb_pad);
  if (ksel <= 16)
    return launch_t<D, 16>(mq, cents, cu, nseq, max_nb, T, H, G, B, topk, idx, status, grid,
                           stream, split, nb_pad);
  return launch_t<D, 32>(mq, cents, cu, nseq, max_nb, T, H, G, B, topk, idx, status, grid, stream,
                         split, nb_pad);
}

}  // namespace

cudaError_t launch_gate_tc(const void* q, const float* cents, const int32_t* cu_dev, int nseq,
                           int max_nb, int T, int H, int G, int d, int B, int topk, int32_t* idx,
                           int* status, int num_sms, cudaStream_t stream, const BlockTables* tb,
                           int NB, void* split) {
  if (topk - 1 > 32) return cudaErrorInvalidValue;
  CUtensorMap mq;
  if (!make_q_map(&mq, q, T, H, d)) return cudaErrorInvalidValue;
  const int grid = num_sms > 0 ? num_sms : 1;  // persistent CTAs over the work units
  const int nb_pad = NB + 16;
  const uint8_t* sp = nullptr;
  if (split && tb) {
    const long long pieces = static_cast<long long>(nb_pad) * G * (d / 64) * 8;
    const unsigned g2 = static_cast<unsigned>(
        std::max<long long>(1, std::min<long long>((pieces + 255) / 256, 8LL * grid)));
    if (d == 64)
      split_cents_kernel<64><<<g2, 256, 0, stream>>>(cents, *tb, NB, nb_pad, G,
                                                     static_cast<uint8_t*>(split));
    else
      split_cents_kernel<128><<<g2, 256, 0, stream>>>(cents, *tb, NB, nb_pad, G,
                                                      static_cast<uint8_t*>(split));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    sp = static_cast<const uint8_t*>(split);
  }
  if (d == 64)
    return launch_d<64>(mq, cents, cu_dev, nseq, max_nb, T, H, G, B, topk, idx, status, grid,
                        stream, sp, nb_pad);
  return launch_d<128>(mq, cents, cu_dev, nseq, max_nb, T, H, G, B, topk, idx, status, grid,
                       stream, sp, nb_pad);
}

// Bytes of the pre-split centroid buffer launch_gate_tc fills (hi and lo bf16 per fp32 value,
// 16 padding rows).
size_t gate_split_bytes(int NB, int G, int d) {
  return static_cast<size_t>(NB + 16) * G * d * 4;
}

}  // namespace moba
