// K4 — block-sparse attention on the tcgen05 tensor cores.
//
// Work items (one 128-row query tile each, processed by a persistent CTA per SM):
//   routed tile : up to 128 (t, h) rows of one kv head g that routed to one past block b (a list
//                 built by the routing inversion), attending every key of b — the scattered query
//                 rows are gathered into one dense operand [FlashMoBA story, Gather-and-Densify];
//   diagonal tile: 128 consecutive tokens of one query head inside their own block, attending the
//                 block's keys up to the query position (causal inside the current block)
//                 [MoBA paper summary (atlas.scime.ai), "Approach"].
// Each row's result is a normalised partial O_s (bf16) plus its log-sum-exp (fp32), written to the
// row's slot; the merge kernel combines the slots.
//
// Per item, for every 128-key sub-tile j of the key range:
//   S_j = Q K_j^T           tcgen05.mma kind::f16, A = Q (smem, K-major SW128), B = K_j (smem,
//                           K-major SW128, loaded by TMA), fp32 accumulator in TMEM
//   P_j = exp2(S_j * scale * log2e - m)   one thread per row (TMEM lane), written back to TMEM
//                                         as bf16 over the S columns
//   O  += P_j V_j           tcgen05.mma with A = P read from TMEM, B = V_j (smem, MN-major SW128)
// The running max m is only raised when a row's max grows by more than 2^8 (then O and l are
// rescaled), which keeps every p <= 256 and makes rescaling rare; O / l is exact either way.
//
// Warp roles (256 threads): warp 0 = TMA producer of K/V sub-tiles; warp 1 = TMEM owner and MMA
// issuer; warps 2-3 = Q row gather (cp.async into the swizzled layout); warps 4-7 = softmax and
// epilogue (thread i <-> TMEM lane i <-> query row i). Buffers: Q x2, K x NST, V x NST in shared
// memory; S/P x2 and O x2 in TMEM (512 columns). Every wait is bounded (2 s); on a timeout the
// kernel raises a CTA abort flag, records a status code and every role leaves its loop.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace moba {

struct AttnArgs {
  const __nv_bfloat16* q;  // [T, H, D]
  const int4* tiles;       // routed tiles: {bucket, first entry, rows, -}
  const int* n_routed;     // device count of routed tiles
  const int* entries;      // partial row of every routed (t, h, slot)
  BlockTables tb;
  __nv_bfloat16* part_o;   // [rows, D]
  float* part_lse;         // [rows]
  int* status;
  int T, H, G, r, topk, NB;
  int b0, nblk, T0;        // chunk: global blocks [b0, b0 + nblk), first token T0
  int P;                   // ceil(B / 128): 128-row tiles per block
  int n_diag;              // P * nblk * H diagonal items (some may be empty)
  float scale_log2;        // scale * log2(e)
};

struct Item {
  int kind;  // 0 empty, 1 routed, 2 diagonal
  int g, h, b;
  int key0, klen, nsub;
  int rows, start;       // routed: rows and first entry; diagonal: rows
  int qtok0, p, slot;    // diagonal: first query token, tile position in block, output slot
};

__device__ __forceinline__ Item decode_item(const AttnArgs& a, int w, int n_routed) {
  Item it;
  it.kind = 0;
  if (w < n_routed) {
    const int4 tl = a.tiles[w];
    it.kind = 1;
    it.g = tl.x / a.NB;
    it.b = tl.x % a.NB;
    it.h = 0;
    it.start = tl.y;
    it.rows = tl.z;
    it.key0 = a.tb.blk_start[it.b];
    it.klen = a.tb.blk_len[it.b];
    it.nsub = (it.klen + kTile - 1) / kTile;
    it.qtok0 = 0;
    it.p = 0;
    it.slot = 0;
    return it;
  }
  const int wd = w - n_routed;
  it.h = wd % a.H;
  const int rest = wd / a.H;
  const int bl = rest % a.nblk;
  it.p = a.P - 1 - rest / a.nblk;  // longest diagonal tiles first
  it.b = a.b0 + bl;
  const int len = a.tb.blk_len[it.b];
  if (it.p * kTile >= len) return it;  // empty (short last block)
  it.kind = 2;
  it.g = it.h / a.r;
  it.key0 = a.tb.blk_start[it.b];
  it.klen = min(len, kTile * (it.p + 1));
  it.nsub = it.p + 1;
  it.rows = min(kTile, len - kTile * it.p);
  it.start = 0;
  it.qtok0 = it.key0 + kTile * it.p;
  const int i = it.b - a.tb.blk_off[a.tb.blk_seq[it.b]];
  it.slot = min(a.topk, i + 1) - 1;
  return it;
}

template <int D>
struct AttnCfg {
  static constexpr int NCB = D / 64;                 // 64-column (128-byte) swizzle blocks
  static constexpr int TILE_BYTES = kTile * D * 2;   // one 128 x D bf16 tile
  static constexpr int NST = (D == 128) ? 2 : 4;     // K and V ring depth
  static constexpr int SMEM_TILES = (2 + 2 * NST) * TILE_BYTES;
  static constexpr int SMEM_BYTES = SMEM_TILES + 1024 /*barriers*/ + 1024 /*alignment slack*/;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O0 = 256, TM_O1 = 256 + D;
};

struct AttnBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_full[2], o_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(256, 1)
    attn_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                const AttnArgs a) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                              // [2][NCB][16 KB]
  uint8_t* sK = sQ + 2 * C::TILE_BYTES;            // [NST][NCB][16 KB]
  uint8_t* sV = sK + C::NST * C::TILE_BYTES;       // [NST][NCB][16 KB]
  AttnBars* bars = reinterpret_cast<AttnBars*>(sV + C::NST * C::TILE_BYTES);
  volatile int* abort_flag = &bars->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->q_full[x], 64);
      mbar_init(&bars->q_empty[x], 1);
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_full[x], 128);
      mbar_init(&bars->o_full[x], 1);
      mbar_init(&bars->o_free[x], 128);
    }
    for (int x = 0; x < C::NST; ++x) {
      mbar_init(&bars->k_full[x], 1);
      mbar_init(&bars->k_empty[x], 1);
      mbar_init(&bars->v_full[x], 1);
      mbar_init(&bars->v_empty[x], 1);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->drain, 1);
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const int n_routed = *a.n_routed;
  const int n_items = n_routed + a.n_diag;
  const uint64_t TO = kWaitTimeoutNs;
  int* err = a.status;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (K, V)
    if (lane == 0) {
      uint32_t J = 0, issued_k = 0, issued_v = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        const Item it = decode_item(a, w, n_routed);
        if (it.kind == 0) continue;
        for (int j = 0; j < it.nsub && ok; ++j, ++J) {
          const int st = J % C::NST;
          const uint32_t ph = (J / C::NST) & 1;
          const int tok = it.key0 + j * kTile;
          ok = mbar_wait_bounded(&bars->k_empty[st], ph ^ 1, abort_flag, err, kDevTimeoutAttn, TO);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->k_full[st], C::TILE_BYTES);
#pragma unroll
          for (int c = 0; c < C::NCB; ++c)
            tma_load_3d(sK + st * C::TILE_BYTES + c * 16384, &map_k, &bars->k_full[st], c * 64,
                        it.g, tok);
          ++issued_k;
          ok = mbar_wait_bounded(&bars->v_empty[st], ph ^ 1, abort_flag, err, kDevTimeoutAttn, TO);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->v_full[st], C::TILE_BYTES);
#pragma unroll
          for (int c = 0; c < C::NCB; ++c)
            tma_load_3d(sV + st * C::TILE_BYTES + c * 16384, &map_v, &bars->v_full[st], c * 64,
                        it.g, tok);
          ++issued_v;
        }
      }
      if (!ok) {
        // after an abort, let the loads still in flight land before the CTA exits (bounded)
        volatile int no_abort = 0;
        for (uint32_t x = 0; x < static_cast<uint32_t>(C::NST); ++x) {
          if (issued_k > x) {
            const uint32_t Jx = issued_k - 1 - x;
            mbar_wait_bounded(&bars->k_full[Jx % C::NST], (Jx / C::NST) & 1, &no_abort, nullptr, 0, TO / 4);
          }
          if (issued_v > x) {
            const uint32_t Jx = issued_v - 1 - x;
            mbar_wait_bounded(&bars->v_full[Jx % C::NST], (Jx / C::NST) & 1, &no_abort, nullptr, 0, TO / 4);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      uint32_t J = 0, lt = 0;
      bool ok = true;
      // the PV of sub-tile J-1 is issued after the QK of sub-tile J (software pipelining)
      bool pend = false;
      uint32_t pend_J = 0, pend_ob = 0, pend_lt = 0;
      bool pend_first = false, pend_last = false;
      auto issue_pv = [&](uint32_t Jp, uint32_t ob, uint32_t ltp, bool first, bool last) -> bool {
        const uint32_t sb = Jp & 1;
        const int st = Jp % C::NST;
        if (!mbar_wait_bounded(&bars->p_full[sb], (Jp >> 1) & 1, abort_flag, err, kDevTimeoutAttn, TO))
          return false;
        if (!mbar_wait_bounded(&bars->v_full[st], (Jp / C::NST) & 1, abort_flag, err, kDevTimeoutAttn, TO))
          return false;
        if (first && !mbar_wait_bounded(&bars->o_free[ob], ((ltp >> 1) & 1) ^ 1, abort_flag, err,
                                        kDevTimeoutAttn, TO))
          return false;
        tc_fence_after();
        const uint32_t t_o = tmem + (ob ? C::TM_O1 : C::TM_O0);
        const uint32_t t_p = tmem + (sb ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks) {
          const uint64_t bd =
              smem_desc_sw128(sVa + st * C::TILE_BYTES + ks * 2048, 16384, 1024);
          mma_ts(t_o, t_p + ks * 8, bd, IDESC_PV, (first && ks == 0) ? 0u : 1u);
        }
        mma_commit(&bars->v_empty[st]);
        mma_commit(&bars->o_done);
        if (last) mma_commit(&bars->o_full[ob]);
        return true;
      };
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        const Item it = decode_item(a, w, n_routed);
        if (it.kind == 0) continue;
        const uint32_t qb = lt & 1;
        ok = mbar_wait_bounded(&bars->q_full[qb], (lt >> 1) & 1, abort_flag, err, kDevTimeoutAttn, TO);
        if (!ok) break;
        tc_fence_after();
        for (int j = 0; j < it.nsub; ++j, ++J) {
          const uint32_t sb = J & 1;
          const int st = J % C::NST;
          ok = mbar_wait_bounded(&bars->k_full[st], (J / C::NST) & 1, abort_flag, err, kDevTimeoutAttn, TO);
          if (!ok) break;
          tc_fence_after();
          const uint32_t t_s = tmem + (sb ? C::TM_S1 : C::TM_S0);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
            const uint64_t ad = smem_desc_sw128(sQa + qb * C::TILE_BYTES + off, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sKa + st * C::TILE_BYTES + off, 16, 1024);
            mma_ss(t_s, ad, bd, IDESC_QK, ks > 0 ? 1u : 0u);
          }
          mma_commit(&bars->k_empty[st]);
          mma_commit(&bars->s_full[sb]);
          if (j == it.nsub - 1) mma_commit(&bars->q_empty[qb]);
          if (pend) {
            ok = issue_pv(pend_J, pend_ob, pend_lt, pend_first, pend_last);
            if (!ok) break;
          }
          pend = true;
          pend_J = J;
          pend_ob = lt & 1;
          pend_lt = lt;
          pend_first = (j == 0);
          pend_last = (j == it.nsub - 1);
        }
        ++lt;
      }
      if (ok && pend) ok = issue_pv(pend_J, pend_ob, pend_lt, pend_first, pend_last);
      if (!ok) {
        // after an abort, wait (bounded) until the MMAs already issued have finished with TMEM
        volatile int no_abort = 0;
        mma_commit(&bars->drain);
        mbar_wait_bounded(&bars->drain, 0, &no_abort, nullptr, 0, TO / 4);
      }
    }
  } else if (warp < 4) {
    // -------------------------------------------------------------------- Q row gather
    const int gt = tid - 64;  // 0..63
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    uint32_t lt = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const Item it = decode_item(a, w, n_routed);
      if (it.kind == 0) continue;
      const uint32_t qb = lt & 1;
      ok = mbar_wait_bounded(&bars->q_empty[qb], ((lt >> 1) & 1) ^ 1, abort_flag, err, kDevTimeoutAttn, TO);
      if (!ok) break;
      const uint32_t dst0 = smem_u32(sQ + qb * C::TILE_BYTES);
      for (int e = gt; e < kTile * CPR; e += 64) {
        const int m = e / CPR, c = e % CPR;
        const __nv_bfloat16* src = a.q;
        uint32_t bytes = 0;
        if (m < it.rows) {
          int t, h;
          if (it.kind == 1) {
            const int pr = __ldg(a.entries + it.start + m);
            t = a.T0 + pr / (a.H * a.topk);
            h = (pr / a.topk) % a.H;
          } else {
            t = it.qtok0 + m;
            h = it.h;
          }
          src = a.q + (static_cast<size_t>(t) * a.H + h) * D + c * 8;
          bytes = 16;
        }
        cp_async_16(dst0 + (c >> 3) * 16384 + sw128_offset(m, (c & 7) * 8), src, bytes);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(&bars->q_full[qb]);
      ++lt;
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int row = tid - 128;  // TMEM lane / query row of this thread
    const uint32_t lane_off = static_cast<uint32_t>((warp - 4) * 32) << 16;
    const float sl2 = a.scale_log2;
    uint32_t J = 0, lt = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const Item it = decode_item(a, w, n_routed);
      if (it.kind == 0) continue;
      const bool valid = row < it.rows;
      int prow = 0, limit;
      if (it.kind == 1) {
        if (valid) prow = __ldg(a.entries + it.start + row);
        limit = it.klen;
      } else {
        const int t = it.qtok0 + row;
        prow = ((t - a.T0) * a.H + it.h) * a.topk + it.slot;
        limit = valid ? kTile * it.p + row + 1 : 1;
      }
      float m_ref = -INFINITY, l_sum = 0.f;
      const uint32_t ob = lt & 1;
      const uint32_t t_o = tmem + lane_off + (ob ? C::TM_O1 : C::TM_O0);
      for (int j = 0; j < it.nsub; ++j, ++J) {
        const uint32_t sb = J & 1;
        ok = mbar_wait_bounded(&bars->s_full[sb], (J >> 1) & 1, abort_flag, err, kDevTimeoutAttn, TO);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t t_s = tmem + lane_off + (sb ? C::TM_S1 : C::TM_S0);
        uint32_t sr[128];
        tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_wait_ld();
        const int lim = limit - j * kTile;  // valid columns: c < lim
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const float v = (c < lim) ? __uint_as_float(sr[c]) : -INFINITY;
          sr[c] = __float_as_uint(v);
          mx = fmaxf(mx, v);
        }
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
          // O holds sub-tiles < j: wait for the PV of sub-tile J-1, then rescale O in TMEM
          ok = mbar_wait_bounded(&bars->o_done, (J - 1) & 1, abort_flag, err, kDevTimeoutAttn, TO);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t orr[32];
            tmem_ld32(t_o + c0, orr);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) orr[x] = __float_as_uint(__uint_as_float(orr[x]) * alpha);
            tmem_st32(t_o + c0, orr);
          }
          tmem_wait_st();
        }
        const float neg = -m_ref;
        float ps = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c]), sl2, neg));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c + 1]), sl2, neg));
          ps += p0 + p1;
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        l_sum += ps;
        tmem_st32(t_s + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
        tmem_st32(t_s + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[sb]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 partial row, log-sum-exp
      ok = mbar_wait_bounded(&bars->o_full[ob], (lt >> 1) & 1, abort_flag, err, kDevTimeoutAttn, TO);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv = 1.f / l_sum;
      __nv_bfloat16* dst = a.part_o + static_cast<size_t>(prow) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t orr[32];
        tmem_ld32(t_o + c0, orr);
        tmem_wait_ld();
        if (valid) {
          uint4 pkt[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pkt);
#pragma unroll
          for (int x = 0; x < 16; ++x)
            pw[x] = pack_bf16x2(__uint_as_float(orr[2 * x]) * inv, __uint_as_float(orr[2 * x + 1]) * inv);
#pragma unroll
          for (int x = 0; x < 4; ++x) reinterpret_cast<uint4*>(dst + c0)[x] = pkt[x];
        }
      }
      if (valid) a.part_lse[prow] = (m_ref + __log2f(l_sum)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(&bars->o_free[ob]);
      ++lt;
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
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
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
static bool make_kv_map(CUtensorMap* map, const void* base, int T, int G, int D) {
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

cudaError_t launch_attention(const AttnLaunch& L, cudaStream_t stream) {
  CUtensorMap mk, mv;
  if (!make_kv_map(&mk, L.k, L.T, L.G, L.d) || !make_kv_map(&mv, L.v, L.T, L.G, L.d))
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
  a.P = (L.B + kTile - 1) / kTile;
  a.n_diag = a.P * L.nblk * L.H;
  a.scale_log2 = L.scale * 1.4426950408889634f;
  const int grid = L.grid > 0 ? L.grid : 1;
  if (L.d == 64) {
    const int smem = AttnCfg<64>::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_kernel<64><<<grid, 256, smem, stream>>>(mk, mv, a);
  } else {
    const int smem = AttnCfg<128>::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_kernel<128><<<grid, 256, smem, stream>>>(mk, mv, a);
  }
  return cudaGetLastError();
}

}  // namespace moba
