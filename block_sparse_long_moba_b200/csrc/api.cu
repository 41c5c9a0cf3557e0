// C ABI of libmoba.so: argument validation, the host-side plan (block counts, query chunks,
// workspace layout), launch sequencing and optional per-kernel event timing. Every step of the
// computation runs in the kernels; this file only sizes and orders them.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/moba.h"
#include "common.cuh"
#include "launch.h"

using namespace moba;

namespace {

constexpr size_t kPartialBudgetBytes = 16ull << 30;  // per-chunk partial outputs + routing lists
constexpr int kNumClasses = 13;
enum KernelClass {
  kCentroid = 0, kGate, kRouteCount, kRouteScan, kRouteScatter, kAttn, kMerge, kPlan, kDensify,
  kDecode, kBwdDkdv, kBwdDq, kBwdAux
};

std::atomic<long long> g_launches{0};
// Limit of one pipeline wait inside the attention kernel (0 = the built-in 2 s).
std::atomic<unsigned long long> g_wait_limit_ns{0};
// Diagnostics: when set, the attention kernel's MMA issuer first waits on a barrier that nothing
// arrives on, so that the wait runs out and every CTA takes its abort path.
std::atomic<int> g_diag_stall{0};

// ------------------------------------------------------------------------------- timing hooks
// Timing starts enabled when the process sets MOBA_TIMING=1.
bool timing_from_env() {
  const char* v = std::getenv("MOBA_TIMING");
  return v && v[0] == '1' && v[1] == '\0';
}

struct Timing {
  std::mutex mu;
  bool enabled = timing_from_env();
  double ms[kNumClasses] = {0};
  long long n[kNumClasses] = {0};
  struct Pending { int cls; cudaEvent_t a, b; };
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
Timing& timing() { static Timing t; return t; }

const char* const kClassNames[kNumClasses] = {"moba_centroids", "moba_gate", "moba_route_count",
                                               "moba_route_scan", "moba_route_scatter",
                                               "moba_attention", "moba_merge", "moba_plan",
                                               "moba_densify", "moba_decode",
                                               "moba_bwd_dkdv", "moba_bwd_dq", "moba_bwd_aux"};

// Brackets one kernel launch: an NVTX range named for its class (seen by profilers; a no-op
// otherwise) and, when timing is enabled, CUDA events on the launching stream.
struct Scope {
  int cls; cudaStream_t s; cudaEvent_t a = nullptr, b = nullptr; bool on = false;
  Scope(int c, cudaStream_t st) : cls(c), s(st) {
    nvtxRangePushA(kClassNames[c]);
    Timing& T = timing();
    std::lock_guard<std::mutex> g(T.mu);
    if (T.enabled) { on = true; a = T.get(); b = T.get(); cudaEventRecord(a, s); }
  }
  void done() {
    nvtxRangePop();
    g_launches.fetch_add(1);
    if (!on) return;
    cudaEventRecord(b, s);
    Timing& T = timing();
    std::lock_guard<std::mutex> g(T.mu);
    T.pending.push_back({cls, a, b});
  }
};

// ----------------------------------------------------------------------------------- device
struct DevInfo { int ok = -1; int sms = 0; };
int device_check(int* sms) {
  static DevInfo info[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOBA_ERR_CUDA;
  DevInfo& di = info[dev];
  if (di.ok < 0) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return MOBA_ERR_CUDA;
    di.ok = (p.major == 10 && p.minor == 0) ? 1 : 0;
    di.sms = p.multiProcessorCount;
  }
  if (sms) *sms = di.sms;
  return di.ok ? MOBA_OK : MOBA_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------------------------- plan
struct Chunk { int b0, nblk, T0, ntok; };
struct Plan {
  int T = 0, NB = 0, max_nb = 0;
  std::vector<int> blk_len;  // per global block
  std::vector<Chunk> chunks;
  size_t max_rows = 0, max_entries = 0, max_tiles = 0;
};

int check_cu(int nseq, const int32_t* cu) {
  if (nseq < 1 || nseq > 65535 || !cu) return MOBA_ERR_ARG;
  if (cu[0] != 0) return MOBA_ERR_ARG;
  for (int s = 0; s < nseq; ++s)
    if (cu[s + 1] < cu[s]) return MOBA_ERR_ARG;
  return MOBA_OK;
}

int check_shape(int Hq, int Hkv, int d, int B, int topk) {
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return MOBA_ERR_ARG;
  if (B < 1 || topk < 1) return MOBA_ERR_ARG;
  if (d != 64 && d != 128) return MOBA_ERR_UNSUPPORTED;
  if (B % 64 != 0) return MOBA_ERR_UNSUPPORTED;
  if (topk > kMaxTopk) return MOBA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 256) return MOBA_ERR_UNSUPPORTED;
  return MOBA_OK;
}

int make_plan(int nseq, const int32_t* cu, int Hq, int Hkv, int d, int B, int topk, Plan* P,
              size_t partial_budget = kPartialBudgetBytes) {
  P->T = cu[nseq];
  P->blk_len.clear();
  for (int s = 0; s < nseq; ++s) {
    const int L = cu[s + 1] - cu[s];
    const int nb = blocks_of(L, B);
    if (nb > kMaxBlocksPerSeq) return MOBA_ERR_UNSUPPORTED;
    P->max_nb = std::max(P->max_nb, nb);
    for (int j = 0; j < nb; ++j) P->blk_len.push_back(std::min(B, L - j * B));
  }
  P->NB = static_cast<int>(P->blk_len.size());
  if (static_cast<long long>(P->T) * Hq >= (1LL << 31) / 2) return MOBA_ERR_UNSUPPORTED;
  if (P->max_nb > 65535) return MOBA_ERR_UNSUPPORTED;
  // query chunks of whole blocks, so that partial rows (t, h, slot) fit the budget
  // per partial row: its bf16 output, log-sum-exp and routing entry; at d = 64 also the copy of
  // the routed query row that the attention kernel reads as a dense tile
  const size_t row_bytes =
      static_cast<size_t>(d) * 2 + 4 + 4 + (d == 64 ? static_cast<size_t>(d) * 2 : 0);
  size_t max_rows = std::max<size_t>(partial_budget / row_bytes, 1);
  const size_t per_tok = static_cast<size_t>(Hq) * topk;
  max_rows = std::min<size_t>(max_rows, (1ull << 31) - 1);
  P->chunks.clear();
  int b = 0, t = 0;
  while (b < P->NB) {
    Chunk c{b, 0, t, 0};
    while (b < P->NB) {
      const size_t rows = static_cast<size_t>(c.ntok + P->blk_len[b]) * per_tok;
      if (c.nblk > 0 && rows > max_rows) break;
      if (rows >= (1ull << 31)) return MOBA_ERR_UNSUPPORTED;
      c.ntok += P->blk_len[b];
      c.nblk += 1;
      ++b;
    }
    t += c.ntok;
    P->chunks.push_back(c);
    const size_t rows = static_cast<size_t>(c.ntok) * per_tok;
    const size_t ent = static_cast<size_t>(c.ntok) * Hq * (topk - 1);
    P->max_rows = std::max(P->max_rows, rows);
    P->max_entries = std::max(P->max_entries, ent);
    P->max_tiles = std::max(P->max_tiles, ent / kItemRows + static_cast<size_t>(Hkv) * P->NB + 1);
  }
  return MOBA_OK;
}

// --------------------------------------------------------------------------- workspace carve
struct Layout {
  size_t status, blk_off, blk_seq, blk_start, blk_len, cents, split, idx, counts, cursor, tiles,
      entries, qdense, part_o, part_lse, total;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

Layout layout_of(const Plan& P, int nseq, int Hq, int Hkv, int d, int topk) {
  Layout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = up256(o + bytes); return at; };
  L.status = take(256);
  L.blk_off = take(static_cast<size_t>(nseq + 1) * 4);
  L.blk_seq = take(static_cast<size_t>(P.NB) * 4);
  L.blk_start = take(static_cast<size_t>(P.NB) * 4);
  L.blk_len = take(static_cast<size_t>(P.NB) * 4);
  L.cents = take(static_cast<size_t>(P.NB) * Hkv * d * 4);
  L.split = take(gate_split_bytes(P.NB, Hkv, d));
  L.idx = take(static_cast<size_t>(Hq) * P.T * topk * 4);
  L.counts = take(static_cast<size_t>(Hkv) * P.NB * 4);
  L.cursor = take(static_cast<size_t>(Hkv) * P.NB * 4);
  L.tiles = take(P.max_tiles * 16);
  L.entries = take(std::max<size_t>(P.max_entries, 1) * 4);
  L.qdense = take(d == 64 ? std::max<size_t>(P.max_entries, 1) * d * 2 : 0);
  L.part_o = take(P.max_rows * d * 2);
  L.part_lse = take(P.max_rows * 4);
  L.total = o;
  return L;
}

template <class T>
T* at(void* base, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(base) + off); }

// The tensor-core gates keep at most 32 past blocks per row in registers, so they serve
// topk <= 33; larger topk uses the CUDA-core gate. Sequences of at most 257 blocks take the
// streaming gate (all past centroids resident, query tiles streamed by a producer warp).
cudaError_t run_gate(const void* q, const float* cents, const int32_t* cu_dev,
                     const int32_t* cu_host, int nseq, int max_nb, int T, int H, int G, int d,
                     int B, int topk, int32_t* idx, int* status, int sms, cudaStream_t s,
                     const BlockTables* tb = nullptr, int NB = 0, void* split = nullptr) {
  if (gate_stream_supported(max_nb, topk))
    return launch_gate_stream(q, cents, cu_dev, cu_host, nseq, max_nb, T, H, G, d, B, topk, idx,
                              status, sms, s);
  if (topk <= 33)
    return launch_gate_tc(q, cents, cu_dev, nseq, max_nb, T, H, G, d, B, topk, idx, status, sms, s,
                          tb, NB, split);
  return launch_gate(q, cents, cu_dev, nseq, max_nb, T, H, G, d, B, topk, idx, s);
}

#define MOBA_LAUNCH(cls, stream, expr)                      \
  do {                                                      \
    Scope _sc((cls), (stream));                             \
    cudaError_t _e = (expr);                                \
    _sc.done();                                             \
    if (_e != cudaSuccess) return MOBA_ERR_CUDA;            \
  } while (0)

}  // namespace

extern "C" {

const char* moba_status_string(int status) {
  switch (status) {
    case MOBA_OK: return "MOBA_OK";
    case MOBA_ERR_ARG: return "MOBA_ERR_ARG: invalid argument";
    case MOBA_ERR_UNSUPPORTED: return "MOBA_ERR_UNSUPPORTED: shape or device not supported";
    case MOBA_ERR_WORKSPACE: return "MOBA_ERR_WORKSPACE: workspace too small";
    case MOBA_ERR_CUDA: return "MOBA_ERR_CUDA: CUDA call or kernel launch failed";
    case MOBA_ERR_DEVICE_CHECK: return "MOBA_ERR_DEVICE_CHECK: device-side check failed";
    case MOBA_ERR_TIMEOUT: return "MOBA_ERR_TIMEOUT: a bounded device wait ran out";
    default: return "MOBA_UNKNOWN_STATUS";
  }
}

int moba_version(void) { return (0 << 16) | (1 << 8) | 0; }

size_t moba_workspace_bytes(int nseq, const int32_t* cu_seqlens_host, int Hq, int Hkv, int d,
                            int block_size, int topk) {
  if (check_cu(nseq, cu_seqlens_host) != MOBA_OK) return 0;
  if (check_shape(Hq, Hkv, d, block_size, topk) != MOBA_OK) return 0;
  Plan P;
  if (make_plan(nseq, cu_seqlens_host, Hq, Hkv, d, block_size, topk, &P) != MOBA_OK) return 0;
  return layout_of(P, nseq, Hq, Hkv, d, topk).total;
}

int moba_centroids_kconv(const void* k, const float* conv_w, int conv_width,
                         const int32_t* cu_dev, const int32_t* cu_host, int nseq, int Hkv, int d,
                         int block_size, float* centroids, void* stream) {
  if (!conv_w || !aligned16(conv_w)) return MOBA_ERR_ARG;
  if (conv_width < 1) return MOBA_ERR_ARG;
  if (conv_width > kMaxKconvWidth) return MOBA_ERR_UNSUPPORTED;
  int st = check_cu(nseq, cu_host);
  if (st != MOBA_OK) return st;
  if (Hkv < 1 || block_size < 1) return MOBA_ERR_ARG;
  if (d != 64 && d != 128) return MOBA_ERR_UNSUPPORTED;
  if (block_size % 64 != 0) return MOBA_ERR_UNSUPPORTED;
  Plan P;
  if ((st = make_plan(nseq, cu_host, Hkv, Hkv, d, block_size, 1, &P)) != MOBA_OK) return st;
  if (P.T == 0 || P.NB == 0) return MOBA_OK;
  if (!k || !cu_dev || !centroids || !aligned16(k) || !aligned16(centroids)) return MOBA_ERR_ARG;
  int sms = 0;
  if ((st = device_check(&sms)) != MOBA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOBA_LAUNCH(kCentroid, s,
              launch_centroids(k, cu_dev, nseq, P.max_nb, Hkv, d, block_size, P.NB, sms, centroids,
                               s, conv_w, conv_width));
  return MOBA_OK;
}

int moba_centroids(const void* k, const int32_t* cu_dev, const int32_t* cu_host, int nseq,
                   int Hkv, int d, int block_size, float* centroids, void* stream) {
  int st = check_cu(nseq, cu_host);
  if (st != MOBA_OK) return st;
  if (Hkv < 1 || block_size < 1) return MOBA_ERR_ARG;
  if (d != 64 && d != 128) return MOBA_ERR_UNSUPPORTED;
  if (block_size % 64 != 0) return MOBA_ERR_UNSUPPORTED;
  Plan P;
  if ((st = make_plan(nseq, cu_host, Hkv, Hkv, d, block_size, 1, &P)) != MOBA_OK) return st;
  if (P.T == 0 || P.NB == 0) return MOBA_OK;
  if (!k || !cu_dev || !centroids || !aligned16(k) || !aligned16(centroids)) return MOBA_ERR_ARG;
  int sms = 0;
  if ((st = device_check(&sms)) != MOBA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOBA_LAUNCH(kCentroid, s,
              launch_centroids(k, cu_dev, nseq, P.max_nb, Hkv, d, block_size, P.NB, sms, centroids, s));
  return MOBA_OK;
}

int moba_gate_topk(const void* q, const float* centroids, const int32_t* cu_dev,
                   const int32_t* cu_host, int nseq, int Hq, int Hkv, int d, int block_size,
                   int topk, int32_t* block_idx, void* stream) {
  int st = check_cu(nseq, cu_host);
  if (st != MOBA_OK) return st;
  if ((st = check_shape(Hq, Hkv, d, block_size, topk)) != MOBA_OK) return st;
  Plan P;
  if ((st = make_plan(nseq, cu_host, Hq, Hkv, d, block_size, topk, &P)) != MOBA_OK) return st;
  if (P.T == 0) return MOBA_OK;
  if (!q || !centroids || !cu_dev || !block_idx || !aligned16(q) || !aligned16(centroids) ||
      !aligned16(block_idx))
    return MOBA_ERR_ARG;
  int sms = 0;
  if ((st = device_check(&sms)) != MOBA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOBA_LAUNCH(kGate, s,
              run_gate(q, centroids, cu_dev, cu_host, nseq, P.max_nb, P.T, Hq, Hkv, d,
                       block_size, topk, block_idx, nullptr, sms, s));
  return MOBA_OK;
}

}  // extern "C"

namespace moba {

// Body of moba_attn_fwd; `partial_budget` bounds the partial outputs of one query chunk.
int attn_fwd_impl(const void* q, const void* k, const void* v, const int32_t* cu_dev,
                  const int32_t* cu_host, int nseq, int Hq, int Hkv, int d, int block_size,
                  int topk, float scale, const int32_t* block_idx_in, int32_t* block_idx_out,
                  void* o, float* lse, void* workspace, size_t workspace_bytes, void* stream,
                  size_t partial_budget, const float* conv_w, int conv_width) {
  int st = check_cu(nseq, cu_host);
  if (st != MOBA_OK) return st;
  if (conv_w && (!aligned16(conv_w) || conv_width < 1)) return MOBA_ERR_ARG;
  if (conv_w && conv_width > kMaxKconvWidth) return MOBA_ERR_UNSUPPORTED;
  if ((st = check_shape(Hq, Hkv, d, block_size, topk)) != MOBA_OK) return st;
  if (!(scale > 0.f) || scale > 1e30f) return MOBA_ERR_ARG;
  Plan P;
  if ((st = make_plan(nseq, cu_host, Hq, Hkv, d, block_size, topk, &P, partial_budget)) != MOBA_OK)
    return st;
  if (P.T == 0) return MOBA_OK;
  if (!q || !k || !v || !cu_dev || !o || !lse || !workspace) return MOBA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return MOBA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOBA_ERR_ARG;
  if ((block_idx_in && !aligned16(block_idx_in)) || (block_idx_out && !aligned16(block_idx_out)))
    return MOBA_ERR_ARG;
  const Layout L = layout_of(P, nseq, Hq, Hkv, d, topk);
  if (workspace_bytes < L.total) return MOBA_ERR_WORKSPACE;
  int sms = 0;
  if ((st = device_check(&sms)) != MOBA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  BlockTables tb;
  tb.blk_off = at<int>(workspace, L.blk_off);
  tb.blk_seq = at<int>(workspace, L.blk_seq);
  tb.blk_start = at<int>(workspace, L.blk_start);
  tb.blk_len = at<int>(workspace, L.blk_len);
  int* status = at<int>(workspace, L.status);
  int* n_tiles = status + 1;
  int* counts = at<int>(workspace, L.counts);
  int* cursor = at<int>(workspace, L.cursor);
  int4* tiles = at<int4>(workspace, L.tiles);
  int* entries = at<int>(workspace, L.entries);
  void* part_o = at<void>(workspace, L.part_o);
  float* part_lse = at<float>(workspace, L.part_lse);
  float* cents = at<float>(workspace, L.cents);
  void* qdense = (d == 64) ? at<void>(workspace, L.qdense) : nullptr;
  const int NBK = Hkv * P.NB;

  MOBA_LAUNCH(kPlan, s, launch_plan(cu_dev, nseq, block_size, P.NB, tb, counts, NBK, status, s));

  const int32_t* idx = block_idx_in;
  if (!idx) {
    int32_t* idx_w = block_idx_out ? block_idx_out : at<int32_t>(workspace, L.idx);
    MOBA_LAUNCH(kCentroid, s,
                launch_centroids(k, cu_dev, nseq, P.max_nb, Hkv, d, block_size, P.NB, sms, cents, s,
                                 conv_w, conv_width));
    MOBA_LAUNCH(kGate, s,
                run_gate(q, cents, cu_dev, cu_host, nseq, P.max_nb, P.T, Hq, Hkv, d, block_size,
                         topk, idx_w, status, sms, s, &tb, P.NB, at<void>(workspace, L.split)));
    idx = idx_w;
  } else if (block_idx_out && block_idx_out != block_idx_in) {
    if (cudaMemcpyAsync(block_idx_out, block_idx_in, static_cast<size_t>(Hq) * P.T * topk * 4,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return MOBA_ERR_CUDA;
  }

  for (const Chunk& c : P.chunks) {
    MOBA_LAUNCH(kRouteCount, s,
                launch_route_count(idx, tb, P.T, Hq, Hkv, topk, P.NB, c.b0, c.nblk, c.T0, P.max_nb,
                                   counts, status, s));
    MOBA_LAUNCH(kRouteScan, s,
                launch_route_scan(counts, NBK, cursor, tiles, n_tiles,
                                  static_cast<long long>(P.max_tiles), status, s));
    MOBA_LAUNCH(kRouteScatter, s,
                launch_route_scatter(idx, tb, P.T, Hq, Hkv, topk, P.NB, c.b0, c.nblk, c.T0,
                                     P.max_nb, cursor, entries,
                                     static_cast<long long>(std::max<size_t>(P.max_entries, 1)),
                                     status, s));
    if (qdense)
      MOBA_LAUNCH(kDensify, s,
                  launch_densify(entries, n_tiles + 1, q, Hq, topk, c.T0,
                                 static_cast<long long>(P.max_entries), qdense, sms,
                                 static_cast<long long>(P.T) * Hq, status, s));
    AttnLaunch A;
    A.q = q; A.k = k; A.v = v;
    A.tiles = tiles; A.n_routed = n_tiles; A.entries = entries; A.tb = tb;
    A.qdense = qdense;
    A.qdense_rows = static_cast<long long>(std::max<size_t>(P.max_entries, 1));
    A.rows_cap = static_cast<long long>(P.max_rows);
    A.part_o = part_o; A.part_lse = part_lse; A.status = status;
    A.T = P.T; A.H = Hq; A.G = Hkv; A.d = d; A.B = block_size; A.topk = topk; A.NB = P.NB;
    A.b0 = c.b0; A.nblk = c.nblk; A.T0 = c.T0; A.scale = scale;
    A.wait_ns = g_wait_limit_ns.load();
    A.diag_stall = g_diag_stall.load();
    const long long P256 = (block_size + kItemRows - 1) / kItemRows;
    const long long items = static_cast<long long>(P.max_tiles) + P256 * c.nblk * Hq;
    A.grid = static_cast<int>(std::min<long long>(sms, items));
    MOBA_LAUNCH(kAttn, s, launch_attention(A, s));
    MOBA_LAUNCH(kMerge, s,
                launch_merge(part_o, part_lse, cu_dev, nseq, P.T, Hq, d, block_size, topk, c.T0,
                             c.ntok, o, lse, s));
  }
  return MOBA_OK;
}

int read_status_word(const void* word_dev, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyAsync(&word, word_dev, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOBA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOBA_ERR_CUDA;
  if (word == 0) return MOBA_OK;
  if (word == kDevTimeoutAttn || word == kDevDrainTimeout) return MOBA_ERR_TIMEOUT;
  // kDevBadRouting, kDevSmemAlign, kDevCheckFail
  return MOBA_ERR_DEVICE_CHECK;
}

size_t workspace_bytes_for(int nseq, const int32_t* cu_host, int Hq, int Hkv, int d,
                           int block_size, int topk, size_t partial_budget) {
  if (check_cu(nseq, cu_host) != MOBA_OK) return 0;
  if (check_shape(Hq, Hkv, d, block_size, topk) != MOBA_OK) return 0;
  Plan P;
  if (make_plan(nseq, cu_host, Hq, Hkv, d, block_size, topk, &P, partial_budget) != MOBA_OK)
    return 0;
  return layout_of(P, nseq, Hq, Hkv, d, topk).total;
}

}  // namespace moba

extern "C" {

int moba_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_dev,
                  const int32_t* cu_host, int nseq, int Hq, int Hkv, int d, int block_size,
                  int topk, float scale, const int32_t* block_idx_in, int32_t* block_idx_out,
                  void* o, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  return attn_fwd_impl(q, k, v, cu_dev, cu_host, nseq, Hq, Hkv, d, block_size, topk, scale,
                       block_idx_in, block_idx_out, o, lse, workspace, workspace_bytes, stream,
                       kPartialBudgetBytes);
}

int moba_attn_fwd_kconv(const void* q, const void* k, const void* v, const float* conv_w,
                        int conv_width, const int32_t* cu_dev, const int32_t* cu_host, int nseq,
                        int Hq, int Hkv, int d, int block_size, int topk, float scale,
                        int32_t* block_idx_out, void* o, float* lse, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!conv_w) return MOBA_ERR_ARG;
  return attn_fwd_impl(q, k, v, cu_dev, cu_host, nseq, Hq, Hkv, d, block_size, topk, scale,
                       nullptr, block_idx_out, o, lse, workspace, workspace_bytes, stream,
                       kPartialBudgetBytes, conv_w, conv_width);
}

}  // extern "C"

namespace {

// Host-side plan of a decode / chunked-prefill call: cache blocks and the query rows.
struct DecodePlan {
  int T = 0, Tq = 0, NB = 0, max_nb = 0;
};

int decode_plan(int nseq, const int32_t* cu, const int32_t* cuq, int Hq, int Hkv, int d, int B,
                int topk, DecodePlan* P) {
  int st = check_cu(nseq, cu);
  if (st != MOBA_OK) return st;
  if ((st = check_cu(nseq, cuq)) != MOBA_OK) return st;
  if ((st = check_shape(Hq, Hkv, d, B, topk)) != MOBA_OK) return st;
  for (int s = 0; s < nseq; ++s) {
    const int L = cu[s + 1] - cu[s], n = cuq[s + 1] - cuq[s];
    if (n > L) return MOBA_ERR_ARG;  // query rows are the newest tokens of the cache
    const int nb = blocks_of(L, B);
    if (nb > kMaxBlocksPerSeq) return MOBA_ERR_UNSUPPORTED;
    P->max_nb = std::max(P->max_nb, nb);
    P->NB += nb;
  }
  P->T = cu[nseq];
  P->Tq = cuq[nseq];
  if (static_cast<long long>(P->Tq) * Hq >= (1LL << 31) / 2) return MOBA_ERR_UNSUPPORTED;
  if (static_cast<long long>(P->T) * Hkv >= (1LL << 31) / 2) return MOBA_ERR_UNSUPPORTED;
  return MOBA_OK;
}

struct DecodeLayout {
  size_t status, blk_off, blk_seq, blk_start, blk_len, idx, part, total;
};

DecodeLayout decode_layout(const DecodePlan& P, int nseq, int Hq, int d, int B, int topk) {
  DecodeLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = up256(o + bytes); return at; };
  L.status = take(256);
  L.blk_off = take(static_cast<size_t>(nseq + 1) * 4);
  L.blk_seq = take(static_cast<size_t>(P.NB) * 4);
  L.blk_start = take(static_cast<size_t>(P.NB) * 4);
  L.blk_len = take(static_cast<size_t>(P.NB) * 4);
  L.idx = take(static_cast<size_t>(Hq) * P.Tq * topk * 4);
  L.part = take(static_cast<size_t>(P.Tq) * Hq * decode_parts(B, topk) * (d + 2) * 4);
  L.total = o;
  return L;
}

}  // namespace

extern "C" {

size_t moba_decode_workspace_bytes(int nseq, const int32_t* cu_host, const int32_t* cuq_host,
                                   int Hq, int Hkv, int d, int block_size, int topk) {
  DecodePlan P;
  if (decode_plan(nseq, cu_host, cuq_host, Hq, Hkv, d, block_size, topk, &P) != MOBA_OK) return 0;
  return decode_layout(P, nseq, Hq, d, block_size, topk).total;
}

int moba_decode_fwd(const void* q, const void* k_cache, const void* v_cache,
                    const float* centroids, const int32_t* cu_dev, const int32_t* cu_host,
                    const int32_t* cuq_dev, const int32_t* cuq_host, int nseq, int Hq, int Hkv,
                    int d, int block_size, int topk, float scale, const int32_t* block_idx_in,
                    int32_t* block_idx_out, void* o, float* lse, void* workspace,
                    size_t workspace_bytes, void* stream) {
  DecodePlan P;
  int st = decode_plan(nseq, cu_host, cuq_host, Hq, Hkv, d, block_size, topk, &P);
  if (st != MOBA_OK) return st;
  if (!(scale > 0.f) || scale > 1e30f) return MOBA_ERR_ARG;
  if (P.Tq == 0) return MOBA_OK;
  if (!q || !k_cache || !v_cache || !cu_dev || !cuq_dev || !o || !lse || !workspace)
    return MOBA_ERR_ARG;
  if (!block_idx_in && !centroids) return MOBA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      !aligned16(lse) || (centroids && !aligned16(centroids)))
    return MOBA_ERR_ARG;
  if ((block_idx_in && !aligned16(block_idx_in)) || (block_idx_out && !aligned16(block_idx_out)))
    return MOBA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOBA_ERR_ARG;
  const DecodeLayout L = decode_layout(P, nseq, Hq, d, block_size, topk);
  if (workspace_bytes < L.total) return MOBA_ERR_WORKSPACE;
  int sms = 0;
  if ((st = device_check(&sms)) != MOBA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  BlockTables tb;
  tb.blk_off = at<int>(workspace, L.blk_off);
  tb.blk_seq = at<int>(workspace, L.blk_seq);
  tb.blk_start = at<int>(workspace, L.blk_start);
  tb.blk_len = at<int>(workspace, L.blk_len);
  int* status = at<int>(workspace, L.status);
  MOBA_LAUNCH(kPlan, s, launch_plan(cu_dev, nseq, block_size, P.NB, tb, nullptr, 0, status, s));
  int32_t* idx = block_idx_out ? block_idx_out : at<int32_t>(workspace, L.idx);
  if (block_idx_in && idx != block_idx_in) {
    if (cudaMemcpyAsync(idx, block_idx_in, static_cast<size_t>(Hq) * P.Tq * topk * 4,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return MOBA_ERR_CUDA;
  }
  DecodeLaunch D;
  D.q = q; D.k = k_cache; D.v = v_cache; D.cents = centroids;
  D.cu = cu_dev; D.cuq = cuq_dev; D.blk_off = tb.blk_off;
  D.idx = idx; D.idx_given = block_idx_in != nullptr;
  D.part = at<float>(workspace, L.part);
  D.o = o; D.lse = lse;
  D.nseq = nseq; D.Tq = P.Tq; D.H = Hq; D.G = Hkv; D.d = d; D.B = block_size; D.topk = topk;
  D.max_nb = P.max_nb; D.scale = scale;
  MOBA_LAUNCH(kDecode, s, launch_decode(D, s));
  return MOBA_OK;
}

}  // extern "C"

namespace {

constexpr size_t kBwdDenseBudgetBytes = 16ull << 30;  // routed rows of one chunk, densified

// Host-side plan of the backward pass: query chunks of whole blocks whose routed entries, with
// their densified query / dO rows and per-row columns, fit the budget.
struct BwdPlan {
  Plan P;
  std::vector<Chunk> chunks;
  size_t max_entries = 0;   // largest chunk
  size_t last_entries = 0;  // the chunk being filled
};

int bwd_plan(int nseq, const int32_t* cu, int Hq, int Hkv, int d, int B, int topk, BwdPlan* BP) {
  int st = check_cu(nseq, cu);
  if (st != MOBA_OK) return st;
  if ((st = check_shape(Hq, Hkv, d, B, topk)) != MOBA_OK) return st;
  if ((st = make_plan(nseq, cu, Hq, Hkv, d, B, topk, &BP->P, ~static_cast<size_t>(0) >> 1)) !=
      MOBA_OK)
    return st;
  const size_t per_entry = 4 + static_cast<size_t>(d) * 4 + 12;
  const size_t max_ent = std::max<size_t>(kBwdDenseBudgetBytes / per_entry, 1);
  BP->chunks.clear();
  BP->max_entries = 0;
  int b = 0, t = 0;
  for (int s = 0; s < nseq; ++s) {
    const int L = cu[s + 1] - cu[s];
    for (int i = 0; i < blocks_of(L, B); ++i, ++b) {
      const int n = std::min(B, L - i * B);
      const size_t ent = static_cast<size_t>(n) * Hq * (std::min(topk, i + 1) - 1);
      if (BP->chunks.empty() ||
          (BP->chunks.back().nblk > 0 && BP->last_entries + ent > max_ent)) {
        BP->chunks.push_back(Chunk{b, 0, t, 0});
        BP->last_entries = 0;
      }
      Chunk& c = BP->chunks.back();
      c.nblk += 1;
      c.ntok += n;
      BP->last_entries += ent;
      BP->max_entries = std::max(BP->max_entries, BP->last_entries);
      if (static_cast<long long>(c.ntok) * Hq * topk >= (1LL << 31)) return MOBA_ERR_UNSUPPORTED;
      t += n;
    }
  }
  return MOBA_OK;
}

struct BwdLayout {
  size_t status, blk_off, blk_seq, blk_start, blk_len, counts, cursor, tiles, entries, qd, dd,
      col_lse, col_d, col_t, dsum, dq_acc, dk_acc, dv_acc, total;
};

BwdLayout bwd_layout(const BwdPlan& BP, int nseq, int Hq, int Hkv, int d) {
  const Plan& P = BP.P;
  BwdLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = up256(o + bytes); return at; };
  const size_t rows = static_cast<size_t>(P.T) * Hq;
  const size_t ent = std::max<size_t>(BP.max_entries, 1);
  L.status = take(256);
  L.blk_off = take(static_cast<size_t>(nseq + 1) * 4);
  L.blk_seq = take(static_cast<size_t>(P.NB) * 4);
  L.blk_start = take(static_cast<size_t>(P.NB) * 4);
  L.blk_len = take(static_cast<size_t>(P.NB) * 4);
  L.counts = take(static_cast<size_t>(Hkv) * P.NB * 4);
  L.cursor = take(static_cast<size_t>(Hkv) * P.NB * 4);
  L.tiles = take((ent / kItemRows + static_cast<size_t>(Hkv) * P.NB + 1) * 16);
  L.entries = take(ent * 4);
  L.qd = take(ent * d * 2);
  L.dd = take(ent * d * 2);
  L.col_lse = take(ent * 4);
  L.col_d = take(ent * 4);
  L.col_t = take(ent * 4);
  L.dsum = take(rows * 4);
  L.dq_acc = take(rows * d * 4);
  L.dk_acc = take(static_cast<size_t>(P.T) * Hkv * d * 4);
  L.dv_acc = take(static_cast<size_t>(P.T) * Hkv * d * 4);
  L.total = o;
  return L;
}

}  // namespace

extern "C" {

size_t moba_bwd_workspace_bytes(int nseq, const int32_t* cu_seqlens_host, int Hq, int Hkv, int d,
                                int block_size, int topk) {
  BwdPlan BP;
  if (bwd_plan(nseq, cu_seqlens_host, Hq, Hkv, d, block_size, topk, &BP) != MOBA_OK) return 0;
  return bwd_layout(BP, nseq, Hq, Hkv, d).total;
}

int moba_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* d_o, const int32_t* block_idx, const int32_t* cu_dev,
                  const int32_t* cu_host, int nseq, int Hq, int Hkv, int d, int block_size,
                  int topk, float scale, void* dq, void* dk, void* dv, void* workspace,
                  size_t workspace_bytes, void* stream) {
  BwdPlan BP;
  int st = bwd_plan(nseq, cu_host, Hq, Hkv, d, block_size, topk, &BP);
  if (st != MOBA_OK) return st;
  const Plan& P = BP.P;
  if (!(scale > 0.f) || scale > 1e30f) return MOBA_ERR_ARG;
  if (P.T == 0) return MOBA_OK;
  const void* ptrs[] = {q, k, v, o, lse, d_o, block_idx, dq, dk, dv};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MOBA_ERR_ARG;
  if (!cu_dev || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return MOBA_ERR_ARG;
  const BwdLayout L = bwd_layout(BP, nseq, Hq, Hkv, d);
  if (workspace_bytes < L.total) return MOBA_ERR_WORKSPACE;
  int sms = 0;
  if ((st = device_check(&sms)) != MOBA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  BlockTables tb;
  tb.blk_off = at<int>(workspace, L.blk_off);
  tb.blk_seq = at<int>(workspace, L.blk_seq);
  tb.blk_start = at<int>(workspace, L.blk_start);
  tb.blk_len = at<int>(workspace, L.blk_len);
  int* status = at<int>(workspace, L.status);
  int* n_tiles = status + 1;
  int* counts = at<int>(workspace, L.counts);
  int* cursor = at<int>(workspace, L.cursor);
  int4* tiles = at<int4>(workspace, L.tiles);
  int* entries = at<int>(workspace, L.entries);
  const int NBK = Hkv * P.NB;
  BwdLaunch B;
  B.q = q; B.k = k; B.v = v; B.o = o; B.dout = d_o; B.lse = lse;
  B.entries = entries; B.bucket_end = cursor; B.tiles = tiles; B.n_routed = n_tiles;
  B.tb = tb;
  B.dsum = at<float>(workspace, L.dsum);
  B.dq_acc = at<float>(workspace, L.dq_acc);
  B.dk_acc = at<float>(workspace, L.dk_acc);
  B.dv_acc = at<float>(workspace, L.dv_acc);
  B.qd = at<void>(workspace, L.qd);
  B.dd = at<void>(workspace, L.dd);
  B.col_lse = at<float>(workspace, L.col_lse);
  B.col_d = at<float>(workspace, L.col_d);
  B.col_t = at<int>(workspace, L.col_t);
  B.dense_rows = static_cast<long long>(std::max<size_t>(BP.max_entries, 1));
  B.dq = dq; B.dk = dk; B.dv = dv; B.status = status;
  B.T = P.T; B.H = Hq; B.G = Hkv; B.d = d; B.B = block_size; B.topk = topk; B.NB = P.NB;
  B.num_sms = sms; B.scale = scale;
  B.T0 = 0; B.b0 = 0; B.nblk = P.NB;
  B.wait_ns = g_wait_limit_ns.load();
  MOBA_LAUNCH(kPlan, s, launch_plan(cu_dev, nseq, block_size, P.NB, tb, counts, NBK, status, s));
  MOBA_LAUNCH(kBwdAux, s, launch_bwd_pre(B, s));
  for (const Chunk& c : BP.chunks) {
    B.T0 = c.T0; B.b0 = c.b0; B.nblk = c.nblk;
    MOBA_LAUNCH(kRouteCount, s,
                launch_route_count(block_idx, tb, P.T, Hq, Hkv, topk, P.NB, c.b0, c.nblk, c.T0,
                                   P.max_nb, counts, status, s));
    MOBA_LAUNCH(kRouteScan, s,
                launch_route_scan(counts, NBK, cursor, tiles, n_tiles,
                                  static_cast<long long>(BP.max_entries / kItemRows + NBK + 1),
                                  status, s));
    MOBA_LAUNCH(kRouteScatter, s,
                launch_route_scatter(block_idx, tb, P.T, Hq, Hkv, topk, P.NB, c.b0, c.nblk, c.T0,
                                     P.max_nb, cursor, entries, B.dense_rows, status, s));
    MOBA_LAUNCH(kBwdAux, s, launch_bwd_densify(B, s));
    MOBA_LAUNCH(kBwdDkdv, s, launch_bwd_dkdv(B, s));
    MOBA_LAUNCH(kBwdDq, s, launch_bwd_dq(B, s));
  }
  MOBA_LAUNCH(kBwdAux, s, launch_bwd_finish(B, s));
  return MOBA_OK;
}

int moba_device_status(const void* workspace, void* stream) {
  if (!workspace) return MOBA_ERR_ARG;
  return moba::read_status_word(workspace, stream);
}

unsigned long long moba_set_wait_limit_ns(unsigned long long ns) {
  const unsigned long long was = g_wait_limit_ns.exchange(ns);
  return was ? was : kWaitTimeoutNs;
}

int moba_set_diag_stall(int on) { return g_diag_stall.exchange(on != 0 ? 1 : 0); }

int moba_timing_enable(int enable) {
  Timing& T = timing();
  std::lock_guard<std::mutex> g(T.mu);
  const int was = T.enabled ? 1 : 0;
  T.enabled = enable != 0;
  return was;
}

int moba_timing_reset(void) {
  Timing& T = timing();
  std::lock_guard<std::mutex> g(T.mu);
  for (auto& p : T.pending) {
    cudaEventSynchronize(p.b);
    T.pool.push_back(p.a);
    T.pool.push_back(p.b);
  }
  T.pending.clear();
  for (int c = 0; c < kNumClasses; ++c) { T.ms[c] = 0; T.n[c] = 0; }
  return MOBA_OK;
}

int moba_timing_read(double* ms_per_class, long long* launches_per_class, int n) {
  Timing& T = timing();
  std::lock_guard<std::mutex> g(T.mu);
  for (auto& p : T.pending) {
    if (cudaEventSynchronize(p.b) != cudaSuccess) return MOBA_ERR_CUDA;
    float ms = 0.f;
    cudaEventElapsedTime(&ms, p.a, p.b);
    T.ms[p.cls] += ms;
    T.n[p.cls] += 1;
    T.pool.push_back(p.a);
    T.pool.push_back(p.b);
  }
  T.pending.clear();
  for (int c = 0; c < kNumClasses && c < n; ++c) {
    if (ms_per_class) ms_per_class[c] = T.ms[c];
    if (launches_per_class) launches_per_class[c] = T.n[c];
  }
  return kNumClasses;
}

long long moba_launch_count(void) { return g_launches.load(); }

}  // extern "C"
