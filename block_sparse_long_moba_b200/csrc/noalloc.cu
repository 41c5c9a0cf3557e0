// moba_attn_fwd_noalloc: the forward pass for callers that cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc (or to ask anyone else to allocate for them):
// plug-in code running inside a host application whose device memory is entirely owned by that
// application's own allocator or fixed memory pool, and latency-critical paths where a
// cudaMalloc — which may implicitly synchronise the device — is not acceptable. This entry point
// runs the same kernels as moba_attn_fwd but takes its scratch memory (block tables, centroids,
// routing, routing lists and per-block partial outputs) from one statically sized device array
// that is part of the library, so the caller passes only inputs and outputs.
//
// Limits and sharing rules:
//   * The array holds MOBA_NOALLOC_SCRATCH_BYTES (64 MiB). Every GPU that loads the library keeps
//     that much memory reserved until the process exits.
//   * Problems whose scratch need exceeds the array are rejected with MOBA_ERR_WORKSPACE before
//     anything is launched. The query range is processed in chunks so that partial outputs stay
//     within a quarter of the array; the routing itself ([Hq, T, topk] int32) must fit too.
//   * Every call uses the same array and leaves its contents behind; each call re-initialises
//     what has to start at zero (bucket counters, status word) on the stream before use.
//     Calls whose work overlaps on the GPU (several streams, several host threads) race on the
//     array: serialise them.
//   * The first call on each device looks up the array's device address (cudaGetSymbolAddress,
//     with that device current). Make that first call before any stream capture begins.
//   * The device status word of a call (a bounded wait that ran out, a routing row that broke
//     its contract) sits at the start of the array; moba_noalloc_status reads it.
#include <mutex>

#include "../../include/moba.h"
#include "launch.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOBA_NOALLOC_SCRATCH_BYTES];

constexpr size_t kNoallocPartialBudget = MOBA_NOALLOC_SCRATCH_BYTES / 4;

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

// Device address of the scratch array on the current device (set up once per device).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOBA_ERR_CUDA;
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOBA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOBA_OK;
}

}  // namespace

extern "C" int moba_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                     const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                                     int nseq, int Hq, int Hkv, int d, int block_size, int topk,
                                     float scale, void* o, float* lse, void* stream) {
  if (!cu_seqlens_host || nseq < 1) return MOBA_ERR_ARG;
  const size_t need = moba::workspace_bytes_for(nseq, cu_seqlens_host, Hq, Hkv, d, block_size,
                                                topk, kNoallocPartialBudget);
  if (need == 0) {
    // invalid arguments: let the shared validation report the precise status
    return moba::attn_fwd_impl(q, k, v, cu_seqlens_dev, cu_seqlens_host, nseq, Hq, Hkv, d,
                               block_size, topk, scale, nullptr, nullptr, o, lse, nullptr, 0,
                               stream, kNoallocPartialBudget);
  }
  if (need > MOBA_NOALLOC_SCRATCH_BYTES) return MOBA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != MOBA_OK) return st;
  return moba::attn_fwd_impl(q, k, v, cu_seqlens_dev, cu_seqlens_host, nseq, Hq, Hkv, d,
                             block_size, topk, scale, nullptr, nullptr, o, lse, scratch,
                             MOBA_NOALLOC_SCRATCH_BYTES, stream, kNoallocPartialBudget);
}

extern "C" int moba_noalloc_status(void* stream) {
  void* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != MOBA_OK) return st;
  return moba::read_status_word(scratch, stream);
}
