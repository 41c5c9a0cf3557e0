// K5 — LSE-weighted merge of the per-block partial results of every (t, h) row.
//
// Each selected block s of a row left a normalised partial O_s (bf16, = sum_u p_u v_u / l_s) and
// its log-sum-exp lse_s (fp32, natural log). With M = max_s lse_s and w_s = exp(lse_s - M):
//   O = sum_s w_s O_s / sum_s w_s,   LSE = M + log(sum_s w_s),
// which equals one softmax over the union of the selected blocks' keys
// [MoBA paper summary (atlas.scime.ai), "Approach": exact attention over the routed blocks].
// HBM-bound: one warp per (t, h) row reads the row's k contiguous partial slots once.
#include "common.cuh"
#include "launch.h"

namespace moba {

// A row's k partial slots are contiguous (k * D bf16). Every lane reads 16 bytes per instruction,
// so one warp instruction covers SPI = 32 / (D / 8) whole slots (4 at d = 64, 2 at d = 128); all
// NIT instructions of a row are issued before any is used (predicated off past the row's n slots),
// which keeps enough bytes in flight to run at HBM speed. The lane groups are summed by shuffles.
template <int D, int NIT>
__global__ void __launch_bounds__(256) merge_kernel(const __nv_bfloat16* __restrict__ part_o,
                                                    const float* __restrict__ part_lse,
                                                    const int32_t* __restrict__ cu, int nseq,
                                                    int T, int H, int B, int topk, int T0,
                                                    int ntok, __nv_bfloat16* __restrict__ o,
                                                    float* __restrict__ lse) {
  constexpr int LPS = D / 8;     // lanes per slot (16-byte chunks of one partial row)
  constexpr int SPI = 32 / LPS;  // slots per warp instruction
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= ntok * H) return;
  const int tl = warp / H, h = warp % H;
  const int t = T0 + tl;
  int lo = 0, hi = nseq;  // sequence of t: largest s with cu[s] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  const int i = (t - __ldg(cu + lo)) / B;
  const int n = min(topk, i + 1);
  const size_t p0 = (static_cast<size_t>(tl) * H + h) * topk;
  // partial rows first (the bulk of the bytes), then the slot weights
  const int sub = lane / LPS, ch = lane % LPS;
  const uint4* src = reinterpret_cast<const uint4*>(part_o + p0 * D) + ch;
  uint4 v[NIT];
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    const int sl = it * SPI + sub;
    v[it] = sl < n ? __ldcs(src + static_cast<size_t>(sl) * LPS) : make_uint4(0, 0, 0, 0);
  }
  const float l0 = lane < n ? __ldcs(part_lse + p0 + lane) : -INFINITY;
  const float l1 = lane + 32 < n ? __ldcs(part_lse + p0 + lane + 32) : -INFINITY;
  float m = fmaxf(l0, l1);
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, x));
  const float w0 = lane < n ? __expf(l0 - m) : 0.f;
  const float w1 = lane + 32 < n ? __expf(l1 - m) : 0.f;
  float wsum = w0 + w1;
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, x);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    const int sl = it * SPI + sub;  // the SPI slots of one instruction are all < 32 or all >= 32
    const float w = __shfl_sync(0xffffffffu, it * SPI < 32 ? w0 : w1, sl & 31);
    const uint32_t x[4] = {v[it].x, v[it].y, v[it].z, v[it].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += w * __uint_as_float(x[e] << 16);
      acc[2 * e + 1] += w * __uint_as_float(x[e] & 0xffff0000u);
    }
  }
#pragma unroll
  for (int x = LPS; x < 32; x <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], x);
  }
  if (lane < LPS) {
    const float inv = 1.f / wsum;
    uint4 pk;
    __nv_bfloat162 b0 = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
    __nv_bfloat162 b1 = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
    __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[4] * inv, acc[5] * inv);
    __nv_bfloat162 b3 = __floats2bfloat162_rn(acc[6] * inv, acc[7] * inv);
    pk.x = *reinterpret_cast<uint32_t*>(&b0);
    pk.y = *reinterpret_cast<uint32_t*>(&b1);
    pk.z = *reinterpret_cast<uint32_t*>(&b2);
    pk.w = *reinterpret_cast<uint32_t*>(&b3);
    reinterpret_cast<uint4*>(o + (static_cast<size_t>(t) * H + h) * D)[ch] = pk;
  }
  if (lane == 0) lse[static_cast<size_t>(h) * T + t] = m + __logf(wsum);
}

template <int D>
static cudaError_t launch_merge_d(const __nv_bfloat16* po, const float* part_lse,
                                  const int32_t* cu_dev, int nseq, int T, int H, int B, int topk,
                                  int T0, int ntok, __nv_bfloat16* op, float* lse, unsigned grid,
                                  cudaStream_t stream) {
  constexpr int SPI = 32 / (D / 8);
  const int nit = (topk + SPI - 1) / SPI;
#define MOBA_MERGE(N)                                                                          \
  merge_kernel<D, N><<<grid, 256, 0, stream>>>(po, part_lse, cu_dev, nseq, T, H, B, topk, T0, \
                                               ntok, op, lse)
  if (nit <= 1) MOBA_MERGE(1);
  else if (nit <= 2) MOBA_MERGE(2);
  else if (nit <= 4) MOBA_MERGE(4);
  else if (nit <= 8) MOBA_MERGE(8);
  else if (nit <= 16) MOBA_MERGE(16);
  else MOBA_MERGE(32);
#undef MOBA_MERGE
  return cudaGetLastError();
}

cudaError_t launch_merge(const void* part_o, const float* part_lse, const int32_t* cu_dev,
                         int nseq, int T, int H, int d, int B, int topk, int T0, int ntok,
                         void* o, float* lse, cudaStream_t stream) {
  const long long warps = static_cast<long long>(ntok) * H;
  const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
  if (grid == 0) return cudaSuccess;
  const __nv_bfloat16* po = static_cast<const __nv_bfloat16*>(part_o);
  __nv_bfloat16* op = static_cast<__nv_bfloat16*>(o);
  if (topk > kMaxTopk) return cudaErrorInvalidValue;
  if (d == 64)
    return launch_merge_d<64>(po, part_lse, cu_dev, nseq, T, H, B, topk, T0, ntok, op, lse, grid,
                              stream);
  return launch_merge_d<128>(po, part_lse, cu_dev, nseq, T, H, B, topk, T0, ntok, op, lse, grid,
                             stream);
}

}  // namespace moba
