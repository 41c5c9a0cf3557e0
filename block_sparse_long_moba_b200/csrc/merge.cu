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

template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const __nv_bfloat16* __restrict__ part_o,
                                                    const float* __restrict__ part_lse,
                                                    const int32_t* __restrict__ cu, int nseq,
                                                    int T, int H, int B, int topk, int T0,
                                                    int ntok, __nv_bfloat16* __restrict__ o,
                                                    float* __restrict__ lse) {
  constexpr int EPL = D / 32;  // elements per lane: 2 (d=64) or 4 (d=128)
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
  const float l0 = lane < n ? __ldg(part_lse + p0 + lane) : -INFINITY;
  const float l1 = lane + 32 < n ? __ldg(part_lse + p0 + lane + 32) : -INFINITY;
  float m = fmaxf(l0, l1);
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, x));
  const float w0 = lane < n ? __expf(l0 - m) : 0.f;
  const float w1 = lane + 32 < n ? __expf(l1 - m) : 0.f;
  float wsum = w0 + w1;
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, x);
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  const __nv_bfloat16* src = part_o + p0 * D + lane * EPL;
  for (int sl = 0; sl < n; ++sl) {
    const float w = __shfl_sync(0xffffffffu, sl < 32 ? w0 : w1, sl & 31);
    if (EPL == 4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(src + static_cast<size_t>(sl) * D));
      acc[0] += w * __uint_as_float(v.x << 16);
      acc[1] += w * __uint_as_float(v.x & 0xffff0000u);
      acc[2 % EPL] += w * __uint_as_float(v.y << 16);
      acc[3 % EPL] += w * __uint_as_float(v.y & 0xffff0000u);
    } else {
      const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(src + static_cast<size_t>(sl) * D));
      acc[0] += w * __uint_as_float(v << 16);
      acc[1 % EPL] += w * __uint_as_float(v & 0xffff0000u);
    }
  }
  const float inv = 1.f / wsum;
  __nv_bfloat16* dst = o + (static_cast<size_t>(t) * H + h) * D + lane * EPL;
  if (EPL == 4) {
    __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1 % EPL] * inv);
    __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 % EPL] * inv, acc[3 % EPL] * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&a);
    pk.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(dst) = pk;
  } else {
    __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1 % EPL] * inv);
    *reinterpret_cast<__nv_bfloat162*>(dst) = a;
  }
  if (lane == 0) lse[static_cast<size_t>(h) * T + t] = m + __logf(wsum);
}

cudaError_t launch_merge(const void* part_o, const float* part_lse, const int32_t* cu_dev,
                         int nseq, int T, int H, int d, int B, int topk, int T0, int ntok,
                         void* o, float* lse, cudaStream_t stream) {
  const long long warps = static_cast<long long>(ntok) * H;
  const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
  if (grid == 0) return cudaSuccess;
  const __nv_bfloat16* po = static_cast<const __nv_bfloat16*>(part_o);
  __nv_bfloat16* op = static_cast<__nv_bfloat16*>(o);
  if (d == 64)
    merge_kernel<64><<<grid, 256, 0, stream>>>(po, part_lse, cu_dev, nseq, T, H, B, topk, T0, ntok, op, lse);
  else
    merge_kernel<128><<<grid, 256, 0, stream>>>(po, part_lse, cu_dev, nseq, T, H, B, topk, T0, ntok, op, lse);
  return cudaGetLastError();
}

}  // namespace moba
