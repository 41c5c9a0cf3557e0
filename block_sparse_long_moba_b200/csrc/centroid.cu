// K1 — block centroids: c[b, g, :] = mean of the keys of global block b, kv head g, in fp32
// [MoBA paper summary (atlas.scime.ai), "Approach": blocks are represented by mean-pooled keys].
//
// HBM-bound: K is read exactly once with 16-byte loads. One thread-block cluster of CL CTAs
// reduces one (block, kv head); each CTA sums a contiguous slice of the block's keys and the
// cluster's rank-0 CTA adds the slices in rank order through distributed shared memory, so the
// result is deterministic and no workspace is needed.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace moba {

template <int D>
__global__ void __launch_bounds__(256) centroid_kernel(const __nv_bfloat16* __restrict__ k,
                                                       const int32_t* __restrict__ cu, int G,
                                                       int B, int CL, float* __restrict__ out) {
  constexpr int CPR = D / 8;     // 16-byte chunks per key row
  constexpr int RP = 256 / CPR;  // key rows covered by one pass of the CTA
  __shared__ float part[RP][D];
  __shared__ float red[D];
  __shared__ int red_smem[32];

  const int g = blockIdx.x / CL, rank = blockIdx.x % CL;
  const int j = blockIdx.y, s = blockIdx.z;
  const int seq0 = cu[s];
  const int L = cu[s + 1] - seq0;
  if (j >= blocks_of(L, B)) return;  // uniform over the cluster (same j, s)
  const int base = seq_block_base(cu, s, B, red_smem);
  const int t0 = seq0 + j * B;
  const int n = min(B, L - j * B);
  const int lo = static_cast<int>(static_cast<long long>(n) * rank / CL);
  const int hi = static_cast<int>(static_cast<long long>(n) * (rank + 1) / CL);

  const int c = threadIdx.x % CPR, rr = threadIdx.x / CPR;
  const size_t row_stride = static_cast<size_t>(G) * D;
  const __nv_bfloat16* src = k + (static_cast<size_t>(t0) * G + g) * D + c * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  auto add = [&](const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(w[e] << 16);
      acc[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
    }
  };
  int t = lo + rr;
  for (; t + 3 * RP < hi; t += 4 * RP) {
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * row_stride));
    const uint4 v1 =
        __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t + RP) * row_stride));
    const uint4 v2 =
        __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t + 2 * RP) * row_stride));
    const uint4 v3 =
        __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t + 3 * RP) * row_stride));
    add(v0);
    add(v1);
    add(v2);
    add(v3);
  }
  for (; t < hi; t += RP)
    add(__ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * row_stride)));
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rr][c * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
    for (int x = 0; x < RP; ++x) sum += part[x][threadIdx.x];
    red[threadIdx.x] = sum;
  }
  float* dst = out + (static_cast<size_t>(base + j) * G + g) * D;
  if (CL > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && threadIdx.x < D) {
      float sum = red[threadIdx.x];
      for (int q = 1; q < CL; ++q) sum += cluster.map_shared_rank(red, q)[threadIdx.x];
      dst[threadIdx.x] = sum / static_cast<float>(n);
    }
    cluster.sync();  // peers keep their shared memory alive until rank 0 has read it
  } else {
    __syncthreads();
    if (threadIdx.x < D) dst[threadIdx.x] = red[threadIdx.x] / static_cast<float>(n);
  }
}

cudaError_t launch_centroids(const void* k, const int32_t* cu_dev, int nseq, int max_nb, int G,
                             int d, int B, int total_nb, int num_sms, float* out,
                             cudaStream_t stream) {
  int CL = 1;
  while (CL < 8 && static_cast<long long>(total_nb) * G * CL < 8LL * num_sms) CL *= 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G * CL), static_cast<unsigned>(max_nb),
                     static_cast<unsigned>(nseq));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(k);
  if (d == 64) return cudaLaunchKernelEx(&cfg, centroid_kernel<64>, kp, cu_dev, G, B, CL, out);
  return cudaLaunchKernelEx(&cfg, centroid_kernel<128>, kp, cu_dev, G, B, CL, out);
}

}  // namespace moba
