// K1 — block centroids: c[b, g, :] = mean of the keys of global block b, kv head g, in fp32
// [MoBA paper summary (atlas.scime.ai), "Approach": blocks are represented by mean-pooled keys].
//
// HBM-bound: K is read exactly once with 16-byte loads. One thread-block cluster of CL CTAs
// reduces one key block for every kv head at once: a token's keys of all heads are one contiguous
// row of G * d bf16, so each CTA streams a contiguous slice of the block's rows (a warp reads 512
// contiguous bytes per instruction, eight rows in flight per thread), and every thread keeps the
// running sums of fixed 8-column pieces of the row. The cluster's rank-0 CTA adds the slices in
// rank order through distributed shared memory, so the result is deterministic and no workspace
// is needed. Rows wider than 1024 pieces (G * d > 8192), and problems with too few blocks to fill
// the GPU in whole rows, take the per-head form below (one cluster per block and kv head).
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace moba {

// Short key convolution before pooling [FlashMoBA story: short convolutions within blocks].
// With kconv[t] = sum_{m<W} w[m] k[t-m] inside the block (terms before the block's first key left
// out), the block sum of the convolved keys follows from the plain block sum S and the block's
// last W-1 keys, since key u contributes w[m] for every m with u + m still inside the block:
//   sum_t kconv[t] = (sum_m w[m]) S - sum_{m=1}^{W-1} w[m] (k[e-1] + ... + k[e-m]),  e = block end
// (the tail sum stops growing once it holds the whole block). `x` is the column in a token's row
// of G * d keys, `last` points at column x of the block's last key, `ld` is the row stride.
__device__ __forceinline__ float kconv_block_sum(float S, const float* __restrict__ cw, int W,
                                                 int GD, int x, const __nv_bfloat16* last,
                                                 size_t ld, int n) {
  float wsum = 0.f;
  for (int m = 0; m < W; ++m) wsum += __ldg(cw + static_cast<size_t>(m) * GD + x);
  float res = wsum * S, tail = 0.f;
  for (int m = 1; m < W; ++m) {
    if (m <= n) tail += __bfloat162float(last[-static_cast<ptrdiff_t>((m - 1) * ld)]);
    res = fmaf(-__ldg(cw + static_cast<size_t>(m) * GD + x), tail, res);
  }
  return res;
}

template <int D>
__global__ void __launch_bounds__(256) centroid_kernel(const __nv_bfloat16* __restrict__ k,
                                                       const int32_t* __restrict__ cu, int G,
                                                       int B, int CL, float* __restrict__ out,
                                                       const float* __restrict__ cw, int W) {
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
  for (; t + 7 * RP < hi; t += 8 * RP) {  // eight rows in flight per thread
    uint4 v[8];
#pragma unroll
    for (int x = 0; x < 8; ++x)
      v[x] = __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t + x * RP) * row_stride));
#pragma unroll
    for (int x = 0; x < 8; ++x) add(v[x]);
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
  auto finish = [&](float sum) -> float {
    if (W > 0) {
      const int x = g * D + threadIdx.x;
      sum = kconv_block_sum(sum, cw, W, G * D, x,
                            k + static_cast<size_t>(t0 + n - 1) * row_stride + x, row_stride, n);
    }
    return sum / static_cast<float>(n);
  };
  if (CL > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && threadIdx.x < D) {
      float sum = red[threadIdx.x];
      for (int q = 1; q < CL; ++q) sum += cluster.map_shared_rank(red, q)[threadIdx.x];
      dst[threadIdx.x] = finish(sum);
    }
    cluster.sync();  // peers keep their shared memory alive until rank 0 has read it
  } else {
    __syncthreads();
    if (threadIdx.x < D) dst[threadIdx.x] = finish(red[threadIdx.x]);
  }
}

// Whole-row form: NS 8-column pieces per thread (NS = 1 when a row has at most 256 pieces, and
// then 256 / pieces rows are read side by side).
template <int NS>
__global__ void __launch_bounds__(256) centroid_rows_kernel(const __nv_bfloat16* __restrict__ k,
                                                            const int32_t* __restrict__ cu,
                                                            int GD, int B, int CL,
                                                            float* __restrict__ out,
                                                            const float* __restrict__ cw, int W) {
  extern __shared__ float sm_c[];  // NS == 1: [RPP][CPR][8] partial sums; then [CPR * 8] totals
  __shared__ int red_smem[32];
  const int rank = blockIdx.x % CL;
  const int j = blockIdx.y, s = blockIdx.z;
  const int seq0 = cu[s];
  const int L = cu[s + 1] - seq0;
  if (j >= blocks_of(L, B)) return;  // uniform over the cluster (same j, s)
  const int base = seq_block_base(cu, s, B, red_smem);
  const int t0 = seq0 + j * B;
  const int n = min(B, L - j * B);
  const int lo = static_cast<int>(static_cast<long long>(n) * rank / CL);
  const int hi = static_cast<int>(static_cast<long long>(n) * (rank + 1) / CL);
  const int CPR = GD / 8;  // 16-byte pieces per row
  const int RPP = (NS == 1) ? 256 / CPR : 1;
  const int tid = threadIdx.x;
  const int ro = (NS == 1) ? tid / CPR : 0;
  const int p0 = (NS == 1) ? tid % CPR : tid;
  float acc[NS][8];
#pragma unroll
  for (int u = 0; u < NS; ++u)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
  auto add = [&](int u, const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[u][2 * e] += __uint_as_float(w[e] << 16);
      acc[u][2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
    }
  };
  const __nv_bfloat16* rowp = k + static_cast<size_t>(t0) * GD;
  if (NS == 1) {
    if (ro < RPP) {
      const uint4* src = reinterpret_cast<const uint4*>(rowp) + p0;
      const size_t rs = static_cast<size_t>(CPR);  // row stride in pieces
      int t = lo + ro;
      for (; t + 7 * RPP < hi; t += 8 * RPP) {
        uint4 v[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) v[x] = __ldg(src + static_cast<size_t>(t + x * RPP) * rs);
#pragma unroll
        for (int x = 0; x < 8; ++x) add(0, v[x]);
      }
      for (; t < hi; t += RPP) add(0, __ldg(src + static_cast<size_t>(t) * rs));
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_c[(ro * CPR + p0) * 8 + e] = acc[0][e];
    }
    __syncthreads();
    // totals of this CTA's slice, one 8-column piece per thread (CPR <= 256)
    float tot[8];
    if (tid < CPR) {
#pragma unroll
      for (int e = 0; e < 8; ++e) tot[e] = 0.f;
      for (int x = 0; x < RPP; ++x)
#pragma unroll
        for (int e = 0; e < 8; ++e) tot[e] += sm_c[(x * CPR + tid) * 8 + e];
    }
    __syncthreads();
    if (tid < CPR)
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_c[tid * 8 + e] = tot[e];
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(rowp);
    const size_t rs = static_cast<size_t>(CPR);
    int t = lo;
    for (; t + 1 < hi; t += 2) {
      uint4 v[2][NS];
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int u = 0; u < NS; ++u)
          v[x][u] = (p0 + 256 * u < CPR) ? __ldg(src + static_cast<size_t>(t + x) * rs + p0 + 256 * u)
                                         : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int u = 0; u < NS; ++u) add(u, v[x][u]);
    }
    for (; t < hi; ++t)
#pragma unroll
      for (int u = 0; u < NS; ++u)
        if (p0 + 256 * u < CPR) add(u, __ldg(src + static_cast<size_t>(t) * rs + p0 + 256 * u));
#pragma unroll
    for (int u = 0; u < NS; ++u)
      if (p0 + 256 * u < CPR)
#pragma unroll
        for (int e = 0; e < 8; ++e) sm_c[(p0 + 256 * u) * 8 + e] = acc[u][e];
  }
  float* dst = out + static_cast<size_t>(base + j) * GD;
  const float inv_n = 1.f / static_cast<float>(n);
  auto finish = [&](float sum, int x) -> float {
    if (W > 0)
      sum = kconv_block_sum(sum, cw, W, GD, x, rowp + static_cast<size_t>(n - 1) * GD + x,
                            static_cast<size_t>(GD), n);
    return sum * inv_n;
  };
  if (CL > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0) {
      for (int x = tid; x < GD; x += 256) {
        float sum = sm_c[x];
        for (int q = 1; q < CL; ++q) sum += cluster.map_shared_rank(sm_c, q)[x];
        dst[x] = finish(sum, x);
      }
    }
    cluster.sync();  // peers keep their shared memory alive until rank 0 has read it
  } else {
    __syncthreads();
    for (int x = tid; x < GD; x += 256) dst[x] = finish(sm_c[x], x);
  }
}

cudaError_t launch_centroids(const void* k, const int32_t* cu_dev, int nseq, int max_nb, int G,
                             int d, int B, int total_nb, int num_sms, float* out,
                             cudaStream_t stream, const float* conv_w, int conv_width) {
  const int W = conv_w ? conv_width : 0;
  const int GD = G * d;
  // whole rows need enough blocks to spread over the SMs (measured: 256 blocks of 4096 keys at
  // 91% of HBM, while 32 such blocks reached only a quarter of it in whole rows but half of it per
  // kv head)
  if (GD <= 8192 && static_cast<long long>(total_nb) * 8 >= 4LL * num_sms) {
    // whole rows: CL CTAs per block, enough CTAs for a few per SM
    int CL = 1;
    while (CL < 8 && static_cast<long long>(total_nb) * CL < 4LL * num_sms) CL *= 2;
    const int CPR = GD / 8;
    const int NS = CPR <= 256 ? 1 : (CPR <= 512 ? 2 : 4);
    const size_t smem = (NS == 1) ? static_cast<size_t>(256 / CPR) * CPR * 8 * 4
                                  : static_cast<size_t>(CPR) * 8 * 4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(CL), static_cast<unsigned>(max_nb),
                       static_cast<unsigned>(nseq));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(k);
    if (NS == 1)
      return cudaLaunchKernelEx(&cfg, centroid_rows_kernel<1>, kp, cu_dev, GD, B, CL, out, conv_w, W);
    if (NS == 2)
      return cudaLaunchKernelEx(&cfg, centroid_rows_kernel<2>, kp, cu_dev, GD, B, CL, out, conv_w, W);
    return cudaLaunchKernelEx(&cfg, centroid_rows_kernel<4>, kp, cu_dev, GD, B, CL, out, conv_w, W);
  }
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
  if (d == 64)
    return cudaLaunchKernelEx(&cfg, centroid_kernel<64>, kp, cu_dev, G, B, CL, out, conv_w, W);
  return cudaLaunchKernelEx(&cfg, centroid_kernel<128>, kp, cu_dev, G, B, CL, out, conv_w, W);
}

}  // namespace moba
