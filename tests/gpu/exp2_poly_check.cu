// Accuracy of the FMA-pipe exponential used by the attention softmax (exp2_poly, exp2_poly2 in
// csrc/sm100.cuh), measured on the GPU against 2^t computed on the host in double precision.
//
//   exp2_poly_check            prints one JSON line:
//   {"points": N, "max_rel": e, "max_rel_pair": e2, "pair_mismatch": m, "nonmonotone": n}
//
// Sweep: t = -120 + i / 8192 over [-120, 8] (every split point n + 1/2 is on the grid, as are
// the points on both sides of it). max_rel: max |exp2_poly(t) / 2^t - 1|; max_rel_pair: the same
// for exp2_poly2; pair_mismatch: points where the paired form differs from the single form in
// any bit; nonmonotone: consecutive points where the result decreases.
#include <cmath>
#include <cstdio>
#include <vector>

#include "sm100.cuh"

__global__ void sweep(float t0, float step, int n, float* single, float* pair) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i >= n) return;
  const float ta = t0 + step * static_cast<float>(2 * i);
  const float tb = t0 + step * static_cast<float>(2 * i + 1);
  single[2 * i] = moba::exp2_poly(ta);
  if (2 * i + 1 < n) single[2 * i + 1] = moba::exp2_poly(tb);
  float pa, pb;
  moba::exp2_poly2(ta, tb, pa, pb);
  pair[2 * i] = pa;
  if (2 * i + 1 < n) pair[2 * i + 1] = pb;
}

int main() {
  const float t0 = -120.f, step = 1.f / 8192.f;
  const int n = 128 * 8192 + 1;
  float *ds = nullptr, *dp = nullptr;
  if (cudaMalloc(&ds, n * sizeof(float)) != cudaSuccess) return 2;
  if (cudaMalloc(&dp, n * sizeof(float)) != cudaSuccess) return 2;
  const int threads = 256, blocks = ((n + 1) / 2 + threads - 1) / threads;
  sweep<<<blocks, threads>>>(t0, step, n, ds, dp);
  if (cudaDeviceSynchronize() != cudaSuccess) return 3;
  std::vector<float> s(n), p(n);
  cudaMemcpy(s.data(), ds, n * sizeof(float), cudaMemcpyDeviceToHost);
  cudaMemcpy(p.data(), dp, n * sizeof(float), cudaMemcpyDeviceToHost);
  cudaFree(ds);
  cudaFree(dp);
  double max_rel = 0, max_rel_pair = 0;
  long mismatch = 0, nonmono = 0;
  for (int i = 0; i < n; ++i) {
    // the same float t the kernel formed (t0 + step * i is exact in float for these values)
    const float t = t0 + step * static_cast<float>(i);
    const double exact = std::exp2(static_cast<double>(t));
    max_rel = std::fmax(max_rel, std::fabs(static_cast<double>(s[i]) / exact - 1.0));
    max_rel_pair = std::fmax(max_rel_pair, std::fabs(static_cast<double>(p[i]) / exact - 1.0));
    if (s[i] != p[i]) ++mismatch;
    if (i > 0 && s[i] < s[i - 1]) ++nonmono;
  }
  std::printf("{\"points\": %d, \"max_rel\": %.6e, \"max_rel_pair\": %.6e, \"pair_mismatch\": %ld, "
              "\"nonmonotone\": %ld}\n", n, max_rel, max_rel_pair, mismatch, nonmono);
  return 0;
}
