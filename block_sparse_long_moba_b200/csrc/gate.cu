// K2 — parameter-less causal top-k gate [MoBA paper summary (atlas.scime.ai), "Approach";
// MoBA README, "Parameter-less Gating Mechanism"].
//
// For query t in local block i of its sequence and query head h (kv head g = h / r):
//   s_j = q[t,h] . c[base + j, g] for the past blocks j < i; the routing is {i} plus the top-(k-1)
//   past blocks by s_j (equal scores keep the lower j), or every block 0..i when k-1 >= i.
// One thread owns one (t, h) row: its query row sits in registers as fp32, the centroids of the
// past blocks stream through shared memory in chunks shared by the CTA's r*TPC rows (all rows of
// a CTA belong to the same query block and kv head, so they score the same candidates), and the
// running top list lives in registers. The T x NB score matrix is never materialised
// [FlashMoBA story, FlashTopK: no materialised score matrix].
#include "common.cuh"
#include "launch.h"

namespace moba {

constexpr int kGateChunk = 64;  // centroid rows staged in shared memory at a time

template <int KCAP>
__device__ __forceinline__ void topk_insert(float (&vals)[KCAP], int (&ids)[KCAP], float s,
                                            int j) {
  if (s > vals[KCAP - 1]) {  // strict: an equal later block never displaces an earlier one
    vals[KCAP - 1] = s;
    ids[KCAP - 1] = j;
#pragma unroll
    for (int x = KCAP - 1; x > 0; --x) {
      if (vals[x] > vals[x - 1]) {
        const float tv = vals[x];
        vals[x] = vals[x - 1];
        vals[x - 1] = tv;
        const int ti = ids[x];
        ids[x] = ids[x - 1];
        ids[x - 1] = ti;
      }
    }
  }
}

template <int D, int KCAP>
__global__ void __launch_bounds__(256, 1)
    gate_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ cents,
                const int32_t* __restrict__ cu, int T, int H, int G, int B, int topk, int TPC,
                int32_t* __restrict__ idx) {
  extern __shared__ float4 csm4[];  // [kGateChunk][D/4]
  __shared__ int red_smem[32];
  const int g = blockIdx.x % G, chunk = blockIdx.x / G;
  const int i = blockIdx.y, s = blockIdx.z;
  const int r = H / G;
  const int seq0 = cu[s];
  const int L = cu[s + 1] - seq0;
  if (i >= blocks_of(L, B)) return;
  const int blen = min(B, L - i * B);
  const int tl0 = chunk * TPC;
  if (tl0 >= blen) return;
  const int ntok = min(TPC, blen - tl0);
  const int hh = threadIdx.x / TPC, tl = threadIdx.x % TPC;
  const bool valid = (hh < r) && (tl < ntok);
  const int h = g * r + hh;
  const int t = seq0 + i * B + tl0 + tl;
  const int ksel = topk - 1;
  int32_t* out = idx + (static_cast<size_t>(h) * T + t) * topk;

  if (ksel >= i) {  // few causal blocks: every block 0..i, then -1 padding
    if (valid)
      for (int x = 0; x < topk; ++x) out[x] = (x <= i) ? x : -1;
    return;
  }
  if (ksel == 0) {  // topk == 1: only the current block
    if (valid) out[0] = i;
    return;
  }
  const int base = seq_block_base(cu, s, B, red_smem);

  float qf[D];
  if (valid) {
    const uint4* qp = reinterpret_cast<const uint4*>(q + (static_cast<size_t>(t) * H + h) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 v = __ldg(qp + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qf[c * 8 + 2 * e] = __uint_as_float(w[e] << 16);
        qf[c * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int x = 0; x < D; ++x) qf[x] = 0.f;
  }

  float vals[KCAP];
  int ids[KCAP];
#pragma unroll
  for (int x = 0; x < KCAP; ++x) {
    vals[x] = -INFINITY;
    ids[x] = 0x7fffffff;
  }

  for (int j0 = 0; j0 < i; j0 += kGateChunk) {
    const int nj = min(kGateChunk, i - j0);
    __syncthreads();
    for (int e = threadIdx.x; e < nj * (D / 4); e += blockDim.x) {
      const int jj = e / (D / 4), c4 = e % (D / 4);
      csm4[e] = __ldg(reinterpret_cast<const float4*>(
                          cents + (static_cast<size_t>(base + j0 + jj) * G + g) * D) +
                      c4);
    }
    __syncthreads();
    int jj = 0;
    for (; jj + 1 < nj; jj += 2) {
      const float4* c0 = csm4 + jj * (D / 4);
      const float4* c1 = c0 + D / 4;
      float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
      for (int x = 0; x < D / 4; x += 2) {
        const float4 u0 = c0[x], u1 = c0[x + 1], w0 = c1[x], w1 = c1[x + 1];
        a0 = fmaf(qf[4 * x + 0], u0.x, a0);
        a0 = fmaf(qf[4 * x + 1], u0.y, a0);
        a0 = fmaf(qf[4 * x + 2], u0.z, a0);
        a0 = fmaf(qf[4 * x + 3], u0.w, a0);
        a1 = fmaf(qf[4 * x + 4], u1.x, a1);
        a1 = fmaf(qf[4 * x + 5], u1.y, a1);
        a1 = fmaf(qf[4 * x + 6], u1.z, a1);
        a1 = fmaf(qf[4 * x + 7], u1.w, a1);
        b0 = fmaf(qf[4 * x + 0], w0.x, b0);
        b0 = fmaf(qf[4 * x + 1], w0.y, b0);
        b0 = fmaf(qf[4 * x + 2], w0.z, b0);
        b0 = fmaf(qf[4 * x + 3], w0.w, b0);
        b1 = fmaf(qf[4 * x + 4], w1.x, b1);
        b1 = fmaf(qf[4 * x + 5], w1.y, b1);
        b1 = fmaf(qf[4 * x + 6], w1.z, b1);
        b1 = fmaf(qf[4 * x + 7], w1.w, b1);
      }
      topk_insert<KCAP>(vals, ids, a0 + a1, j0 + jj);
      topk_insert<KCAP>(vals, ids, b0 + b1, j0 + jj + 1);
    }
    if (jj < nj) {
      const float4* c0 = csm4 + jj * (D / 4);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int x = 0; x < D / 4; x += 2) {
        const float4 u0 = c0[x], u1 = c0[x + 1];
        a0 = fmaf(qf[4 * x + 0], u0.x, a0);
        a0 = fmaf(qf[4 * x + 1], u0.y, a0);
        a0 = fmaf(qf[4 * x + 2], u0.z, a0);
        a0 = fmaf(qf[4 * x + 3], u0.w, a0);
        a1 = fmaf(qf[4 * x + 4], u1.x, a1);
        a1 = fmaf(qf[4 * x + 5], u1.y, a1);
        a1 = fmaf(qf[4 * x + 6], u1.z, a1);
        a1 = fmaf(qf[4 * x + 7], u1.w, a1);
      }
      topk_insert<KCAP>(vals, ids, a0 + a1, j0 + jj);
    }
  }
  if (!valid) return;
  // the first ksel entries are the routed past blocks; emit them ascending, then the current one
  int sel[KCAP];
#pragma unroll
  for (int x = 0; x < KCAP; ++x) sel[x] = (x < ksel) ? ids[x] : 0x7fffffff;
#pragma unroll
  for (int a = 0; a < KCAP - 1; ++a) {
#pragma unroll
    for (int b = 0; b < KCAP - 1 - a; ++b) {
      if (sel[b] > sel[b + 1]) {
        const int tmp = sel[b];
        sel[b] = sel[b + 1];
        sel[b + 1] = tmp;
      }
    }
  }
#pragma unroll
  for (int x = 0; x < KCAP; ++x)
    if (x < ksel) out[x] = sel[x];
  out[ksel] = i;
}

template <int D, int KCAP>
static cudaError_t launch_gate_t(dim3 grid, int threads, cudaStream_t stream,
                                 const __nv_bfloat16* q, const float* cents, const int32_t* cu,
                                 int T, int H, int G, int B, int topk, int TPC, int32_t* idx) {
  const int smem = kGateChunk * D * 4;
  cudaError_t e = cudaFuncSetAttribute(gate_kernel<D, KCAP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gate_kernel<D, KCAP><<<grid, threads, smem, stream>>>(q, cents, cu, T, H, G, B, topk, TPC, idx);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_gate_d(dim3 grid, int threads, cudaStream_t stream,
                                 const __nv_bfloat16* q, const float* cents, const int32_t* cu,
                                 int T, int H, int G, int B, int topk, int TPC, int32_t* idx) {
  const int ksel = topk - 1;
  if (ksel <= 2)
    return launch_gate_t<D, 2>(grid, threads, stream, q, cents, cu, T, H, G, B, topk, TPC, idx);
  if (ksel <= 4)
    return launch_gate_t<D, 4>(grid, threads, stream, q, cents, cu, T, H, G, B, topk, TPC, idx);
  if (ksel <= 8)
    return launch_gate_t<D, 8>(grid, threads, stream, q, cents, cu, T, H, G, B, topk, TPC, idx);
  if (ksel <= 16)
    return launch_gate_t<D, 16>(grid, threads, stream, q, cents, cu, T, H, G, B, topk, TPC, idx);
  if (ksel <= 32)
    return launch_gate_t<D, 32>(grid, threads, stream, q, cents, cu, T, H, G, B, topk, TPC, idx);
  return launch_gate_t<D, 64>(grid, threads, stream, q, cents, cu, T, H, G, B, topk, TPC, idx);
}

cudaError_t launch_gate(const void* q, const float* cents, const int32_t* cu_dev, int nseq,
                        int max_nb, int T, int H, int G, int d, int B, int topk, int32_t* idx,
                        cudaStream_t stream) {
  const int r = H / G;
  int TPC = 256 / r;          // tokens per CTA: r * TPC <= 256 rows, one per thread
  if (TPC > B) TPC = B;
  if (TPC < 1) TPC = 1;
  int threads = ((r * TPC + 31) / 32) * 32;
  const int nchunk = (B + TPC - 1) / TPC;
  dim3 grid(static_cast<unsigned>(nchunk * G), static_cast<unsigned>(max_nb),
            static_cast<unsigned>(nseq));
  const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(q);
  if (d == 64) return launch_gate_d<64>(grid, threads, stream, qp, cents, cu_dev, T, H, G, B, topk, TPC, idx);
  return launch_gate_d<128>(grid, threads, stream, qp, cents, cu_dev, T, H, G, B, topk, TPC, idx);
}

}  // namespace moba
