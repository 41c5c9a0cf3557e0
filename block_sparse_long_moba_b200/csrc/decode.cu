// MoBA decode and chunked prefill against a KV cache: query rows that are the last n_s tokens of
// cached sequences [MoBA paper summary (atlas.scime.ai), "Approach" for the routing; its
// "Limitations" note that the paper's generation fell back to full attention, so this is the
// same routing applied to the newest rows of a cache].
//
// For query row r of sequence s (absolute position t, local block i = (t - cu[s]) / B):
//   D1 decode_gate_kernel   one CTA per (row, query head): scores q . c_j of the past blocks
//                           j < i from the cached centroids into shared memory (one warp per
//                           block, lanes over d), then the exact top-(k-1) by a 4-pass radix
//                           select on order-preserving 32-bit keys (ties: lower block first), and
//                           the ascending routing row {selected} + {i}, -1 padded.
//   D2 decode_attn_kernel   one CTA per (row, head, slot, 512-key chunk of the slot's block): the
//                           chunk's keys up to t, fp32 logits, chunk max, exp, sum and the
//                           unnormalised value sum -> one fp32 partial (m, l, o[d]).
//   D3 decode_merge_kernel  one warp per (row, head): LSE-weighted merge of its partials.
// Everything is HBM-bound: the selected blocks' K and V rows are read once per (row, head).
#include <algorithm>
#include <cfloat>

#include "common.cuh"
#include "launch.h"

namespace moba {

constexpr int kDecodeChunk = 512;  // keys per attention CTA
constexpr int kDecodeThreads = 256;

struct DecodeRow {
  int s, t, i, base;  // sequence, absolute position, local block, first global block
};

__device__ __forceinline__ DecodeRow decode_row(const int32_t* __restrict__ cu,
                                                const int32_t* __restrict__ cuq,
                                                const int* __restrict__ blk_off, int nseq, int r,
                                                int B) {
  int lo = 0, hi = nseq;  // sequence of row r: largest s with cuq[s] <= r
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cuq + mid) <= r) lo = mid; else hi = mid;
  }
  DecodeRow d;
  d.s = lo;
  const int c0 = __ldg(cu + lo), L = __ldg(cu + lo + 1) - c0;
  const int nq = __ldg(cuq + lo + 1) - __ldg(cuq + lo);
  const int tl = L - nq + (r - __ldg(cuq + lo));
  d.t = c0 + tl;
  d.i = tl / B;
  d.base = blk_off[lo];
  return d;
}

// order-preserving image of a float: larger score -> larger unsigned key
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one value per thread (256 threads); returns the exclusive prefix
// and writes the total to *total.
__device__ __forceinline__ int cta_exclusive_scan(int v, int* warp_tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) warp_tmp[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < kDecodeThreads / 32; ++w) {
    const int x = warp_tmp[w];
    if (w < warp) before += x;
    all += x;
  }
  *total = all;
  return before + incl - v;
}

template <int D>
__global__ void __launch_bounds__(kDecodeThreads) decode_gate_kernel(
    const __nv_bfloat16* __restrict__ q, const float* __restrict__ cents,
    const int32_t* __restrict__ cu, const int32_t* __restrict__ cuq,
    const int* __restrict__ blk_off, int nseq, int Tq, int H, int G, int B, int topk,
    int32_t* __restrict__ idx) {
  extern __shared__ float sc[];  // scores of the past blocks, then reused as keys
  __shared__ float qs[D];
  __shared__ int hist[256];
  __shared__ int warp_tmp[kDecodeThreads / 32];
  __shared__ int sel_prefix, sel_want;
  const int r = blockIdx.x, h = blockIdx.y, g = h / (H / G);
  const DecodeRow row = decode_row(cu, cuq, blk_off, nseq, r, B);
  int32_t* out = idx + (static_cast<size_t>(h) * Tq + r) * topk;
  const int i = row.i;
  if (topk - 1 >= i) {  // every block 0..i
    for (int x = threadIdx.x; x < topk; x += blockDim.x) out[x] = x <= i ? x : -1;
    return;
  }
  if (topk == 1) {  // the current block only
    if (threadIdx.x == 0) out[0] = i;
    return;
  }
  for (int x = threadIdx.x; x < D; x += blockDim.x)
    qs[x] = __bfloat162float(q[(static_cast<size_t>(r) * H + h) * D + x]);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int PER = D / 32;
  float qr[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) qr[e] = qs[lane * PER + e];
  for (int j = warp; j < i; j += kDecodeThreads / 32) {
    const float* c = cents + (static_cast<size_t>(row.base + j) * G + g) * D + lane * PER;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc = fmaf(qr[e], __ldg(c + e), acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) sc[j] = acc;
  }
  __syncthreads();
  uint32_t* key = reinterpret_cast<uint32_t*>(sc);
  for (int j = threadIdx.x; j < i; j += blockDim.x) key[j] = order_key(sc[j]);
  // radix select of the (k-1)-th largest key, 8 bits per pass from the top
  uint32_t prefix = 0, mask = 0;
  int want = topk - 1;  // rank (1 = largest) inside the keys that match prefix under mask
  for (int shift = 24; shift >= 0; shift -= 8) {
    hist[threadIdx.x] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < i; j += blockDim.x) {
      const uint32_t kj = key[j];
      if ((kj & mask) == prefix) atomicAdd(&hist[(kj >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int acc = 0, b = 255;
      for (; b > 0; --b) {
        if (acc + hist[b] >= want) break;
        acc += hist[b];
      }
      sel_prefix = static_cast<int>(b);
      sel_want = want - acc;
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel_prefix) << shift;
    mask |= 255u << shift;
    want = sel_want;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const int need_eq = want;  // keys equal to tau that are taken, lowest blocks first
  // each thread owns a contiguous range of blocks, so selection order is block order
  const int per = (i + kDecodeThreads - 1) / kDecodeThreads;
  const int j0 = min(i, static_cast<int>(threadIdx.x) * per), j1 = min(i, j0 + per);
  int n_eq = 0;
  for (int j = j0; j < j1; ++j) n_eq += key[j] == tau;
  int tot;
  int eq_before = cta_exclusive_scan(n_eq, warp_tmp, &tot);
  int n_sel = 0;
  {
    int e = eq_before;
    for (int j = j0; j < j1; ++j) {
      const uint32_t kj = key[j];
      if (kj > tau || (kj == tau && e++ < need_eq)) ++n_sel;
    }
  }
  const int pos0 = cta_exclusive_scan(n_sel, warp_tmp, &tot);
  {
    int e = eq_before, p = pos0;
    for (int j = j0; j < j1; ++j) {
      const uint32_t kj = key[j];
      if (kj > tau || (kj == tau && e++ < need_eq)) out[p++] = j;
    }
  }
  if (threadIdx.x == 0) {
    out[topk - 1] = i;  // tot == topk - 1 selected past blocks precede it
  }
}

template <int D>
__global__ void __launch_bounds__(kDecodeThreads) decode_attn_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ cu,
    const int32_t* __restrict__ cuq, const int* __restrict__ blk_off, int nseq, int Tq, int H,
    int G, int B, int topk, int cpb, float scale_log2, const int32_t* __restrict__ idx,
    float* __restrict__ part) {
  __shared__ float qs[D];
  __shared__ float red[kDecodeThreads / 32];
  __shared__ float po[kDecodeThreads / 32][D];
  const int rh = blockIdx.x;
  const int r = rh / H, h = rh % H, g = h / (H / G);
  const int slot = blockIdx.y / cpb, ch = blockIdx.y % cpb;
  float* dst = part + (static_cast<size_t>(rh) * topk * cpb + blockIdx.y) * (D + 2);
  const DecodeRow row = decode_row(cu, cuq, blk_off, nseq, r, B);
  const int j = __ldg(idx + (static_cast<size_t>(h) * Tq + r) * topk + slot);
  int u0 = 0, u1 = 0;  // absolute key range of this chunk
  if (j >= 0 && j <= row.i) {
    const int bstart = __ldg(cu + row.s) + j * B;
    const int bend = min(__ldg(cu + row.s + 1), bstart + B);
    u0 = bstart + ch * kDecodeChunk;
    u1 = min(min(bend, u0 + kDecodeChunk), row.t + 1);  // keys up to the query's position
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (u1 <= u0) {  // nothing to attend in this chunk
    if (threadIdx.x < D) dst[2 + threadIdx.x] = 0.f;
    if (threadIdx.x == 0) {
      dst[0] = -INFINITY;
      dst[1] = 0.f;
    }
    return;
  }
  for (int x = threadIdx.x; x < D; x += blockDim.x)
    qs[x] = __bfloat162float(q[(static_cast<size_t>(r) * H + h) * D + x]);
  __syncthreads();
  // logits: keys u0 + 2 tid and u0 + 2 tid + 1 (up to 512 keys), one whole key row per thread
  const size_t ld = static_cast<size_t>(G) * D;
  float z[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int u = u0 + 2 * threadIdx.x + x;
    z[x] = -INFINITY;
    if (u < u1) {
      const uint4* kr = reinterpret_cast<const uint4*>(k + static_cast<size_t>(u) * ld + g * D);
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 w = __ldg(kr + c);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc = fmaf(__uint_as_float(wv[e] << 16), qs[c * 8 + 2 * e], acc);
          acc = fmaf(__uint_as_float(wv[e] & 0xffff0000u), qs[c * 8 + 2 * e + 1], acc);
        }
      }
      z[x] = acc * scale_log2;
    }
  }
  float m = fmaxf(z[0], z[1]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < kDecodeThreads / 32; ++w) m = fmaxf(m, red[w]);
  const float p0 = exp2f(z[0] - m), p1 = exp2f(z[1] - m);  // 0 for keys past the chunk
  float l = p0 + p1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  __syncthreads();
  if (lane == 0) red[warp] = l;
  // value sum: warp w takes the keys of threads 32 w .. 32 w + 31 (64 keys), lanes over d
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  // keys of this warp that lie in the chunk; the loop is unrolled with the loads predicated on it
  // (not cut short), so several value rows are in flight at once
  const int nk = max(0, min(64, u1 - (u0 + 64 * warp)));
#pragma unroll 8
  for (int x = 0; x < 64; ++x) {
    const int src = x >> 1;
    const float p = __shfl_sync(0xffffffffu, (x & 1) ? p1 : p0, src);
    if (x >= nk) continue;  // uniform over the warp
    const int u = u0 + 64 * warp + x;  // key 2 (32 warp + src) + (x & 1) of the chunk
    const __nv_bfloat16* vr = v + static_cast<size_t>(u) * ld + g * D + lane * PER;
    if constexpr (PER == 4) {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(vr));
      acc[0] = fmaf(p, __uint_as_float(w.x << 16), acc[0]);
      acc[1] = fmaf(p, __uint_as_float(w.x & 0xffff0000u), acc[1]);
      acc[2] = fmaf(p, __uint_as_float(w.y << 16), acc[2]);
      acc[3] = fmaf(p, __uint_as_float(w.y & 0xffff0000u), acc[3]);
    } else {
      const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(vr));
      acc[0] = fmaf(p, __uint_as_float(w << 16), acc[0]);
      acc[1] = fmaf(p, __uint_as_float(w & 0xffff0000u), acc[1]);
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) po[warp][lane * PER + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeThreads / 32; ++w) o += po[w][threadIdx.x];
    dst[2 + threadIdx.x] = o;
  }
  if (threadIdx.x == 0) {
    float ls = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeThreads / 32; ++w) ls += red[w];
    dst[0] = m;   // log2-domain max of the scaled logits
    dst[1] = ls;  // sum of 2^(z - m)
  }
}

template <int D>
__global__ void __launch_bounds__(256) decode_merge_kernel(const float* __restrict__ part,
                                                           int nparts, int Tq, int H,
                                                           __nv_bfloat16* __restrict__ o,
                                                           float* __restrict__ lse) {
  const int rh = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (rh >= Tq * H) return;
  const float* p = part + static_cast<size_t>(rh) * nparts * (D + 2);
  float M = -INFINITY;
  for (int x = lane; x < nparts; x += 32) M = fmaxf(M, p[static_cast<size_t>(x) * (D + 2)]);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, s));
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float L = 0.f;
  if (M > -INFINITY) {
    for (int x = 0; x < nparts; ++x) {
      const float* px = p + static_cast<size_t>(x) * (D + 2);
      const float mx = px[0];
      if (mx == -INFINITY) continue;
      const float w = exp2f(mx - M);
      L = fmaf(w, px[1], L);
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, px[2 + lane * PER + e], acc[e]);
    }
  }
  const int r = rh / H, h = rh % H;
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e)
    o[static_cast<size_t>(rh) * D + lane * PER + e] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0)
    lse[static_cast<size_t>(h) * Tq + r] =
        L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

int decode_parts(int B, int topk) { return topk * ((B + kDecodeChunk - 1) / kDecodeChunk); }

cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t stream) {
  if (L.Tq == 0) return cudaSuccess;
  const int cpb = (L.B + kDecodeChunk - 1) / kDecodeChunk;
  const size_t gate_smem = static_cast<size_t>(std::max(L.max_nb, 1)) * 4;
  const auto* qp = static_cast<const __nv_bfloat16*>(L.q);
  const auto* kp = static_cast<const __nv_bfloat16*>(L.k);
  const auto* vp = static_cast<const __nv_bfloat16*>(L.v);
  auto* op = static_cast<__nv_bfloat16*>(L.o);
  cudaError_t e;
  if (!L.idx_given) {
    if (L.d == 64) {
      e = cudaFuncSetAttribute(decode_gate_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(gate_smem));
      if (e != cudaSuccess) return e;
      decode_gate_kernel<64><<<dim3(L.Tq, L.H), kDecodeThreads, gate_smem, stream>>>(
          qp, L.cents, L.cu, L.cuq, L.blk_off, L.nseq, L.Tq, L.H, L.G, L.B, L.topk, L.idx);
    } else {
      e = cudaFuncSetAttribute(decode_gate_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(gate_smem));
      if (e != cudaSuccess) return e;
      decode_gate_kernel<128><<<dim3(L.Tq, L.H), kDecodeThreads, gate_smem, stream>>>(
          qp, L.cents, L.cu, L.cuq, L.blk_off, L.nseq, L.Tq, L.H, L.G, L.B, L.topk, L.idx);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const dim3 grid(static_cast<unsigned>(L.Tq * L.H), static_cast<unsigned>(L.topk * cpb));
  const float sl2 = L.scale * 1.4426950408889634f;
  if (L.d == 64)
    decode_attn_kernel<64><<<grid, kDecodeThreads, 0, stream>>>(
        qp, kp, vp, L.cu, L.cuq, L.blk_off, L.nseq, L.Tq, L.H, L.G, L.B, L.topk, cpb, sl2, L.idx,
        L.part);
  else
    decode_attn_kernel<128><<<grid, kDecodeThreads, 0, stream>>>(
        qp, kp, vp, L.cu, L.cuq, L.blk_off, L.nseq, L.Tq, L.H, L.G, L.B, L.topk, cpb, sl2, L.idx,
        L.part);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const unsigned mgrid = static_cast<unsigned>((static_cast<long long>(L.Tq) * L.H + 7) / 8);
  if (L.d == 64)
    decode_merge_kernel<64><<<mgrid, 256, 0, stream>>>(L.part, L.topk * cpb, L.Tq, L.H, op, L.lse);
  else
    decode_merge_kernel<128><<<mgrid, 256, 0, stream>>>(L.part, L.topk * cpb, L.Tq, L.H, op, L.lse);
  return cudaGetLastError();
}

}  // namespace moba
