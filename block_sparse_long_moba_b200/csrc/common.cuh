// Shared definitions of the MoBA kernels (device side) and their host launchers.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace moba {

constexpr int kTile = 128;           // rows of one MMA half-tile, keys per key sub-tile
constexpr int kItemRows = 256;       // query rows per attention work item (two 128-row halves)
constexpr int kMaxTopk = 64;
constexpr int kMaxBlocksPerSeq = 32768;
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s per bounded device wait
// After an abort, a CTA waits for its own copies and matrix products still in flight before it
// exits. That drain has its own limit, independent of the pipeline-wait limit (which a caller
// may shorten for diagnostics), so that a short pipeline limit never cuts a drain short.
constexpr unsigned long long kDrainTimeoutNs = 2000000000ull;

// Device status word codes (written with atomicCAS(word, 0, code); first failure wins).
constexpr int kDevTimeoutAttn = 0x101;   // a pipeline wait ran out          -> MOBA_ERR_TIMEOUT
constexpr int kDevDrainTimeout = 0x102;  // an abort drain ran out            -> MOBA_ERR_TIMEOUT
constexpr int kDevBadRouting = 0x201;    // a routing row breaks its contract -> MOBA_ERR_DEVICE_CHECK
constexpr int kDevSmemAlign = 0x301;     // dynamic shared memory misaligned  -> MOBA_ERR_DEVICE_CHECK
constexpr int kDevCheckFail = 0x401;     // an index check of the MOBA_CHECKS build failed
                                         //                                   -> MOBA_ERR_DEVICE_CHECK

// MOBA_CHECKS build (compiled with -DMOBA_CHECKS=1): every index the kernels derive from data on
// the device (routing lists, work items, partial-row indices, densified rows) is checked against
// the size of the buffer it indexes before use; a failing check records kDevCheckFail and the
// access is skipped. In the normal build the checks compile to nothing.
#ifndef MOBA_CHECKS
#define MOBA_CHECKS 0
#endif
__device__ __forceinline__ bool in_range(long long x, long long n, int* status) {
#if MOBA_CHECKS
  if (x < 0 || x >= n) {
    if (status) atomicCAS(status, 0, kDevCheckFail);
    return false;
  }
#endif
  return true;
}

// Block tables built on the device from cu_seqlens (workspace resident).
struct BlockTables {
  int* blk_off;    // [nseq + 1] first global block of each sequence
  int* blk_seq;    // [NB] sequence of each global block
  int* blk_start;  // [NB] first token of each block (absolute)
  int* blk_len;    // [NB] number of keys in each block
};

// Number of key blocks of a sequence of length L.
__host__ __device__ __forceinline__ int blocks_of(int L, int B) { return (L + B - 1) / B; }

// Cooperative (whole CTA) computation of the first global block of sequence s:
// sum over s' < s of ceil(len_s' / B). Every thread of the CTA must call it.
__device__ __forceinline__ int seq_block_base(const int32_t* cu, int s, int B, int* red_smem) {
  int acc = 0;
  for (int x = threadIdx.x; x < s; x += blockDim.x) acc += blocks_of(cu[x + 1] - cu[x], B);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const int warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red_smem[warp] = acc;
  __syncthreads();
  int tot = 0;
  for (int w = 0; w < nw; ++w) tot += red_smem[w];
  __syncthreads();
  return tot;
}

}  // namespace moba
