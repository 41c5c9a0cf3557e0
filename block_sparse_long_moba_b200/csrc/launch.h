// Host-side launchers of the MoBA kernels (internal to libmoba.so).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace moba {

cudaError_t launch_plan(const int32_t* cu_dev, int nseq, int B, int NB, const BlockTables& tb,
                        int* counts, int ncounts, int* status, cudaStream_t stream);

// conv_w (nullable): weights [conv_width, G, d] fp32 of the short key convolution applied
// inside each block before pooling.
constexpr int kMaxKconvWidth = 16;
cudaError_t launch_centroids(const void* k, const int32_t* cu_dev, int nseq, int max_nb, int G,
                             int d, int B, int total_nb, int num_sms, float* out,
                             cudaStream_t stream, const float* conv_w = nullptr,
                             int conv_width = 0);

cudaError_t launch_gate(const void* q, const float* cents, const int32_t* cu_dev, int nseq,
                        int max_nb, int T, int H, int G, int d, int B, int topk, int32_t* idx,
                        cudaStream_t stream);

// Per-CTA starts of the streaming gate's tile ranges (host-computed, passed by value).
constexpr int kGateMaxCtas = 160;
struct GateSched {
  int n_cta;
  int seg[kGateMaxCtas];    // s * Hkv + g of the first tile
  int blk[kGateMaxCtas];    // its local block i
  int pos[kGateMaxCtas];    // its index inside the block: head-in-group * tiles(i) + piece
  int base[kGateMaxCtas];   // first global block of its sequence
  int count[kGateMaxCtas];  // tiles of the range
};

// Streaming tensor-core gate for sequences of at most 257 blocks and topk <= 33.
bool gate_stream_supported(int max_nb, int topk);
int gate_stream_schedule(const int32_t* cu_host, int nseq, int H, int G, int d, int B, int topk,
                         int num_ctas, GateSched* S);
cudaError_t launch_gate_stream(const void* q, const float* cents, const int32_t* cu_dev,
                               const int32_t* cu_host, int nseq, int max_nb, int T, int H, int G,
                               int d, int B, int topk, int32_t* idx, int* status, int num_sms,
                               cudaStream_t stream);

// Tensor-core gate (scores on tcgen05, top-k in registers). `status` may be null. With `split`
// (gate_split_bytes(NB, G, d) bytes) and the block tables, the centroids are split into hi / lo
// bf16 once into that buffer and the kernel copies chunks of it; otherwise it converts them itself.
cudaError_t launch_gate_tc(const void* q, const float* cents, const int32_t* cu_dev, int nseq,
                           int max_nb, int T, int H, int G, int d, int B, int topk, int32_t* idx,
                           int* status, int num_sms, cudaStream_t stream,
                           const BlockTables* tb = nullptr, int NB = 0, void* split = nullptr);
size_t gate_split_bytes(int NB, int G, int d);

// Counts the routed entries per (kv head, block) and checks every routing row of the chunk
// against its contract (kDevBadRouting in *status on the first bad row).
cudaError_t launch_route_count(const int32_t* idx, const BlockTables& tb, int T, int H, int G,
                               int topk, int NB, int b0, int nblk, int T0, int max_nb,
                               int* counts, int* status, cudaStream_t stream);

cudaError_t launch_route_scan(int* counts, int nbk, int* cursor, int4* tiles, int* n_tiles,
                              long long tiles_cap, int* status, cudaStream_t stream);

cudaError_t launch_route_scatter(const int32_t* idx, const BlockTables& tb, int T, int H, int G,
                                 int topk, int NB, int b0, int nblk, int T0, int max_nb,
                                 int* cursor, int* entries, long long ent_cap, int* status,
                                 cudaStream_t stream);

// d = 64: copies the query row of every routed entry of the chunk into qdense (row = entry).
cudaError_t launch_densify(const int* entries, const int* n_entries, const void* q, int H,
                           int topk, int T0, long long max_entries, void* qdense, int num_sms,
                           long long q_rows, int* status, cudaStream_t stream);

struct AttnLaunch {
  const void* q;
  const void* k;
  const void* v;
  const int4* tiles;
  const int* n_routed;
  const int* entries;
  const void* qdense;      // d = 64: routed query rows, one per entry (nullptr otherwise)
  long long qdense_rows;   // rows of qdense (= capacity of the entries list)
  long long rows_cap;      // partial-output rows
  BlockTables tb;
  void* part_o;
  float* part_lse;
  int* status;
  int T, H, G, d, B, topk, NB;
  int b0, nblk, T0;
  float scale;
  int grid;
  unsigned long long wait_ns = 0;  // pipeline-wait limit; 0 = kWaitTimeoutNs
  int diag_stall = 0;              // diagnostics: make the MMA issuer's first wait run out
};

cudaError_t launch_attention(const AttnLaunch& L, cudaStream_t stream);

// TMA tensor maps (csrc/attn.cu): the driver's cuTensorMapEncodeTiled, a [T, G, D] bf16 key or
// value tensor as a 3-D map (D, G, T) with a (64, 1, 128) box and the 128-byte swizzle, and
// [rows, D] bf16 rows as a 2-D map with a one-row box (for tile::gather4), 128-byte swizzle.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_fn();
bool make_kv_map(CUtensorMap* map, const void* base, int T, int G, int D);
bool make_q_rows_map(CUtensorMap* map, const void* base, long long rows, int D);

cudaError_t launch_merge(const void* part_o, const float* part_lse, const int32_t* cu_dev,
                         int nseq, int T, int H, int d, int B, int topk, int T0, int ntok,
                         void* o, float* lse, cudaStream_t stream);

// Decode / chunked prefill against a KV cache (csrc/decode.cu).
struct DecodeLaunch {
  const void* q;       // [Tq, H, d] bf16: the query rows (the last n_s tokens of each sequence)
  const void* k;       // [T, G, d] bf16 cache
  const void* v;
  const float* cents;  // [NB, G, d] centroids of the cache's blocks
  const int32_t* cu;   // [nseq + 1] cache lengths (device)
  const int32_t* cuq;  // [nseq + 1] query rows per sequence (device)
  const int* blk_off;  // [nseq + 1] first global block of each sequence (device)
  int32_t* idx;        // [H, Tq, topk] routing (written by the gate unless idx_given)
  bool idx_given;
  float* part;         // [Tq, H, decode_parts] x (d + 2) fp32 partials
  void* o;             // [Tq, H, d] bf16
  float* lse;          // [H, Tq]
  int nseq, Tq, H, G, d, B, topk, max_nb;
  float scale;
};
int decode_parts(int B, int topk);
cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t stream);

// Backward pass of the routed attention (csrc/attn_bwd.cu), one query chunk at a time.
struct BwdLaunch {
  const void *q, *k, *v, *o, *dout;  // bf16 [T, H or G, d]
  const float* lse;                  // [H, T]
  const int* entries;                // chunk's routed entries grouped by (g, b)
  const int* bucket_end;             // [G * NB] end of every list after the scatter
  const int4* tiles;                 // routed 256-row items
  const int* n_routed;               // [0] routed items, [1] routed entries of the chunk
  BlockTables tb;
  float* dsum;                       // [T * H] scratch: D = dO . O
  float* dq_acc;                     // [T * H, d] fp32 accumulators
  float* dk_acc;                     // [T * G, d]
  float* dv_acc;
  void* qd;                          // [dense_rows, d] densified query rows of the chunk
  void* dd;                          // [dense_rows, d] densified dO rows
  float* col_lse;                    // [dense_rows] log2-domain LSE, D, position per dense row
  float* col_d;
  int* col_t;
  long long dense_rows;              // capacity of the dense arrays (max entries of a chunk)
  void *dq, *dk, *dv;                // bf16 outputs
  int* status;
  int T, H, G, d, B, topk, NB, num_sms;
  int T0, b0, nblk;                  // the chunk
  float scale;
  unsigned long long wait_ns = 0;
};
// Once: D = dO . O and the zeroed accumulators. Per chunk: densify the routed rows, the
// key-stationary dK / dV kernel, the query-stationary dQ kernel. Once: bf16 outputs.
cudaError_t launch_bwd_pre(const BwdLaunch& L, cudaStream_t stream);
cudaError_t launch_bwd_densify(const BwdLaunch& L, cudaStream_t stream);
cudaError_t launch_bwd_dkdv(const BwdLaunch& L, cudaStream_t stream);
cudaError_t launch_bwd_dq(const BwdLaunch& L, cudaStream_t stream);
cudaError_t launch_bwd_finish(const BwdLaunch& L, cudaStream_t stream);

// Whole forward pass on a caller-provided workspace (the body of moba_attn_fwd); the partial
// outputs of one query chunk are kept under `partial_budget` bytes.
int attn_fwd_impl(const void* q, const void* k, const void* v, const int32_t* cu_dev,
                  const int32_t* cu_host, int nseq, int Hq, int Hkv, int d, int block_size,
                  int topk, float scale, const int32_t* block_idx_in, int32_t* block_idx_out,
                  void* o, float* lse, void* workspace, size_t workspace_bytes, void* stream,
                  size_t partial_budget, const float* conv_w = nullptr, int conv_width = 0);

// Synchronises `stream`, reads the device status word at `word_dev` and maps it to a status.
int read_status_word(const void* word_dev, void* stream);

// Workspace bytes attn_fwd_impl needs with the given chunk budget (0 on invalid arguments).
size_t workspace_bytes_for(int nseq, const int32_t* cu_host, int Hq, int Hkv, int d,
                           int block_size, int topk, size_t partial_budget);

}  // namespace moba
