/*
 * moba.h — C ABI of libmoba.so: the MoBA (Mixture of Block Attention) causal prefill forward
 * pass on NVIDIA B200 (sm_100a).
 *
 * The method [MoBA paper summary (atlas.scime.ai), "Approach"; MoBA README (rpkg.in mirror),
 * "Introducing MoBA"]: keys of every sequence are cut into fixed-size blocks; each block is
 * mean-pooled into a centroid; every query head scores the PAST blocks of its sequence by
 * q . centroid (a gate with no parameters), never a future block, always keeps its own current
 * block and routes to the top-k blocks (the current one counted in k). Attention is exact softmax
 * attention over the keys of the selected blocks, causal inside the current block.
 *
 * Conventions shared by every entry point
 *   - Layouts (row-major, contiguous):
 *       q            bf16  [T, Hq,  d]
 *       k, v         bf16  [T, Hkv, d]
 *       cu_seqlens   int32 [nseq + 1], cu[0] = 0, non-decreasing, cu[nseq] = T (packed varlen)
 *       centroids    fp32  [NB, Hkv, d]   NB = sum_s ceil((cu[s+1]-cu[s]) / block_size)
 *       block_idx    int32 [Hq, T, topk]  local block ids of the sequence, ascending, the
 *                                         current block last among the valid ones, -1 padded
 *       o            bf16  [T, Hq, d]
 *       lse          fp32  [Hq, T]        natural-log sum-exp of the scaled logits
 *     Global block b numbers the blocks of sequence 0, then sequence 1, ... Blocks never cross
 *     sequence boundaries; the last block of a sequence may be short.
 *   - Query head h reads kv head h / (Hq / Hkv) (contiguous GQA groups).
 *   - The gate score is the unscaled dot product q . centroid in fp32; `scale` only multiplies the
 *     attention logits.
 *   - cu_seqlens is passed twice: on the device (read by kernels) and on the host (read to size
 *     grids and the workspace without a device sync). Both must hold the same values.
 *   - Memory: the caller owns every buffer (inputs, outputs and the workspace). The library never
 *     allocates device memory. All device pointers must be 16-byte aligned.
 *   - Streams: all work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     Calls return after enqueueing; they never synchronise the device. Outputs are valid once
 *     the stream reaches that point.
 *   - Errors: every call returns a moba_status. Argument errors are detected on the host before
 *     anything is launched. Kernels never trap: a device-side failure (a bounded wait that ran
 *     out) is recorded in the workspace's status word; read it with moba_device_status().
 *   - Supported shapes: d in {64, 128}; Hq % Hkv == 0; block_size a positive multiple of 64;
 *     1 <= topk <= 64; at most 32768 blocks in one sequence; T < 2^31 / Hq.
 *   - Device: compute capability 10.0 (B200, sm_100a); anything else gives
 *     MOBA_ERR_UNSUPPORTED.
 */
#ifndef MOBA_H_
#define MOBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOBA_OK = 0,
  MOBA_ERR_ARG = -1,          /* invalid argument (null / misaligned pointer, bad sizes)      */
  MOBA_ERR_UNSUPPORTED = -2,  /* valid but outside the supported shapes or device             */
  MOBA_ERR_WORKSPACE = -3,    /* workspace smaller than moba_workspace_bytes()                */
  MOBA_ERR_CUDA = -4,         /* a CUDA runtime / driver call or a kernel launch failed       */
  MOBA_ERR_DEVICE_CHECK = -5, /* a device-side check failed, e.g. a routing row that breaks its
                                 contract (see moba_device_status)                            */
  MOBA_ERR_TIMEOUT = -6       /* a bounded device-side wait ran out (see moba_device_status)  */
} moba_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* moba_status_string(int status);

/* Library version, (major << 16) | (minor << 8) | patch. */
int moba_version(void);

/*
 * Bytes of device workspace moba_attn_fwd needs for this problem (0 on invalid arguments).
 * Depends only on the host-side sizes. The workspace holds block tables, centroids, the routing
 * (when the caller passes no block_idx_out), the inverted routing lists (at d = 64 with a copy of
 * each routed query row) and the per-block partial outputs of one query chunk; chunks are sized
 * so that these per-chunk parts stay under a fixed budget.
 */
size_t moba_workspace_bytes(int nseq, const int32_t* cu_seqlens_host, int Hq, int Hkv, int d,
                            int block_size, int topk);

/*
 * Step 1 — block centroids [MoBA paper summary, "Approach": mean-pooled keys].
 *   centroids[b, g, :] = (1 / n_b) * sum of k[t, g, :] over the n_b keys of global block b,
 *   accumulated in fp32 (one pass over K with 16-byte loads).
 * k: device bf16 [T, Hkv, d]; centroids: device fp32 [NB, Hkv, d] (written).
 */
int moba_centroids(const void* k, const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                   int nseq, int Hkv, int d, int block_size, float* centroids, void* stream);

/*
 * Step 1 with a short key convolution before pooling [FlashMoBA story: short convolutions inside
 * blocks cluster related keys and raise the routing signal]. The keys of every block first pass
 * through a depthwise causal convolution of width W that never reaches into another block:
 *   kconv[t, g, :] = sum_{m=0}^{W-1} conv_w[m, g, :] * k[t - m, g, :]   (terms with t - m before
 *                    the block's first key left out),
 * and the centroid is the mean of kconv over the block. Linear, no bias or activation (the pages
 * give no kernel width, weights or activation). Only the routing sees the convolved keys;
 * attention reads k as given.
 * conv_w: device fp32 [W, Hkv, d], 16-byte aligned, 1 <= W <= 16 (MOBA_ERR_UNSUPPORTED above);
 * the other arguments as for moba_centroids. Costs K's single pass plus W - 1 key rows per block.
 */
int moba_centroids_kconv(const void* k, const float* conv_w, int conv_width,
                         const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host, int nseq,
                         int Hkv, int d, int block_size, float* centroids, void* stream);

/*
 * Step 2 — parameter-less causal top-k gate [MoBA paper summary, "Approach"; MoBA README,
 * "Parameter-less Gating Mechanism"].
 *   For query t in local block i of its sequence and head h (kv head g = h / (Hq/Hkv)):
 *   s_j = q[t,h] . centroids[base + j, g] for past blocks j < i; the selection is {i} plus the
 *   top-(topk-1) past blocks by s_j (equal scores: lower j first); if topk-1 >= i every block
 *   0..i is selected. The T x NB score matrix is never materialised.
 * q: device bf16 [T, Hq, d]; centroids: device fp32 [NB, Hkv, d] (e.g. from moba_centroids);
 * block_idx: device int32 [Hq, T, topk] (written: ascending, -1 padded).
 */
int moba_gate_topk(const void* q, const float* centroids, const int32_t* cu_seqlens_dev,
                   const int32_t* cu_seqlens_host, int nseq, int Hq, int Hkv, int d,
                   int block_size, int topk, int32_t* block_idx, void* stream);

/*
 * The whole forward pass: centroids -> gate -> routing inversion -> block-sparse attention ->
 * LSE merge [MoBA paper summary, "Approach"; FlashMoBA story: gathering scattered blocks into
 * dense tiles].
 *   o[t, h, :] = sum_u softmax_u(scale * q[t,h] . k[u,g]) v[u, g] over the keys u of the selected
 *   blocks (keys <= t inside the current block); lse[h, t] = log sum_u exp(scale * q . k_u).
 * block_idx_in : nullable. When given (device int32 [Hq, T, topk], same format as the gate's
 *                output), this routing is used and no centroid / gate work runs. Every row must
 *                hold exactly n = min(topk, i + 1) blocks for a query in local block i: slots
 *                0 .. n-2 strictly ascending past blocks (0 <= j < i), slot n-1 the current block
 *                i, the other slots -1. The partial results of a row live in the slots of its
 *                blocks and the merge reads slots 0 .. n-1, so a row with fewer blocks would mix
 *                in slots nobody wrote. Rows are checked on the device: a row that breaks the
 *                contract makes moba_device_status return MOBA_ERR_DEVICE_CHECK (the outputs of
 *                that call are then undefined; out-of-range entries are never dereferenced).
 * block_idx_out: nullable. When given, receives the routing that was used.
 * workspace    : device buffer of at least moba_workspace_bytes(...) bytes, 256-byte aligned.
 */
int moba_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_dev,
                  const int32_t* cu_seqlens_host, int nseq, int Hq, int Hkv, int d,
                  int block_size, int topk, float scale, const int32_t* block_idx_in,
                  int32_t* block_idx_out, void* o, float* lse, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * moba_attn_fwd whose routing is computed on short-convolved keys (see moba_centroids_kconv):
 * the same forward pass, with the centroids pooled from the convolved keys. There is no routing
 * input (a given routing makes the convolution irrelevant); the workspace is sized by
 * moba_workspace_bytes as for moba_attn_fwd.
 */
int moba_attn_fwd_kconv(const void* q, const void* k, const void* v, const float* conv_w,
                        int conv_width, const int32_t* cu_seqlens_dev,
                        const int32_t* cu_seqlens_host, int nseq, int Hq, int Hkv, int d,
                        int block_size, int topk, float scale, int32_t* block_idx_out, void* o,
                        float* lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * MoBA decode and chunked prefill against a KV cache [MoBA paper summary, "Approach" for the
 * routing; its "Limitations": the paper's generation fell back to full attention, this applies
 * the same block routing to the newest rows of a cache].
 *   The cache holds nseq packed sequences: k_cache, v_cache bf16 [T, Hkv, d] with cu_seqlens as in
 *   moba_attn_fwd (sequence s has L_s = cu[s+1] - cu[s] cached tokens, the new ones included).
 *   Query rows: cu_seqlens_q [nseq + 1] (cuq[0] = 0, non-decreasing) gives n_s = cuq[s+1] - cuq[s]
 *   <= L_s rows per sequence, which are its last n_s tokens (decode: n_s = 1). q bf16 [Tq, Hq, d]
 *   with Tq = cuq[nseq]; row r of sequence s sits at position L_s - n_s + (r - cuq[s]).
 *   Each row gets exactly the result moba_attn_fwd would give that token over its whole
 *   sequence: the gate scores the past blocks j < i of its own position with the cached
 *   centroids (fp32 [NB, Hkv, d], e.g. from moba_centroids on k_cache; only past blocks, which
 *   are complete, are read, so a block's centroid needs computing once, when it completes), keeps
 *   the current block and the top-(topk-1) past blocks, and attends their keys up to its own
 *   position.
 * block_idx_in : nullable [Hq, Tq, topk] routing to use instead of the gate (same contract as
 *                moba_attn_fwd's; centroids may then be NULL).
 * block_idx_out: nullable [Hq, Tq, topk], receives the routing used.
 * o: bf16 [Tq, Hq, d]; lse: fp32 [Hq, Tq] (a sequence with no cached key gives o = 0, lse = -inf).
 * workspace: at least moba_decode_workspace_bytes(...) bytes, 256-byte aligned.
 * The path is HBM-bound: each (row, head) reads the K and V rows of its selected blocks once.
 */
size_t moba_decode_workspace_bytes(int nseq, const int32_t* cu_seqlens_host,
                                   const int32_t* cu_seqlens_q_host, int Hq, int Hkv, int d,
                                   int block_size, int topk);
int moba_decode_fwd(const void* q, const void* k_cache, const void* v_cache,
                    const float* centroids, const int32_t* cu_seqlens_dev,
                    const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_q_dev,
                    const int32_t* cu_seqlens_q_host, int nseq, int Hq, int Hkv, int d,
                    int block_size, int topk, float scale, const int32_t* block_idx_in,
                    int32_t* block_idx_out, void* o, float* lse, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * Backward pass of the routed attention [MoBA README, "Introducing MoBA": trainable block sparse
 * attention]. The routing is held fixed: the top-k gate is piecewise constant in q and the
 * centroids, so no gradient flows through the selection (as in top-k mixture-of-experts routing).
 * For every row (t, h) over its attended keys u (the keys of its selected blocks, causal inside
 * its own block), with p_u = exp(scale q.k_u - lse[h, t]), D = dO[t,h] . o[t,h] and
 * dS_u = p_u (dO[t,h] . v_u - D):
 *   dq[t, h] = scale sum_u dS_u k_u,  dk[u, g] = scale sum dS_u q[t, h],  dv[u, g] = sum p_u dO,
 * the last two summed over every row that attends u and every query head h of kv group g.
 * q, k, v, o, d_o: bf16 as in moba_attn_fwd (o and lse are that call's outputs; d_o [T, Hq, d]);
 * block_idx: the routing the forward pass used ([Hq, T, topk], same contract as block_idx_in; a
 * row that breaks it is reported by moba_device_status as MOBA_ERR_DEVICE_CHECK);
 * dq [T, Hq, d], dk, dv [T, Hkv, d]: bf16 outputs (fp32 accumulation; dq through an fp32
 * accumulator in the workspace, dk / dv in tensor memory, each key row written once).
 * workspace: at least moba_bwd_workspace_bytes(...) bytes, 256-byte aligned (routing lists of all
 * rows, D and the fp32 dq accumulator). T * Hq * topk < 2^31.
 */
size_t moba_bwd_workspace_bytes(int nseq, const int32_t* cu_seqlens_host, int Hq, int Hkv, int d,
                                int block_size, int topk);
int moba_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* d_o, const int32_t* block_idx, const int32_t* cu_seqlens_dev,
                  const int32_t* cu_seqlens_host, int nseq, int Hq, int Hkv, int d,
                  int block_size, int topk, float scale, void* dq, void* dk, void* dv,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * moba_attn_fwd for callers that cannot allocate device memory. The paper has no counterpart:
 * this is a deployment variant of the same computation.
 *
 * Some callers may not call cudaMalloc: plug-in code whose host application owns all device
 * memory through its own allocator or a fixed pool, and latency-critical paths that cannot
 * afford the implicit synchronisation an allocation may cause. This entry point allocates
 * nothing: its scratch memory is one static device array inside libmoba.so of
 * MOBA_NOALLOC_SCRATCH_BYTES, reserved on every GPU that loads the library until the process
 * exits. Arguments and results are those of moba_attn_fwd without routing in/out and workspace.
 *   - Returns MOBA_ERR_WORKSPACE, launching nothing, when the problem needs more scratch than the
 *     array holds (the routing [Hq, T, topk] int32 plus block tables, centroids and the chunked
 *     routing lists and partial outputs; partial outputs are chunked to a quarter of the array).
 *   - All calls share the array and it keeps the previous call's contents; each call clears what
 *     must start at zero on its own stream. Calls that overlap on the GPU race on the array and
 *     must be serialised by the caller.
 *   - The first call on a device looks up the array's device address (with that device
 *     current); make that first call before any stream capture begins.
 *   - The status word of the last call lives in the array; read it with moba_noalloc_status.
 */
#define MOBA_NOALLOC_SCRATCH_BYTES (64u << 20)
int moba_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                          const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host, int nseq,
                          int Hq, int Hkv, int d, int block_size, int topk, float scale, void* o,
                          float* lse, void* stream);

/*
 * Synchronises `stream`, then reads the status word of the last moba_attn_fwd_noalloc call on
 * the current device (the word sits in the library's static scratch array): MOBA_OK,
 * MOBA_ERR_TIMEOUT or MOBA_ERR_DEVICE_CHECK, as for moba_device_status. Calls that overlap on
 * the GPU share the word like the rest of the array.
 */
int moba_noalloc_status(void* stream);

/*
 * Synchronises `stream`, then reads the status word a moba_attn_fwd call left in `workspace`:
 * MOBA_OK; MOBA_ERR_TIMEOUT when a bounded device wait (or the drain after it) ran out; or
 * MOBA_ERR_DEVICE_CHECK when a routing row broke its contract or the kernel found its shared
 * memory misaligned. Outputs of a call with a status other than MOBA_OK are undefined. The word
 * is cleared by the next moba_attn_fwd on the same workspace; the first failure of a call wins.
 */
int moba_device_status(const void* workspace, void* stream);

/*
 * Diagnostics: sets the limit of one pipeline wait inside the attention kernel for later calls
 * (process-wide; ns = 0 restores the built-in 2 s) and returns the previous limit. A short limit
 * makes a wait run out on purpose, so that a test can see the abort path report
 * MOBA_ERR_TIMEOUT while the context stays usable; after an abort each CTA still waits for its
 * own copies and matrix products in flight, under a separate fixed 2 s limit, before it exits.
 */
unsigned long long moba_set_wait_limit_ns(unsigned long long ns);

/*
 * Diagnostics: with on != 0, later moba_attn_fwd calls make the attention kernel's MMA issuer
 * first wait on a barrier that nothing arrives on. The wait runs out after the pipeline-wait
 * limit (set a short one with moba_set_wait_limit_ns), the CTA raises its abort flag, every other
 * role gives up its own wait, drains its copies in flight and returns, and moba_device_status
 * reports MOBA_ERR_TIMEOUT: a way to exercise the abort path without a fault. Process-wide;
 * returns the previous setting. Never set in normal use.
 */
int moba_set_diag_stall(int on);

/*
 * Instrumentation (off by default; on from the start when the environment sets MOBA_TIMING=1).
 * When enabled, every kernel launch of the library is bracketed by CUDA events recorded on the
 * launching stream. Every launch is also bracketed by an NVTX range named for its class
 * (moba_centroids, moba_gate, ...), which profilers show and which costs nothing without one.
 * moba_timing_enable switches the timing on (enable != 0) or off and returns whether it was on
 * before the call (1 or 0). moba_timing_read synchronises the
 * recorded events and writes, for each kernel class, the summed device milliseconds and launch
 * count since the last reset; kernel classes, in order: centroid, gate, route_count, route_scan,
 * route_scatter, attention, merge, plan, densify (d = 64: the routed query rows copied into one
 * dense array), decode (moba_decode_fwd's kernels), bwd_dkdv, bwd_dq and bwd_aux (moba_attn_bwd's
 * key-stationary and query-stationary kernels, and its D / dQ conversion passes). Returns the
 * number of classes (13), or a negative status.
 */
int moba_timing_enable(int enable);
int moba_timing_reset(void);
int moba_timing_read(double* ms_per_class, long long* launches_per_class, int n);

/* Number of kernels this library has launched since it was loaded (all entry points). */
long long moba_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_H_ */
