/*
 * bpt.h -- C ABI of libbpt: the forward pass of one pre-LN Blockwise Parallel
 * Transformer (BPT) layer on an NVIDIA B200 (sm_100a).
 *
 * What the layer computes ("Blockwise Parallel Transformer — BPT",
 * aicassindra.com, sections "The bottleneck that survives FlashAttention" and
 * "The fused blockwise algorithm"), per batch element and token row:
 *
 *   U = LN1(x);  Q = U W_Q;  K = U W_K;  V = U W_V
 *   per head t (columns t*d_k .. (t+1)*d_k, d_k = d / h):
 *       o_t = softmax(Q_t K_t^T / sqrt(d_k) [causal: keys j <= i]) V_t
 *   y = x + o W_O
 *   Z = y + GELU(LN2(y) W_1 + b_1) W_2 + b_2
 *
 * LN(v) = gamma * (v - mean) / sqrt(var + 1e-5) + beta over the d features of
 * a token (biased variance); GELU(z) = z/2 (1 + erf(z / sqrt 2)).  Q, K, V and
 * W_O carry no bias.
 *
 * How it is computed: blockwise, as the pages' two-level loop.  The outer loop
 * over query blocks of b rows (b = 128 for bf16, 64 for fp32) runs in waves of
 * at most BPT_WAVE_BLOCKS concurrent blocks; for each wave the kernels run
 * exact blockwise attention with an online softmax (causal blocks j > i are
 * skipped), then W_O + residual, LN2, W_1 + b_1 + GELU and W_2 + b_2 +
 * residual for the wave's rows only.  Neither the [N, N] scores nor the
 * [N, d_ff] FFN hidden state ever exists; the only sequence-shaped buffers are
 * x, out and the Q/K/V projection in the workspace.
 *
 * Conventions shared by every entry point:
 *   - All pointers except `bytes` and the profile arrays are DEVICE pointers
 *     on the current CUDA device, 16-byte aligned.  The caller owns every
 *     buffer; the library never allocates or frees device memory.
 *   - Weights are row-major [d_in, d_out] (the layer computes x W).
 *   - Work is enqueued on `stream` and the call returns before it finishes.
 *   - Argument errors are reported by the return value BEFORE anything is
 *     enqueued.  A wait inside a kernel that runs out of time (a lost
 *     signal; never expected) makes the kernel exit early and sets an error
 *     word in the workspace header, read by bpt_read_device_error.
 */
#ifndef BPT_H_
#define BPT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BPT_OK = 0,
  BPT_ERR_INVALID_ARG = 1, /* null or misaligned pointer, inconsistent sizes */
  BPT_ERR_UNSUPPORTED = 2, /* valid layer the kernels do not handle (see below) */
  BPT_ERR_WORKSPACE = 3,   /* workspace smaller than bpt_layer_workspace_size */
  BPT_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  BPT_ERR_TIMEOUT = 5,     /* a kernel gave up waiting (device error word) */
  BPT_ERR_RANGE = 6        /* an fp16 tensor-core operand overflowed (device error word) */
} bpt_status;

typedef enum {
  BPT_F32 = 0,  /* x, weights, params fp32; fp32 arithmetic on CUDA cores */
  BPT_BF16 = 1  /* x, weights, params bf16; tensor cores with fp16 operands
                   (see below), fp32 accumulation */
} bpt_dtype;

/* Same object as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* bpt_stream_t;

/* Maximum query blocks processed concurrently (one wave of the outer loop). */
#define BPT_WAVE_BLOCKS 256

/*
 * bpt_layer_workspace_size -- device workspace bytes bpt_layer_forward needs.
 *
 * Pure host arithmetic.  Layout (each region 1024-byte aligned):
 *   [0, 256)       header; uint32 at offset 0 = device error word
 *   weights        BPT_BF16 only: fp16 copies of W_Q, W_K, W_V, W_O ([d, d]
 *                  each), W_1 [d, d_ff], W_2 [d_ff, d], in that order
 *   QKV            [B*N, 3d] (Q | K | V per row); fp16 for BPT_BF16, fp32
 *                  for BPT_F32 (the "operand type" below)
 *   block scratch  P*b rows of o [d], LN2(y) [d] and FFN hidden [d_ff], in
 *                  the operand type, P = blocks in the largest wave
 *                  (<= BPT_WAVE_BLOCKS)
 * The scratch term does not grow with N once B*ceil(N/b) >= BPT_WAVE_BLOCKS.
 * Returns BPT_ERR_INVALID_ARG for bytes == NULL or negative / inconsistent
 * sizes, BPT_ERR_UNSUPPORTED for shapes bpt_layer_forward rejects.
 */
bpt_status bpt_layer_workspace_size(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                    int causal, bpt_dtype dtype, size_t* bytes);

/*
 * bpt_layer_forward -- Z = layer(x), written to `out`.
 *
 *   x     [B, N, d]  dtype     layer input (residual stream)
 *   ln1   [2, d]     dtype     LN1 gamma (row 0) and beta (row 1)
 *   W_Q, W_K, W_V, W_O [d, d]  dtype
 *   ln2   [2, d]     dtype     LN2 gamma, beta
 *   W_1   [d, d_ff]  dtype;  b_1 [d_ff] dtype
 *   W_2   [d_ff, d]  dtype;  b_2 [d]    dtype
 *   causal  nonzero: token i attends to tokens j <= i; zero: to all tokens
 *   out   [B, N, d]  fp32      layer output; also used as scratch for LN1(x)
 *                              before it is written, so it must not alias any
 *                              input
 *   workspace / workspace_bytes   device buffer of >= the size above
 *
 * Supported shapes: d = h * d_k; d % 8 == 0.
 *   BPT_BF16: d_k in {64, 128}; d % 64 == 0; d_ff % 64 == 0; any N >= 1
 *             (a ragged last block is masked).
 *   BPT_F32:  d_k <= 128; d_ff % 4 == 0; any N >= 1.
 *   B * N <= 2^30 tokens.
 * B == 0 or N == 0: nothing to do, returns BPT_OK without touching memory.
 * Results are deterministic: the same inputs give bitwise the same `out`.
 *
 * Precision of BPT_BF16: the tensor cores take fp16 operands (same rate as
 * bf16, 3 more mantissa bits).  Each call first copies the six bf16 weight
 * matrices to fp16 in the workspace; the copy is exact for magnitudes in
 * [2^-14, 65504] and has absolute error <= 2^-25 below.  LN outputs, Q/K/V,
 * the softmax weights P, the attention output and the FFN hidden state are
 * rounded to fp16; every product is accumulated in fp32; the residual stream
 * y and the output Z stay fp32.  A weight or an fp16 intermediate beyond
 * +-65504 (or NaN) sets BPT_ERR_RANGE in the device error word.
 */
bpt_status bpt_layer_forward(const void* x, const void* ln1, const void* W_Q, const void* W_K,
                             const void* W_V, const void* W_O, const void* ln2, const void* W_1,
                             const void* b_1, const void* W_2, const void* b_2, int64_t B,
                             int64_t N, int64_t d, int64_t h, int64_t d_ff, int causal,
                             bpt_dtype dtype, float* out, void* workspace, size_t workspace_bytes,
                             bpt_stream_t stream);

/*
 * bpt_layer_forward_train -- bpt_layer_forward that also writes the per-row
 * softmax statistics the backward pass recomputes from ("Blockwise Parallel
 * Transformer — BPT", section "The backward pass": the forward keeps the
 * layer input, the layer output and, per row, the softmax statistics (m, l),
 * so that each block's attention can be recomputed exactly in one pass).
 *
 *   stats [B, h, N, 2] fp32, device, caller-owned, 8-byte aligned; must not
 *         overlap x, out or the workspace.  For batch b, head t and query
 *         row i, with s_j = q_i . k_j / sqrt(d_k) over the keys row i may
 *         attend to (j <= i when causal):
 *           stats[b, t, i, 0] = m = max_j s_j
 *           stats[b, t, i, 1] = l = sum_j exp(s_j - m)
 *         computed from the same scores the forward uses (fp16 Q, K for
 *         BPT_BF16), so log(l) + m is that row's log-sum-exp.
 * Every other argument, the supported shapes, the results in `out` and the
 * workspace are those of bpt_layer_forward.  Returns BPT_ERR_INVALID_ARG for
 * stats == NULL, misaligned or overlapping; otherwise as bpt_layer_forward.
 */
bpt_status bpt_layer_forward_train(const void* x, const void* ln1, const void* W_Q,
                                   const void* W_K, const void* W_V, const void* W_O,
                                   const void* ln2, const void* W_1, const void* b_1,
                                   const void* W_2, const void* b_2, int64_t B, int64_t N,
                                   int64_t d, int64_t h, int64_t d_ff, int causal,
                                   bpt_dtype dtype, float* out, float* stats, void* workspace,
                                   size_t workspace_bytes, bpt_stream_t stream);

/*
 * bpt_layer_forward_bsfa -- bpt_layer_forward with block-sparse gating of the
 * attention ("Block Sparse Flash Attention", sections "Methodology and
 * Mechanism" and "Gating Mechanism and Threshold Calibration": exact scores
 * first, then the block's maximum score against a threshold per head and
 * query-block position decides whether the value block is processed).
 *
 * Blocks are the kernel's 128-row query and key blocks; nb = ceil(N / 128).
 * For batch b, head t, query block i and a key block j the attention visits
 * (j <= i when causal, every j otherwise):
 *   s_max = max of s = q.k / sqrt(d_k) over the block pair's valid query rows
 *           (position < N) and allowed keys (position < N; j' <= i' causal),
 *           from the same fp16 Q, K and fp32 accumulation as the scores;
 *   kept  = (j == i) || s_max >= thresholds[t * nb + i].
 * A pruned block contributes nothing: not to the row maxima and sums of the
 * softmax, not to the output (no P V product, no exponentials).  The
 * diagonal block is always kept, so every row has keys.  A NaN threshold
 * prunes every off-diagonal block of its query block.
 *
 *   thresholds [h, nb] fp32, device, 4-byte aligned: T in units of s, shared
 *              by the batch; must not overlap out or the workspace.  -inf
 *              keeps every block (the output is then bitwise that of
 *              bpt_layer_forward); +inf keeps only the diagonal.
 *   block_max  [B, h, nb, nb] fp32 or NULL: s_max of every visited pair
 *              (calibration input); entries of unvisited pairs untouched.
 *   kept       [B, h, nb, nb] uint8 or NULL: 1 where the pair was processed,
 *              0 where pruned; unvisited pairs untouched.
 * block_max and kept must not overlap x, out, the workspace, thresholds or
 * each other.  Every other argument, the supported shapes and the workspace
 * are those of bpt_layer_forward.  V tiles are still loaded for pruned
 * blocks (the K/V ring fetches them before the scores exist).
 * Returns BPT_ERR_UNSUPPORTED for dtype BPT_F32, BPT_ERR_INVALID_ARG for a
 * NULL, misaligned or overlapping buffer; otherwise as bpt_layer_forward.
 */
bpt_status bpt_layer_forward_bsfa(const void* x, const void* ln1, const void* W_Q,
                                  const void* W_K, const void* W_V, const void* W_O,
                                  const void* ln2, const void* W_1, const void* b_1,
                                  const void* W_2, const void* b_2, int64_t B, int64_t N,
                                  int64_t d, int64_t h, int64_t d_ff, int causal,
                                  bpt_dtype dtype, const float* thresholds, float* block_max,
                                  uint8_t* kept, float* out, void* workspace,
                                  size_t workspace_bytes, bpt_stream_t stream);

/*
 * bpt_layer_backward_workspace_size -- device workspace bytes
 * bpt_layer_backward needs (pure host arithmetic) for a layer of the given
 * dtype; the shape rules of bpt_layer_workspace_size.
 */
bpt_status bpt_layer_backward_workspace_size(int64_t B, int64_t N, int64_t d, int64_t h,
                                             int64_t d_ff, int causal, bpt_dtype dtype,
                                             size_t* bytes);

/*
 * bpt_layer_backward -- gradients of sum(Z * dZ) with respect to x and every
 * parameter, by the block recomputation of "Blockwise Parallel Transformer —
 * BPT", section "The backward pass": from the layer input and the per-row
 * softmax statistics of bpt_layer_forward_train, each block's scores,
 * attention output and FFN hidden are recomputed and consumed at once; no
 * [N, N] or [N, d_ff] tensor is formed (the FFN hidden exists for one wave of
 * query blocks at a time, as in the forward).
 *
 *   x, ln1, W_Q .. b_2   the forward's inputs (dtype, as bpt_layer_forward)
 *   stats [B, h, N, 2] fp32   the (m, l) bpt_layer_forward_train wrote
 *   dZ    [B, N, d] fp32      upstream gradient of the layer output
 * Outputs, fp32, overwritten (not accumulated):
 *   dx [B, N, d]; d_ln1 [2, d] (d gamma1; d beta1); dW_Q, dW_K, dW_V, dW_O
 *   [d, d]; d_ln2 [2, d]; dW_1 [d, d_ff]; db_1 [d_ff]; dW_2 [d_ff, d];
 *   db_2 [d].
 * All pointers are device pointers, 16-byte aligned; outputs must not
 * overlap each other, the workspace, x, stats or dZ.  Workspace: >=
 * bpt_layer_backward_workspace_size bytes, caller-owned.
 *
 * Arithmetic, BPT_BF16: the GEMMs run on the tensor cores with fp16 operands
 * (the activations, upstream gradient and intermediate gradients rounded to
 * fp16 as in the forward) and fp32 accumulation; weight gradients accumulate
 * in fp32 across waves; LayerNorm, GELU' and the bias / gamma / beta sums are
 * fp32 (the sums in a fixed order: results are deterministic).  The
 * attention gradients recompute P = exp(s - m) / l on the tensor cores (fp16
 * Q, K, V, dO, P and dS, fp32 accumulation), dK and dV by key block and dQ
 * by query block, without atomics.  BPT_F32: the same schedule with every
 * product and sum in fp32 on the CUDA cores (meant for small layers: the
 * attention gradients take one warp per row and head).
 * Returns BPT_ERR_INVALID_ARG for a null,
 * misaligned or overlapping pointer; BPT_ERR_WORKSPACE if the workspace is
 * too small; otherwise as bpt_layer_forward (device errors via
 * bpt_read_device_error).
 */
bpt_status bpt_layer_backward(const void* x, const void* ln1, const void* W_Q, const void* W_K,
                              const void* W_V, const void* W_O, const void* ln2, const void* W_1,
                              const void* b_1, const void* W_2, const void* b_2,
                              const float* stats, const float* dZ, int64_t B, int64_t N,
                              int64_t d, int64_t h, int64_t d_ff, int causal, bpt_dtype dtype,
                              float* dx, float* d_ln1, float* dW_Q, float* dW_K, float* dW_V,
                              float* dW_O, float* d_ln2, float* dW_1, float* db_1, float* dW_2,
                              float* db_2, void* workspace, size_t workspace_bytes,
                              bpt_stream_t stream);

/*
 * bpt_read_device_error -- synchronises `stream`, reads and clears the error
 * word in the workspace header (written by the latest bpt_layer_forward on
 * this workspace).  Returns BPT_OK if nothing was recorded, BPT_ERR_TIMEOUT if
 * a kernel gave up waiting, BPT_ERR_RANGE if an fp16 operand overflowed
 * (*site, if non-NULL, receives the code of the place that recorded it), or
 * BPT_ERR_CUDA if synchronisation failed.
 */
bpt_status bpt_read_device_error(void* workspace, bpt_stream_t stream, uint32_t* site);

/* Human-readable name of a status code (static string). */
const char* bpt_status_string(bpt_status status);

/*
 * Optional per-kernel timing, for measurement only.  While enabled, every
 * launch made by bpt_layer_forward is bracketed by CUDA events recorded on the
 * launching stream (host-side event objects, no device memory).
 * bpt_profile_read synchronises the recorded events, adds the elapsed time
 * and launch count per kernel kind into ms[k] / launches[k] for
 * k < min(n, BPT_KIND_COUNT), and clears the record.
 */
enum {
  BPT_KIND_LN1 = 0,
  BPT_KIND_QKV = 1,
  BPT_KIND_ATTN = 2,
  BPT_KIND_WO = 3,
  BPT_KIND_LN2 = 4,
  BPT_KIND_W1 = 5,
  BPT_KIND_W2 = 6,
  BPT_KIND_CVT = 7, /* bf16 -> fp16 weight copy */
  BPT_KIND_COUNT = 8
};
bpt_status bpt_profile_enable(int enable);
bpt_status bpt_profile_read(double* ms, int64_t* launches, int n);

/*
 * bpt_debug_set_max_wave -- TEST HOOK: caps the query blocks of a wave at
 * `blocks` (1..BPT_WAVE_BLOCKS; 0 restores BPT_WAVE_BLOCKS) for the calls
 * that follow, so that small layers exercise the multi-wave paths (a
 * sequence split over several waves, or one sequence per wave).  Results
 * are the same up to the order of fp32 sums; workspace sizes must be queried
 * after the call.  Returns BPT_ERR_INVALID_ARG outside that range.
 */
bpt_status bpt_debug_set_max_wave(int64_t blocks);

/*
 * bpt_debug_set_attn_qpc -- TUNING HOOK: query blocks per attention CTA for
 * the calls that follow.  2 (the default) pairs two 128-row query blocks in
 * one CTA, so each K/V tile brought in from L2 serves 256 query rows; 1
 * gives every query block its own CTA.  ("Blockwise Parallel Transformer —
 * BPT", section "Choosing the block size: arithmetic intensity": the FLOPs
 * done per byte re-read equal the rows a block shares them over; the pages
 * state it for the FFN weights, and the same ratio holds for the K/V tiles
 * each query block re-reads, 4 b d_k FLOPs per 4 d_k bytes of K and V per
 * key.)  Outputs are bitwise the same either way: a query block's
 * arithmetic does not depend on its partner.  Returns BPT_ERR_INVALID_ARG
 * for any other value.
 */
bpt_status bpt_debug_set_attn_qpc(int qpc);

/*
 * bpt_debug_inject_fault -- TEST HOOK for the failure-detection path.  The
 * next BPT_BF16 bpt_layer_forward makes one CTA skip one TMA load, so that
 * the wait for it runs out (after about 2 s) instead of completing:
 *   code 1: the QKV GEMM's CTA 0 never loads its first stage;
 *   code 2: the first attention wave's CTA 0 never loads V_0.
 * The kernel then records BPT_ERR_TIMEOUT in the device error word, drains
 * the loads and tensor-core work it did issue, frees its tensor memory and
 * exits; the layer's output is garbage for that call and the context stays
 * usable.  code 0 cancels.  The hook is consumed by one forward call.
 * Returns BPT_ERR_INVALID_ARG for other codes.
 */
bpt_status bpt_debug_inject_fault(int code);

/* Kernel launches one bpt_layer_forward call makes for these sizes. */
bpt_status bpt_layer_launch_count(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                  int causal, bpt_dtype dtype, int64_t* launches);

/*
 * bpt_layer_forward_static -- bpt_layer_forward for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a deployment
 * convenience of this library, not part of the method.
 *
 * Some callers are not allowed to allocate: code that runs while its stream is
 * being captured into a CUDA graph (an allocation may synchronise the device
 * and break the capture), plug-ins whose host framework owns all device memory,
 * and latency-critical loops that cannot pay for an allocation.  This entry
 * point takes the same arguments as bpt_layer_forward minus the workspace and
 * uses instead a workspace of BPT_STATIC_WORKSPACE_BYTES that lives in a
 * file-scope __device__ array of the library.  The caller still provides x,
 * the parameters and out.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 *   - Size limit: layers whose bpt_layer_workspace_size exceeds
 *     BPT_STATIC_WORKSPACE_BYTES are rejected with BPT_ERR_WORKSPACE before
 *     anything is enqueued (for example B=1, N=2048, d=768, d_ff=3072 fits;
 *     the larger long-context layers do not and need bpt_layer_forward).
 *   - Memory: every GPU that loads the library holds the array until the
 *     process exits, whether or not this entry point is used.
 *   - First call on a device: it looks up the array's device address (once
 *     per device, with that device current).  Make that first call before any
 *     stream capture begins.
 *   - Sharing: all calls on a device use the same array, and it keeps the
 *     last call's contents (each call clears the header it needs).  Calls
 *     whose work overlaps on the GPU (different streams, no ordering) race on
 *     the array and give undefined results: order them on one stream or with
 *     events.
 *   - Profiling: returns BPT_ERR_INVALID_ARG while bpt_profile_enable is on
 *     (profiling creates event objects).
 *   - A kernel that gives up waiting records it in the array's header, which
 *     the caller cannot read; as with any timeout, `out` is then undefined.
 */
#define BPT_STATIC_WORKSPACE_BYTES (64u * 1024u * 1024u)
bpt_status bpt_layer_forward_static(const void* x, const void* ln1, const void* W_Q,
                                    const void* W_K, const void* W_V, const void* W_O,
                                    const void* ln2, const void* W_1, const void* b_1,
                                    const void* W_2, const void* b_2, int64_t B, int64_t N,
                                    int64_t d, int64_t h, int64_t d_ff, int causal,
                                    bpt_dtype dtype, float* out, bpt_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BPT_H_ */
