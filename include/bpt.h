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
 * runs over query blocks of b rows (b = 128 for bf16, 64 for fp32).  For
 * BPT_BF16 layers (default schedule, BPT_SCHEDULE_FUSED): after LN1 and the
 * Q/K/V projection, one kernel runs exact blockwise attention with an online
 * softmax (causal blocks j > i are skipped) for every query block and writes
 * each block's output over that block's own queries; then one persistent
 * kernel takes the query blocks two at a time and, per block, forms
 * y = x + o W_O, LN2(y), the FFN hidden chunk by chunk (256 columns of d_ff
 * at a time) and Z = y + FFN + b_2, with the hidden of the blocks in flight
 * in a per-SM-pair scratch.  What exists at once:
 *   - never: the [N, N] scores;
 *   - sequence-shaped: x, out and the Q/K/V projection (workspace);
 *   - block-shaped: LN2(y) and the FFN hidden of at most
 *     2 * BPT_TAIL_MAX_PAIRS query blocks (the blocks in flight), so the
 *     [N, d_ff] hidden exists only when the whole layer has that few blocks
 *     (B * ceil(N / 128) <= 148).
 * BPT_SCHEDULE_WAVES (and every BPT_F32 layer) runs the body instead in
 * waves of at most BPT_WAVE_BLOCKS query blocks, five stream-ordered kernels
 * per wave, with the wave's o, LN2(y) and hidden in the workspace: the
 * [N, d_ff] hidden exists at once whenever B * ceil(N / b) <= BPT_WAVE_BLOCKS.
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

/* Maximum query blocks processed concurrently by one wave of the waves
 * schedule (BPT_SCHEDULE_WAVES, and every BPT_F32 layer). */
#define BPT_WAVE_BLOCKS 256
/* CTA pairs (two SMs each) of the fused schedule's layer-body kernel; each
 * pair has two 128-row query blocks in flight. */
#define BPT_TAIL_MAX_PAIRS 74

/* Schedules of the layer body after attention (bpt_options.schedule). */
enum {
  BPT_SCHEDULE_FUSED = 0, /* default: one persistent kernel, block-shaped scratch */
  BPT_SCHEDULE_WAVES = 1  /* waves of query blocks, one kernel per step per wave */
};

/*
 * bpt_options -- per-call choices of the *_opt entry points.  A NULL pointer,
 * or a zero-initialised struct, means the defaults.  Every choice gives the
 * same result up to the order of fp32 sums; the ones marked "bitwise" give
 * bitwise the same output.
 *   schedule  BPT_SCHEDULE_FUSED or BPT_SCHEDULE_WAVES (bitwise: both run
 *             the same per-element arithmetic).  BPT_F32 layers always use
 *             waves.  The backward pass always uses waves.
 *   attn_block  b, the query rows sharing each K/V tile: 0 = default
 *             (256), 64, 128, 256 or 512 (bitwise: the softmax arithmetic of a
 *             query row does not depend on b).  Each K/V tile brought into
 *             shared memory serves b query rows ("Blockwise Parallel
 *             Transformer — BPT", section "Choosing the block size:
 *             arithmetic intensity": FLOPs per byte re-read equal the rows
 *             sharing it).  256 pairs two 128-row query blocks in one CTA;
 *             128 gives every query block its own CTA; 64 runs one 64-row
 *             block per CTA, two CTAs per SM; 512 runs clusters of two
 *             256-row CTAs that each load half of every K/V tile and copy it
 *             to the other over distributed shared memory.  64 and 512 are
 *             dense attention only: the gated entry points return
 *             BPT_ERR_UNSUPPORTED with them.
 *   max_wave  waves schedule only: query blocks per wave, 0 = default
 *             (BPT_WAVE_BLOCKS), else 1..BPT_WAVE_BLOCKS; small values make
 *             small layers run the multi-wave paths (a sequence split over
 *             several waves).  Workspace sizes depend on it: query them with
 *             the same options.
 *   fault     TEST HOOK for the failure-detection path (BPT_BF16 forward
 *             only), 0 = none.  1: the QKV GEMM's CTA 0 never loads its first
 *             stage; 2: the attention's CTA 0 never loads V_0; 3 (fused
 *             schedule): the layer-body kernel's CTA 0 never loads its first
 *             A tile.  The wait for
 *             the missing load runs out (about 2 s), the kernel records
 *             BPT_ERR_TIMEOUT in the device error word, drains what it issued,
 *             frees its tensor memory and exits; `out` is garbage for that
 *             call and the context stays usable.
 *   reserved  must be 0.
 * Returns BPT_ERR_INVALID_ARG for any other value.
 */
typedef struct {
  int32_t schedule;
  int32_t attn_block;
  int64_t max_wave;
  int32_t fault;
  int32_t reserved;
} bpt_options;

/*
 * bpt_layer_workspace_size -- device workspace bytes bpt_layer_forward needs.
 *
 * Pure host arithmetic.  Layout (each region 1024-byte aligned):
 *   [0, 2048)      header: uint32 at offset 0 = device error word; bytes
 *                  [256, 1440) = counters the fused schedule's layer body
 *                  uses to hand work between CTA pairs
 *   weights        BPT_BF16 only: fp16 copies of W_Q, W_K, W_V, W_O ([d, d]
 *                  each), W_1 [d, d_ff], W_2 [d_ff, d], in that order
 *   QKV            [B*N, 3d] (Q | K | V per row); fp16 for BPT_BF16, fp32
 *                  for BPT_F32 (the "operand type" below).  The fused
 *                  schedule writes each row's attention output over its Q.
 *   block scratch  fused schedule: 256*P rows of LN2(y) [d] and FFN hidden
 *                  [d_ff] (fp16), P = min(BPT_TAIL_MAX_PAIRS, ceil(B*nb/2)),
 *                  nb = ceil(N / 128): at most 148*128*(2d + 2 d_ff) bytes,
 *                  for every N.  Waves schedule: P*b rows of o [d], LN2(y)
 *                  [d] and FFN hidden [d_ff] in the operand type, P = blocks
 *                  in the largest wave (<= BPT_WAVE_BLOCKS).
 * Returns BPT_ERR_INVALID_ARG for bytes == NULL or negative / inconsistent
 * sizes, BPT_ERR_UNSUPPORTED for shapes bpt_layer_forward rejects.
 * bpt_layer_workspace_size_opt: the same for the given options (NULL: the
 * defaults, as bpt_layer_workspace_size).
 */
bpt_status bpt_layer_workspace_size(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                    int causal, bpt_dtype dtype, size_t* bytes);
bpt_status bpt_layer_workspace_size_opt(int64_t B, int64_t N, int64_t d, int64_t h,
                                        int64_t d_ff, int causal, bpt_dtype dtype,
                                        const bpt_options* opts, size_t* bytes);

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
 * bpt_layer_forward_opt -- bpt_layer_forward with per-call options (see
 * bpt_options; NULL = the defaults) and optional statistics: `stats` NULL is
 * bpt_layer_forward, non-NULL is bpt_layer_forward_train (same layout and
 * rules).  The workspace must be at least bpt_layer_workspace_size_opt with
 * the same options.
 */
bpt_status bpt_layer_forward_opt(const void* x, const void* ln1, const void* W_Q,
                                 const void* W_K, const void* W_V, const void* W_O,
                                 const void* ln2, const void* W_1, const void* b_1,
                                 const void* W_2, const void* b_2, int64_t B, int64_t N,
                                 int64_t d, int64_t h, int64_t d_ff, int causal, bpt_dtype dtype,
                                 float* out, float* stats, void* workspace,
                                 size_t workspace_bytes, const bpt_options* opts,
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
 * bpt_layer_forward_train_keep_o -- bpt_layer_forward_train that also keeps
 * the attention output, so that bpt_layer_backward_keep_o need not recompute
 * it.  The pages' backward ("The backward pass") recomputes each block's
 * attention from (m, l); keeping o trades 2 B N d bytes of activation memory
 * for that recomputation (a full causal attention forward).  BPT_BF16 only.
 *
 *   o   [B, N, d] fp16, device, caller-owned, 16-byte aligned; must not
 *       overlap x, any parameter, out, stats or the workspace.  Row (b, i)
 *       holds the attention output of token i of sequence b, heads
 *       concatenated: softmax(q k^T / sqrt(d_k)) v per head, before W_O,
 *       exactly the fp16 values the layer body multiplied by W_O.
 *   opts  NULL or per-call options (as bpt_layer_forward_opt).
 * Everything else as bpt_layer_forward_train.  Returns BPT_ERR_UNSUPPORTED
 * for BPT_F32, BPT_ERR_INVALID_ARG for stats == NULL, o == NULL, misaligned
 * or overlapping buffers.
 */
bpt_status bpt_layer_forward_train_keep_o(const void* x, const void* ln1, const void* W_Q,
                                          const void* W_K, const void* W_V, const void* W_O,
                                          const void* ln2, const void* W_1, const void* b_1,
                                          const void* W_2, const void* b_2, int64_t B,
                                          int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                          int causal, bpt_dtype dtype, float* out, float* stats,
                                          void* o, void* workspace, size_t workspace_bytes,
                                          const bpt_options* opts, bpt_stream_t stream);

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
 * are those of bpt_layer_forward.  The value tile of a block is loaded only
 * when a query block that visits it keeps it (the kernel fetches V after the
 * gate decisions; the two query blocks of an attention CTA share each tile).
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
/* bpt_layer_forward_bsfa with per-call options (bpt_options; NULL = defaults). */
bpt_status bpt_layer_forward_bsfa_opt(const void* x, const void* ln1, const void* W_Q,
                                      const void* W_K, const void* W_V, const void* W_O,
                                      const void* ln2, const void* W_1, const void* b_1,
                                      const void* W_2, const void* b_2, int64_t B, int64_t N,
                                      int64_t d, int64_t h, int64_t d_ff, int causal,
                                      bpt_dtype dtype, const float* thresholds, float* block_max,
                                      uint8_t* kept, float* out, void* workspace,
                                      size_t workspace_bytes, const bpt_options* opts,
                                      bpt_stream_t stream);

/*
 * bpt_layer_backward_workspace_size -- device workspace bytes
 * bpt_layer_backward needs (pure host arithmetic) for a layer of the given
 * dtype; the shape rules of bpt_layer_workspace_size.
 */
bpt_status bpt_layer_backward_workspace_size(int64_t B, int64_t N, int64_t d, int64_t h,
                                             int64_t d_ff, int causal, bpt_dtype dtype,
                                             size_t* bytes);
bpt_status bpt_layer_backward_workspace_size_opt(int64_t B, int64_t N, int64_t d, int64_t h,
                                                 int64_t d_ff, int causal, bpt_dtype dtype,
                                                 const bpt_options* opts, size_t* bytes);

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
/* bpt_layer_backward with per-call options (attn_block and max_wave apply; the
 * backward always runs the waves schedule; fault must be 0). */
bpt_status bpt_layer_backward_opt(const void* x, const void* ln1, const void* W_Q,
                                  const void* W_K, const void* W_V, const void* W_O,
                                  const void* ln2, const void* W_1, const void* b_1,
                                  const void* W_2, const void* b_2, const float* stats,
                                  const float* dZ, int64_t B, int64_t N, int64_t d, int64_t h,
                                  int64_t d_ff, int causal, bpt_dtype dtype, float* dx,
                                  float* d_ln1, float* dW_Q, float* dW_K, float* dW_V,
                                  float* dW_O, float* d_ln2, float* dW_1, float* db_1,
                                  float* dW_2, float* db_2, void* workspace,
                                  size_t workspace_bytes, const bpt_options* opts,
                                  bpt_stream_t stream);

/*
 * bpt_layer_backward_keep_o -- bpt_layer_backward with the attention output
 * `o` that bpt_layer_forward_train_keep_o wrote for the same inputs (fp16
 * [B, N, d], 16-byte aligned, read only; must not overlap any output or the
 * workspace).  Each wave takes its o rows from `o` instead of recomputing
 * the attention forward; the gradients are bitwise those of
 * bpt_layer_backward (the recomputation reproduces o exactly).  BPT_BF16
 * only (BPT_ERR_UNSUPPORTED otherwise); workspace size as
 * bpt_layer_backward_workspace_size_opt with the same options.
 */
bpt_status bpt_layer_backward_keep_o(const void* x, const void* ln1, const void* W_Q,
                                     const void* W_K, const void* W_V, const void* W_O,
                                     const void* ln2, const void* W_1, const void* b_1,
                                     const void* W_2, const void* b_2, const float* stats,
                                     const void* o, const float* dZ, int64_t B, int64_t N,
                                     int64_t d, int64_t h, int64_t d_ff, int causal,
                                     bpt_dtype dtype, float* dx, float* d_ln1, float* dW_Q,
                                     float* dW_K, float* dW_V, float* dW_O, float* d_ln2,
                                     float* dW_1, float* db_1, float* dW_2, float* db_2,
                                     void* workspace, size_t workspace_bytes,
                                     const bpt_options* opts, bpt_stream_t stream);

/*
 * Sequence sharding over G GPUs ("Blockwise Parallel Transformer — BPT",
 * section "BPT and Ring Attention": BPT is the per-device kernel and the
 * sequence is split across devices, each device's queries needing the keys
 * and values of the others; section "Why parallel is in the name": query
 * blocks are independent).  Zig-zag ownership balances the causal work: the
 * sequence of N tokens is cut into 2G chunks of N / (2G) tokens and rank r
 * owns chunks r and 2G-1-r; its n_loc = N / G local rows are chunk r
 * followed by chunk 2G-1-r, in token order within each.  Per forward, each
 * rank calls
 *   1. bpt_layer_shard_project: LN1 and the Q/K/V projection of its own
 *      rows; writes K | V of those rows to kv_loc [B, n_loc, 2d] fp16 and
 *      keeps Q (and the fp16 weights) in its workspace;
 *   2. an all-gather of kv_loc over the G ranks into kv_all
 *      [G, B, n_loc, 2d] fp16 in this GPU's memory, rank-major (one NCCL
 *      all_gather_into_tensor; the library does no communication);
 *   3. bpt_layer_shard_forward: attention of its rows against every rank's
 *      K | V (read from kv_all through the chunk ownership, no reordering
 *      copy), then the fused layer body; writes Z of its rows to out
 *      [B, n_loc, d] fp32.
 * Step 3 must get the workspace step 1 used, unchanged, and the parameters
 * of step 1.  The output rows equal bitwise those of bpt_layer_forward on
 * the whole sequence (same per-element arithmetic).
 * Supported: BPT_BF16 only; N % (256 G) == 0 (whole 128-token blocks per
 * chunk); G >= 1; 0 <= rank < G; the shapes of bpt_layer_forward for
 * n_loc tokens.  x is the rank's local rows [B, n_loc, d].  kv_loc / kv_all
 * must not overlap out, the workspace or the inputs.  The workspace size is
 * bpt_layer_shard_workspace_size (that of bpt_layer_workspace_size for
 * n_loc tokens).  Returns BPT_ERR_UNSUPPORTED for other dtypes or N, and as
 * bpt_layer_forward otherwise.
 */
bpt_status bpt_layer_shard_workspace_size(int64_t B, int64_t N, int64_t G, int64_t d,
                                          int64_t h, int64_t d_ff, int causal, bpt_dtype dtype,
                                          size_t* bytes);
bpt_status bpt_layer_shard_project(const void* x, const void* ln1, const void* W_Q,
                                   const void* W_K, const void* W_V, const void* W_O,
                                   const void* ln2, const void* W_1, const void* b_1,
                                   const void* W_2, const void* b_2, int64_t B, int64_t N,
                                   int64_t G, int64_t rank, int64_t d, int64_t h, int64_t d_ff,
                                   int causal, bpt_dtype dtype, void* kv_loc, float* out,
                                   void* workspace, size_t workspace_bytes,
                                   bpt_stream_t stream);
bpt_status bpt_layer_shard_forward(const void* x, const void* ln1, const void* W_Q,
                                   const void* W_K, const void* W_V, const void* W_O,
                                   const void* ln2, const void* W_1, const void* b_1,
                                   const void* W_2, const void* b_2, int64_t B, int64_t N,
                                   int64_t G, int64_t rank, int64_t d, int64_t h, int64_t d_ff,
                                   int causal, bpt_dtype dtype, const void* kv_all, float* out,
                                   void* workspace, size_t workspace_bytes,
                                   bpt_stream_t stream);

/*
 * bpt_read_device_error -- synchronises `stream`, reads and clears the error
 * word in the workspace header (written by the latest call on this
 * workspace).  workspace == NULL reads the header of the array that
 * bpt_layer_forward_static uses as its workspace, on the current device.
 * Returns BPT_OK if nothing was recorded, BPT_ERR_TIMEOUT if a kernel gave up
 * waiting, BPT_ERR_RANGE if an fp16 operand overflowed (*site, if non-NULL,
 * receives the code of the place that recorded it), or BPT_ERR_CUDA if
 * synchronisation failed.
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
  BPT_KIND_CVT = 7,  /* bf16 -> fp16 weight copy */
  BPT_KIND_TAIL = 8, /* fused schedule: W_O, LN2, W_1, W_2 in one kernel */
  BPT_KIND_COUNT = 9
};
bpt_status bpt_profile_enable(int enable);
bpt_status bpt_profile_read(double* ms, int64_t* launches, int n);

/* Kernel launches one bpt_layer_forward call makes for these sizes (_opt:
 * with those options). */
bpt_status bpt_layer_launch_count(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                  int causal, bpt_dtype dtype, int64_t* launches);

/*
 * bpt_layer_tail_plan -- the work list of the fused schedule's layer body
 * (y = x + o W_O, LN2, the FFN, per two-block item; "Blockwise Parallel
 * Transformer — BPT", section "The fused blockwise algorithm") for a bf16
 * layer of these sizes, when `resident_pairs` CTA pairs (1 ..
 * BPT_TAIL_MAX_PAIRS; 74 on a B200) can run at once.  Pure host arithmetic,
 * computed by the code the kernel runs.
 *
 * Items are two consecutive query blocks (items = ceil(B*nb / 2), nb =
 * ceil(N / 128)), on P = min(resident_pairs, items) pairs (*pairs = P): pair
 * q takes whole items q, q + P, ...  When R whole rounds leave L = items - R*P
 * items with 0 < L <= P / 2, d % 1024 == 0 and d_ff % 512 == 0, those are
 * shared: pair q and pair q + L (q < L) each compute half of item R*P + q by
 * columns (*shared = L; otherwise 0).  A launch that cannot be cooperative,
 * or that is recorded by stream capture, runs unshared.
 * plan: for pairs q < min(P, plan_rows), five int32 per pair: whole items,
 * whole items before the shared one (equal), the shared item or -1, this
 * pair's half of it (0 / 1) or -1, the partner pair or -1.  NULL with
 * plan_rows = 0 asks for *pairs and *shared only.
 * Returns BPT_ERR_INVALID_ARG for NULL pairs / shared, resident_pairs out of
 * range, plan_rows < 0 or plan == NULL with plan_rows > 0, and the statuses of
 * bpt_layer_workspace_size for the sizes (as a bf16 layer).
 */
bpt_status bpt_layer_tail_plan(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                               int causal, int32_t resident_pairs, int32_t* pairs,
                               int32_t* shared, int32_t* plan, int32_t plan_rows);
bpt_status bpt_layer_launch_count_opt(int64_t B, int64_t N, int64_t d, int64_t h, int64_t d_ff,
                                      int causal, bpt_dtype dtype, const bpt_options* opts,
                                      int64_t* launches);

/*
 * bpt_layer_forward_static -- bpt_layer_forward for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a deployment
 * convenience of this library, not part of the method.
 *
 * Some callers are not allowed to allocate device memory: plug-ins and
 * extensions whose host framework owns all device memory and hands out only
 * the tensors of a call, embedded or real-time deployments that reserve
 * memory once at start-up and forbid later allocation, and latency-critical
 * loops that cannot pay for an allocation (it may synchronise the device).
 * This entry point takes the same arguments as bpt_layer_forward minus the
 * workspace and uses instead a workspace of BPT_STATIC_WORKSPACE_BYTES that
 * lives in a file-scope __device__ array of the library.  The caller still
 * provides x, the parameters and out.  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *
 *   - Size limit: layers whose bpt_layer_workspace_size exceeds
 *     BPT_STATIC_WORKSPACE_BYTES are rejected with BPT_ERR_WORKSPACE before
 *     anything is enqueued (for example B=1, N=2048, d=768, d_ff=3072 fits;
 *     the larger long-context layers do not and need bpt_layer_forward).
 *   - Memory: every GPU that loads the library holds the array until the
 *     process exits, whether or not this entry point is used.
 *   - First call on a device: it looks up the array's device address (once
 *     per device and CUDA context, with that device current).  Make that
 *     first call before any stream capture begins.
 *   - Sharing: all calls on a device use the same array, and it keeps the
 *     last call's contents (each call clears the header it needs).  Calls
 *     whose work overlaps on the GPU (different streams, no ordering) race on
 *     the array and give undefined results: order them on one stream or with
 *     events.
 *   - Profiling: returns BPT_ERR_INVALID_ARG while bpt_profile_enable is on
 *     (profiling creates event objects).
 *   - Device errors (a wait that ran out, BPT_ERR_TIMEOUT; an fp16 operand
 *     beyond +-65504, BPT_ERR_RANGE, which large bf16 inputs or weights can
 *     cause) are recorded in the array's header: read them with
 *     bpt_read_device_error(NULL, stream, &site).  `out` is undefined after
 *     either.
 * The result is bitwise that of bpt_layer_forward with default options.
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
