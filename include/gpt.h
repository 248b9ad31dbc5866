/*
 * gpt.h -- C ABI of libgpt_b200.so: one training step of a modernised
 * GPT-2-style decoder with hashed bigram tables, on one B200 (sm_100a).
 *
 * What the step computes (each call below names its source passage):
 *   - forward: token embedding + parameter-free RMSNorm, optional x0 bigram
 *     table, per layer pre-norm attention (RoPE, QK-norm, causal softmax,
 *     optional value bigram table) and a ReLU^2 MLP, final RMSNorm, LM head
 *     (tied or untied, optional logit soft-cap), mean cross-entropy
 *     ("$1000 tier nanochat run", karpathy/nanochat discussion #8, pasted GPT
 *     module `GPT.forward`, `Block.forward`, `CausalSelfAttention.forward`;
 *     modded-nanogpt README, "rotary embeddings, RMSNorm, ReLU^2");
 *   - a hand-written backward (decoder-rtx posts, "speedrun the backward
 *     pass"), with the bigram tables' sparse per-row-magnitude optimizer
 *     applied inside backward so that no table gradient buffer exists
 *     (decoder-rtx posts: "Dropped .grad buffers from the hash tables and
 *     inlined the optimizer in their backward math"; "sparse, no first
 *     moment, and only per-row magnitude");
 *   - AdamW on the dense weights every `grad_accum` backward calls
 *     (nanochat `setup_optimizers`: betas (0.8, 0.95), eps 1e-10).
 *
 * Conventions shared by every entry point:
 *   - Memory: the caller allocates all device memory.  A model lives in one
 *     caller-owned device arena of gpt_workspace_bytes() bytes, which the
 *     library carves and never frees; the library itself calls no cudaMalloc.
 *     Host-side handles are owned by the library and freed by gpt_destroy().
 *   - Streams: every call enqueues work on the model's CUDA stream (or the
 *     stream argument) and returns without synchronising, unless noted.
 *   - Errors: every function returns an int status, GPT_OK (0) on success.
 *     Argument and configuration errors are detected on the host before any
 *     work is enqueued.  Faults found by kernels (token id out of range,
 *     non-finite loss, a bounded wait that gave up) set a device error word
 *     instead of trapping; it is reported by the next gpt_sync_status() /
 *     ngram_sync_status().  gpt_last_error() gives a thread-local message.
 *   - Layouts: row-major; token ids and targets are int32 [B, T]; a target of
 *     -1 is ignored by the loss.  Linear weights are (out, in): y = x W^T.
 */
#ifndef GPT_B200_H
#define GPT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define GPT_OK             0
#define GPT_ERR_ARG        1  /* null pointer, bad size, unknown name        */
#define GPT_ERR_CONFIG     2  /* unsupported or inconsistent configuration   */
#define GPT_ERR_WORKSPACE  3  /* arena or workspace smaller than required    */
#define GPT_ERR_STATE      4  /* call out of order (backward without forward) */
#define GPT_ERR_INPUT      5  /* token/target/row id out of range (device)   */
#define GPT_ERR_NONFINITE  6  /* loss or gradient norm not finite (device)   */
#define GPT_ERR_CUDA       7  /* a CUDA runtime call failed                  */
#define GPT_ERR_TIMEOUT    8  /* a kernel's bounded wait gave up (device)    */

/* ---- element types --------------------------------------------------- */
#define GPT_DTYPE_F32   0   /* fp32 everywhere, SIMT FFMA, no TF32 (tight parity mode) */
#define GPT_DTYPE_BF16  1   /* bf16 activations and GEMM operands, fp32 accumulate,
                               fp32 master weights and optimizer state            */
#define GPT_DTYPE_I32   2

/* ---- tensor kinds for gpt_tensor() ----------------------------------- */
#define GPT_KIND_PARAM      0  /* master value (fp32 dense; tables in the model dtype) */
#define GPT_KIND_GRAD       1  /* fp32 accumulated dense gradient of the last step     */
#define GPT_KIND_ADAM_M     2  /* fp32 AdamW first moment                               */
#define GPT_KIND_ADAM_V     3  /* fp32 AdamW second moment                              */
#define GPT_KIND_ROW_STATE  4  /* fp32 per-row second moment of a bigram table          */
#define GPT_KIND_PARAM_LP   5  /* bf16 copy read by the GEMMs (bf16 mode only)          */
#define GPT_KIND_ACT        6  /* named activation buffers of the last forward          */

/*
 * Model configuration (plain old data).  Fields the pages do not fix carry
 * this library's reading: norm_eps = 1.1920929e-7 (fp32 machine epsilon,
 * PyTorch's default for F.rms_norm without eps), bigram hash constants
 * p1 = 2654435761, p2 = 2246822519, table beta 0.95 / eps 1e-10.
 * Constraints: d_model == n_head * head_dim, n_kv_head == n_head (or 0),
 * head_dim even; in bf16 mode head_dim == 128, d_model, d_ff, vocab are
 * multiples of 64 and seq_len a multiple of 4; x0_rows / v_rows are 0
 * (table absent) or >= 1.
 */
typedef struct gpt_config {
  int n_layer, d_model, n_head, head_dim, n_kv_head, d_ff, vocab, seq_len, micro_batch;
  int grad_accum;         /* A >= 1 backward calls per AdamW step                */
  int dtype;              /* GPT_DTYPE_F32 or GPT_DTYPE_BF16                      */
  int tie_embeddings;     /* 1: LM head shares the token embedding                */
  int qk_norm;            /* 1: RMSNorm each q/k head after RoPE                  */
  float rope_base;        /* 10000                                                */
  float norm_eps;         /* RMSNorm epsilon                                      */
  float softcap;          /* 0 = off; c > 0: z = c * tanh(z / c)                  */
  float init_std;         /* N(0, init_std) initialisation of every weight        */
  float adam_b1, adam_b2, adam_eps, weight_decay;
  float grad_clip;        /* 0 = off; else global L2 clip of the dense gradient   */
  float lr_mult_embed, lr_mult_head, lr_mult_matrix, lr_mult_table;
  long long x0_rows;      /* rows of the table added to x0 (0 = none)             */
  long long v_rows;       /* rows of the table added to the values (0 = none)     */
  float table_beta, table_eps;
  unsigned long long hash_p1, hash_p2;
  int lm_chunk_rows;      /* rows per LM-head/cross-entropy chunk; 0 = default    */
  /* Optimizer of the block matrices (q, k, v blocks of wqkv, wo, w1, w2):
   * GPT_MATRIX_ADAMW (default) or GPT_MATRIX_MUON -- Muon (modded-nanogpt
   * README, "Proposed optimizer"; nanochat discussion #8, `Muon.step`): each
   * of the matrices (the q, k and v blocks of the fused wqkv separately, as
   * nanochat's c_q / c_k / c_v) takes momentum, a Newton-Schulz
   * orthogonalised update and the step lr * lr_mult_matrix * sqrt(max(1,
   * out / in)); the embedding and the head keep AdamW.  The global clip
   * (grad_clip) is taken over all dense gradients before either optimizer.
   * The Muon momentum lives in the ADAM_M buffer of those matrices.  bf16
   * mode only (the iteration runs on the bf16 tensor cores, as the pages run it). */
  int matrix_optimizer;
  float muon_momentum;    /* 0.95                                                 */
  int muon_ns_steps;      /* Newton-Schulz steps, 5                               */
  int muon_nesterov;      /* 1: Nesterov direction (1 - mu) g + mu m              */
  /* Frozen trigram statistics table (decoder-rtx posts: "a 2M row tri-gram
   * stats table (tallied from dataset, frozen), projected and added to
   * values"): tri_rows rows of tri_width statistics (0 rows = absent).  Row of
   * position t: (x_{t-2} * hash_p1 XOR x_{t-1} * hash_p2 XOR x_t * hash_p3) mod
   * tri_rows over uint64 (the vocabulary size for tokens before the start).
   * Every layer adds vproj * S3[row] to the values, vproj [n_head * head_dim,
   * tri_width] a dense weight (matrix learning rate, AdamW); the table gets no
   * gradient.  It starts at zero: fill it with trigram_tally (gpt_tensor name
   * "h3").  tri_width: a multiple of 64 in bf16 mode, of 4 in fp32 mode. */
  long long tri_rows;
  int tri_width;          /* 64                                                   */
  unsigned long long hash_p3;  /* 3266489917                                      */
} gpt_config;

#define GPT_MATRIX_ADAMW 0
#define GPT_MATRIX_MUON  1

typedef struct gpt_model gpt_model;

/* Fill *cfg with the defaults above (tiny fp32 decoder shape).  Host only. */
int gpt_default_config(gpt_config* cfg);

/* Bytes of device arena gpt_create() needs for cfg.  Host only. */
int gpt_workspace_bytes(const gpt_config* cfg, size_t* bytes);

/*
 * Create a model inside `arena` (device pointer, 256-byte aligned, at least
 * gpt_workspace_bytes() bytes, owned by the caller and kept alive until
 * gpt_destroy).  Weights and tables are initialised on the device to
 * N(0, init_std) from a counter-based generator (Philox-4x32-10) keyed by
 * `seed`; optimizer and row states start at zero.  `cuda_stream` is a
 * cudaStream_t (NULL = legacy default stream).  Enqueues the initialisation
 * and returns; *out receives the host handle.
 */
int gpt_create(const gpt_config* cfg, unsigned long long seed, void* arena,
               size_t arena_bytes, void* cuda_stream, gpt_model** out);

/* Release the host handle (the arena stays the caller's).  Synchronises the stream. */
int gpt_destroy(gpt_model* m);

/* Change the stream later calls enqueue on. */
int gpt_set_stream(gpt_model* m, void* cuda_stream);

/*
 * Forward pass and loss of one micro-batch ("$1000 tier nanochat run",
 * `GPT.forward` with targets).  tokens_dev, targets_dev: device int32
 * [micro_batch, seq_len]; targets may be -1 (ignored).  loss_dev: device
 * float, receives the mean cross-entropy over non-ignored targets (0 when
 * there are none).  Activations for the backward pass are kept in the arena.
 * Out-of-range ids set GPT_ERR_INPUT on the device error word.
 */
int gpt_forward_loss(gpt_model* m, const int32_t* tokens_dev, const int32_t* targets_dev,
                     float* loss_dev);

/*
 * Backward pass of the last forward, scaled by 1/grad_accum (nanochat training
 * loop: loss / gradient_accumulation_steps).  Dense gradients accumulate in
 * fp32 (the first backward of a step overwrites).  Both bigram tables are
 * updated in place from this micro-batch's gradient before the call returns
 * (x0 table from dL/dx0 per position, value table from the sum over layers of
 * dL/dv), with learning rate lr * lr_mult_table (unless the table exchange
 * mode is on: see gpt_set_table_exchange).  On every grad_accum-th call
 * the optional global-norm clip and AdamW (learning rate lr * the group's
 * multiplier) are applied to the dense weights; the gradient buffers keep
 * that step's accumulated gradient until the next step starts.
 * Returns GPT_ERR_STATE when no forward precedes it.
 */
int gpt_backward_step(gpt_model* m, float lr);

/*
 * The two halves of gpt_backward_step, for callers that exchange gradients
 * between them (data-parallel training): gpt_backward() runs the backward pass
 * and the table updates (left to the caller in table exchange mode, see
 * gpt_set_table_exchange) and accumulates the dense gradient without stepping;
 * gpt_optimizer_step() applies the clip and AdamW to whatever gradient has
 * accumulated (at least one gpt_backward since the last step), then starts a
 * new accumulation.  gpt_backward_step(m, lr) equals gpt_backward(m, lr)
 * followed, on every grad_accum-th call, by gpt_optimizer_step(m, lr).
 */
int gpt_backward(gpt_model* m, float lr);

/*
 * Table exchange mode (data-parallel training with replicated bigram tables).
 * With on != 0, gpt_backward / gpt_backward_step no longer apply the sparse
 * table updates; they leave each position's table gradient in the buffers
 * gpt_tensor(..., GPT_KIND_ACT) names "table_grad_x" [B*T, d] and
 * "table_grad_v" [B*T, H*hd] (fp32, the gradient the inline update would
 * have applied), next to the rows "rows_x" / "rows_v".  The caller gathers
 * them from every rank and applies one identical ngram_sparse_update (with
 * lr * lr_mult_table, table_beta, table_eps) to its replica of "hx" / "hv";
 * the buffers stay valid until the next gpt_forward_loss.  Off by default.
 */
int gpt_set_table_exchange(gpt_model* m, int on);
int gpt_optimizer_step(gpt_model* m, float lr);

/*
 * Data parallelism with a sharded optimizer step (the dense weights'
 * reduce-scatter -> sharded AdamW -> all-gather form of ZeRO-style sharding;
 * the caller runs the collectives, see dp.py):
 *   gpt_grad_sumsq writes sum_{i in [lo, hi)} G[i]^2 (the accumulated dense
 *     gradient of the flat buffer, gpt_tensor "*" GRAD) to *out_dev (device
 *     double), summed in a fixed order;
 *   gpt_optimizer_step_range runs the AdamW step of gpt_optimizer_step on the
 *     elements [lo, hi) of the flat buffers only (the group learning rates
 *     by position as usual; the bf16 copy of the range refreshed), after the
 *     caller has put the rank-averaged gradient of that range into G; with
 *     grad_clip > 0 the clip coefficient comes from *grad_sumsq_dev, the
 *     global sum of squares (all ranks' gpt_grad_sumsq over their ranges,
 *     all-reduced).  lo, hi: multiples of 4 within [0, flat size].  Advances
 *     the step counter like gpt_optimizer_step.  Not with Muon (it needs
 *     whole matrices).  Both asynchronous on the model's stream.
 */
int gpt_grad_sumsq(gpt_model* m, long long lo, long long hi, double* out_dev);
int gpt_optimizer_step_range(gpt_model* m, float lr, long long lo, long long hi, const double* grad_sumsq_dev);

/* Dense (matmul + embedding) and table parameter counts.  Host only. */
int gpt_num_params(const gpt_model* m, long long* dense, long long* table);

/* Training FLOPs per token, 6 * matmul params + 12 * L * H * hd * T (nanochat
 * `estimate_flops`, PaLM form; the LM-head matrix counted once).  Host only. */
int gpt_flops_per_token(const gpt_config* cfg, long long* flops, long long* flops_causal);

/*
 * Look up a named tensor inside the arena for export / import.  Names:
 * "wte", "lm_head" (untied only), "h<l>.wqkv" [3*H*hd, d] (rows q|k|v),
 * "h<l>.wo" [d, H*hd], "h<l>.w1" [d_ff, d], "h<l>.w2" [d, d_ff], "hx", "hv";
 * kind GPT_KIND_ACT: "per_token_loss" [B, T] fp32, "rows_x" / "rows_v" [B, T]
 * int32, "grad_norm" (fp32 scalar, set when grad_clip > 0), "table_grad_x" /
 * "table_grad_v" (see gpt_set_table_exchange).  The name "*"
 * with kind PARAM / GRAD / ADAM_M / ADAM_V is the whole flat fp32 dense
 * buffer [n] (each tensor padded to a multiple of 64 elements, pads zero),
 * e.g. for an all-reduce of the gradient between gpt_backward and
 * gpt_optimizer_step.  Writes the device pointer, its element type and up to four dims
 * (unused dims are 1).  Host only, no synchronisation.  After writing
 * PARAM tensors from outside, call gpt_params_changed().
 */
int gpt_tensor(gpt_model* m, const char* name, int kind, void** dev_ptr, int* dtype,
               long long shape[4]);

/* Re-derive the bf16 GEMM copies from the fp32 master weights (enqueued). */
int gpt_params_changed(gpt_model* m);

/*
 * Live timing: while enabled, every kernel (or fixed group of kernels) the
 * model enqueues is bracketed by CUDA events on the model's stream.
 * gpt_profile_read() synchronises, sums elapsed time, launches and the
 * algorithmic FLOPs / bytes per kernel class ("gemm", "attention_fwd",
 * "rmsnorm_fwd", "table_update", "adamw", ...) into out[0..cap), sets *n to
 * the number of classes, and clears the records.  Enabling (on = 1) clears.
 */
typedef struct gpt_prof_entry {
  char name[32];
  long long scopes;    /* bracketed groups */
  long long launches;  /* kernels launched inside them */
  double ms;           /* summed CUDA-event time */
  double flops;        /* algorithmic FLOPs (contractions) */
  double bytes;        /* algorithmic bytes (memory-bound kernels) */
} gpt_prof_entry;
int gpt_profile_enable(gpt_model* m, int on);
int gpt_profile_read(gpt_model* m, gpt_prof_entry* out, int cap, int* n);

/* Number of CUDA kernels this library has launched in this process.  Host only. */
int gpt_launch_count(long long* n);

/* Synchronise the model's stream, read and clear the device error word. */
int gpt_sync_status(gpt_model* m);

/* Message of the last failing call on this host thread ("" if none). */
const char* gpt_last_error(void);

/* ---- standalone bigram-table operations (also used inside the step) ---- */

/*
 * Bigram hash rows (decoder-rtx posts, "bi-gram hash tables"): for each
 * position, a = tokens[b, t-1] (a = vocab at t = 0), c = tokens[b, t],
 * key = (a*p1 mod 2^64) XOR (c*p2 mod 2^64), rows_out[b, t] = key mod rows.
 * tokens / rows_out: device int32 [B, T].  Ids outside [0, vocab) set the
 * device error word (ngram_sync_status) and give row 0.  rows <= 2^31-1.
 */
int ngram_hash(const int32_t* tokens, int B, int T, int vocab, unsigned long long p1,
               unsigned long long p2, long long rows, int32_t* rows_out, void* stream);

/*
 * Row gather: out[i, :] (+)= table[rows[i], :] for i < n (decoder-rtx posts:
 * table rows "added to x0" / "added to values").  table: device [n_rows, d]
 * of `dtype` (GPT_DTYPE_F32 or GPT_DTYPE_BF16); out: device [n, d] of the same
 * dtype, overwritten (accumulate = 0) or added to (accumulate = 1).
 * Rows outside [0, n_rows) set the device error word and leave out[i] as is.
 */
int ngram_gather(const int32_t* rows, int n, const void* table, long long n_rows, int d,
                 int dtype, void* out, int accumulate, void* stream);

/* Device workspace bytes ngram_sparse_update() needs for n positions of width d. */
int ngram_sparse_update_workspace_bytes(int n, int d, size_t* bytes);

/*
 * Sparse per-row-magnitude table update, applied in place (decoder-rtx
 * posts: "sparse, no first moment, and only per-row magnitude", inlined
 * into backward).  For every distinct row r among rows[0..n):
 *   G = sum of grad[i, :] over i with rows[i] == r
 *   s_r = beta * s_r + (1 - beta) * mean_j G[j]^2
 *   table[r, :] -= lr * G / (sqrt(s_r) + eps)
 * Other rows and states are untouched.  Positions are bucketed by row with
 * a stable radix sort (no atomics); G is summed in a fixed order (positions
 * in order within chunks of 16 sorted positions, then the chunks' partial
 * sums in fixed groups), so the result is bit-reproducible.
 * table: device [n_rows, d] of `dtype` (bf16 rows are rounded to nearest
 * even); row_state: device fp32 [n_rows]; grad: device fp32 [n, d].
 * updated_rows_out (nullable): device int32 [n], receives the distinct
 * rows in ascending order; n_updated_out_dev (nullable): device int32, their
 * count.  workspace: device, ws_bytes >= ngram_sparse_update_workspace_bytes.
 */
int ngram_sparse_update(void* table, float* row_state, long long n_rows, int d, int dtype,
                        const int32_t* rows, const float* grad, int n, float lr, float beta,
                        float eps, int32_t* updated_rows_out, int* n_updated_out_dev,
                        void* workspace, size_t ws_bytes, void* stream);

/* Synchronise `stream` and read + clear the standalone operations' device
 * error word (GPT_ERR_INPUT for out-of-range ids, GPT_ERR_TIMEOUT for a bounded
 * wait that gave up).  The standalone calls (ngram_*, muon_update,
 * gptx_gemm_bf16) share ONE such word per device, not one per stream: a status
 * read here may report a fault raised by another stream's standalone call on
 * the same device, and clearing it hides that fault from that stream's caller.
 * Callers that run standalone calls on several streams at once should read the
 * status once all of those streams are synchronised.  A model's own word
 * (gpt_sync_status) is separate. */
int ngram_sync_status(void* stream);

/*
 * ngram_sparse_update without a caller workspace.  Same arguments, result and
 * error reporting as ngram_sparse_update, minus `workspace` / `ws_bytes`: the
 * scratch comes from a 16 MiB buffer compiled into the library, so this call
 * never allocates device memory (no cudaMalloc, no cudaFree, no allocating
 * library routine).  It is meant for callers that have no way to hand over
 * scratch memory: a host runtime that owns every byte of device memory through
 * its own pool and forbids allocations on the side, a plugin that is given
 * tensors but no allocator, or a loop that cannot afford cudaMalloc's implicit
 * synchronisation.  The pages have no counterpart of this entry point.
 *
 * Limit: the scratch of ngram_sparse_update_workspace_bytes(n, d) must fit in
 * 16 MiB (about 16 + d/2 bytes per position: e.g. n <= 32768 positions at
 * d <= 768, or n <= 8192 at d = 2048);
 * larger calls return GPT_ERR_WORKSPACE before any work is enqueued.
 * The call runs on the device that owns `stream` (made current for the call
 * and restored after).  The first call on a device looks up the buffer's
 * device address (with that device current) and should come before any
 * stream capture.  All calls share
 * the one buffer: calls whose execution overlaps on the GPU (different
 * streams, or the same buffer used from two host threads' streams) race on it
 * and must be ordered by the caller.  Every GPU that loads the library keeps
 * the 16 MiB until the process exits.
 */
int ngram_sparse_update_noalloc(void* table, float* row_state, long long n_rows, int d, int dtype,
                                const int32_t* rows, const float* grad, int n, float lr, float beta,
                                float eps, int32_t* updated_rows_out, int* n_updated_out_dev,
                                void* stream);

/* ---- frozen trigram statistics ------------------------------------------ */

/* Device workspace bytes trigram_tally() needs: rows * width * 4 (counts). */
int trigram_tally_workspace_bytes(long long rows, int width, size_t* bytes);

/*
 * Tally the trigram statistics table from token streams (decoder-rtx posts:
 * "tri-gram stats table (tallied from dataset, frozen)"): for every position
 * t < L - 1 of each of the S streams (device int32 [S, L], row-major), the row
 * of (x_{t-2}, x_{t-1}, x_t) -- the key of gpt_config's trigram fields,
 * vocab standing for tokens before the start -- counts its next token in
 * bucket x_{t+1} mod width; then table[r, b] = count[r, b] / (row r's total)
 * in `dtype` (GPT_DTYPE_F32 or GPT_DTYPE_BF16), rows never seen 0.  The table
 * (device [rows, width]) is overwritten; `workspace` holds the counts
 * (trigram_tally_workspace_bytes, 256-byte aligned).  Counts are integers, so
 * the result does not depend on the order of the adds.  Out-of-range token
 * ids set the standalone error word (ngram_sync_status) and are not counted.
 * Asynchronous on `stream`.
 */
int trigram_tally(const int32_t* streams, int S, int L, int vocab, unsigned long long p1, unsigned long long p2,
                  unsigned long long p3, long long rows, int width, int dtype, void* table, void* workspace,
                  size_t ws_bytes, void* stream);

/* ---- FP8 (e4m3) GEMM path ----------------------------------------------- */

/* Device workspace bytes fp8_quantize() needs (a fixed count of partial maxima). */
int fp8_quantize_workspace_bytes(size_t* bytes);

/*
 * Per-tensor e4m3 quantization (Karpathy's llm.c post: FP8 training
 * "imminent"; the pages give no recipe, this is the plainest per-tensor one):
 * amax = max |x|, inv = 448 / amax, q[i] = e4m3(x[i] * inv) rounded to nearest
 * even, saturated to +-448 (1 sign, 4 exponent bits, bias 7, 3 mantissa bits);
 * *scale = amax / 448 (1 when amax is 0), the factor the product applies.
 * x: device [n] of `dtype` (GPT_DTYPE_F32 or GPT_DTYPE_BF16), n even; q:
 * device uint8 [n]; scale: device float.  Asynchronous on `stream`.
 */
int fp8_quantize(const void* x, int dtype, long long n, uint8_t* q, float* scale, void* workspace,
                 size_t ws_bytes, void* stream);

/*
 * C[m, n] = (*scale_a) (*scale_b) sum_k A[m, k] B[n, k] with e4m3 codes A
 * [M, K] and B [N, K] (device, row-major, row pitches lda / ldb bytes,
 * multiples of 16) on the tcgen05 tensor cores (kind::f8f6f4, fp32
 * accumulation; SM pairs when gptx_set_gemm_cta_pairs is on).  out_dtype:
 * GPT_DTYPE_F32 or GPT_DTYPE_BF16 for C (device, row pitch ldc elements, 16-byte
 * aligned).  Asynchronous on `stream`.
 */
int gptx_gemm_fp8(int M, int N, int K, const uint8_t* A, long long lda, const uint8_t* B, long long ldb,
                  const float* scale_a, const float* scale_b, int out_dtype, void* C, long long ldc, void* stream);

/* ---- Muon (matrix-parameter optimizer) --------------------------------- */

/* Device workspace bytes muon_update() needs for a rows x cols matrix
 * (rows, cols: positive multiples of 8). */
int muon_update_workspace_bytes(int rows, int cols, size_t* bytes);

/*
 * One Muon step of a matrix parameter, in place (modded-nanogpt README,
 * "Proposed optimizer"; nanochat discussion #8, `zeropower_via_newtonschulz5`
 * and `Muon.step`):
 *   M <- momentum * M + (1 - momentum) * G
 *   U  = (1 - momentum) * G + momentum * M        (nesterov != 0; else U = M)
 *   X  = U / (||U||_F + 1e-7), then ns_steps times
 *        X <- a X + (b A + c A A) X,  A = X X^T   (a, b, c = 3.4445, -4.7750, 2.0315;
 *        a matrix with more rows than columns runs the same polynomial as
 *        X <- a X + X (b A + c A A) with A = X^T X)
 *   W <- W - lr * sqrt(max(1, out / in)) * X
 * out / in = rows / cols when out_rows != 0 (the weight stored [out, in]),
 * else cols / rows.  The iterate X, A and the polynomial are bf16 operands of
 * the tcgen05 GEMM with fp32 accumulation, as the pages run it in bf16; the
 * momentum and the weight stay fp32.  Sums are formed in a fixed order, so the
 * result is bit-reproducible.
 * W, M, G: device fp32 [rows, cols] row-major, 16-byte aligned; W and M are
 * updated, G is read.  workspace: device, ws_bytes >=
 * muon_update_workspace_bytes(rows, cols).  rows, cols: multiples of 8;
 * 0 <= momentum < 1; 0 <= ns_steps <= 64.  Asynchronous on `stream`; a
 * bounded wait that gives up is reported by ngram_sync_status().
 */
int muon_update(float* W, float* M, const float* G, int rows, int cols, int out_rows, float lr, float momentum,
                int nesterov, int ns_steps, void* workspace, size_t ws_bytes, void* stream);

/* ---- kernel-level test entry point ------------------------------------- */

/*
 * One dense contraction on the tcgen05 tensor-core GEMM that the step uses
 * for every product: acc[m, n] = sum_k A[m, k] B[n, k], bf16 operands, fp32
 * accumulation, then the epilogue `mode`:
 *   0 store      C (bf16) = acc                 3 ReLU^2     C (bf16) = relu(acc)^2
 *   1 store fp32 C (fp32) = acc                 4 ReLU^2 bwd C (bf16) = 2 sqrt(aux) acc
 *   2 accumulate C (fp32) = (beta ? C : 0) + acc   (aux: bf16 relu(a)^2, same ld as C)
 *   5 logits     per (row, 128-column block; 64 when N < 256) the block max m of
 *                acc and s = sum exp(acc - m), written as float pairs (m, s) to
 *                `workspace` ([M, n_blocks]); C (bf16) = exp(acc - m), the
 *                block-local softmax numerators.  With aux given it holds one
 *                int32 target column per row (< 0: none) and acc at that
 *                column goes to the M floats after the pairs in `workspace`
 * A is read K-major (a_kmajor = 1: element [m, k] at A[m*lda + k]) or M-major
 * (a_kmajor = 0: at A[k*lda + m]); B likewise with N.  splits > 1 (modes 1 and
 * 2 only) splits K and needs workspace of splits*M*N*4 bytes, the partials
 * being summed in split order.  Operands, C and aux must be 16-byte aligned
 * with row pitches that are multiples of 16 bytes.  Asynchronous on `stream`.
 */
int gptx_gemm_bf16(int M, int N, int K, const void* A, long long lda, int a_kmajor, const void* B,
                   long long ldb, int b_kmajor, int mode, void* C, long long ldc, const void* aux,
                   int beta, int splits, void* workspace, size_t ws_bytes, void* stream);

/*
 * Tile shape of every later GEMM of this process (the step's and
 * gptx_gemm_bf16's): on != 0 (the default) runs products with N >= 256 on
 * pairs of SMs (tcgen05 cta_group::2, 256 x 256 output tiles, each SM loading
 * half of the tile's B rows); 0 runs them on one SM per 128 x 256 (or 128 x 192)
 * tile.  Both forms compute the same sums in the same order per output
 * element.  The environment variable GPT_GEMM_CTA_PAIR=0 sets the initial
 * value to 0.  A tuning and test switch; not thread-safe against GEMMs being
 * enqueued at the same time.
 */
int gptx_set_gemm_cta_pairs(int on);

/*
 * Check of the bounded-wait path (diagnostic): enqueues on `stream` one
 * thread that waits on a shared-memory mbarrier nothing ever arrives on,
 * exactly as the kernels' bounded waits do, gives up after limit_us
 * microseconds (clamped to [1, 2,000,000]), sets the timeout bit of the
 * standalone error word and returns.  The next ngram_sync_status(stream)
 * reports GPT_ERR_TIMEOUT; the context stays usable.  GPT_ERR_CUDA if the
 * launch fails.
 */
int gptx_wait_probe(int limit_us, void* stream);
#ifdef __cplusplus
}
#endif
#endif /* GPT_B200_H */
