/*
 * nanochat_b200.h -- C ABI of one training step (forward + backward) of the
 * nanochat depth-parameterised GPT decoder on an NVIDIA B200 (sm_100a).
 *
 * The model is the one the nanochat pages describe:
 *   - one dial: width C = depth*64 (snapped up to a multiple of 128), C/128
 *     query heads of dim 128, depth blocks ("Nanochat: full-stack LLM training
 *     in 8,000 lines for $72", section "One dial controls everything"; "nanochat
 *     - full-stack ChatGPT in ~8k lines", section "2. Pretrain");
 *   - parameterless RMSNorm after the embedding, before attention, before the
 *     MLP and before the head; RoPE with theta 10,000; QK-norm after RoPE;
 *     causal softmax attention; relu^2 MLP at 4x width; logit softcap
 *     15*tanh(z/15) in fp32; untied embedding / unembedding (first page,
 *     section "A Llama-class transformer with ten modern departures");
 *   - one key/value head shared by all query heads (energyai.berlin page,
 *     section "Multi-Query Attention (MQA)");
 *   - the loss is the mean over all B*T positions of the token cross-entropy.
 *
 * Conventions
 *   - All pointers named "device" are CUDA device pointers on the current
 *     device; the caller owns every buffer passed in (weights, tokens,
 *     targets, workspace, loss, gradients, logits).  The library owns only its
 *     handle, a RoPE cos/sin table and a small device status word.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every compute call only enqueues work on that stream: it never
 *     synchronises the host and never allocates device memory.
 *   - Weight layout: one flat buffer in the model dtype (fp32 or bf16), each
 *     matrix [out, in] row-major (y = x W^T), in this order:
 *       wte[V,C]; per layer l: wq[C,C], wk[128,C], wv[128,C], wo[C,C],
 *       w1[4C,C], w2[C,4C]; lm_head[V,C].
 *     nc_param_layout() returns each tensor's name, element offset and shape.
 *   - Gradients are fp32 in the same layout and are overwritten by each call.
 *   - Errors: every function returns an nc_status.  Argument errors are
 *     detected on the host before anything is enqueued.  Problems that only
 *     the device can see (a token id outside [0, vocab), a non-finite loss, a
 *     kernel wait that ran out of time) set the device status word, which
 *     nc_sync_status() reads and clears.
 */
#ifndef NANOCHAT_B200_H
#define NANOCHAT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NC_OK = 0,
  NC_EINVAL = 1,        /* null pointer, depth < 1, vocab < 2, seq < 1, bad index */
  NC_ESHAPE = 2,        /* B < 1, T < 1 or T > seq */
  NC_ENOMEM = 3,        /* workspace smaller than nc_workspace_bytes() */
  NC_EUNSUPPORTED = 4,  /* current device is not sm_100, or unknown dtype */
  NC_ECUDA = 5,         /* a CUDA runtime call failed (launch, memcpy, event) */
  NC_ERANGE = 6,        /* device: a token or target id outside [0, vocab) */
  NC_ENONFINITE = 7,    /* device: the loss came out NaN or infinite */
  NC_ETIMEOUT = 8,      /* nc_sync_status ran out of time, or a kernel wait expired */
  NC_EALIGN = 9         /* a device pointer is not 16-byte aligned */
} nc_status;

/* Compute dtype, mirroring the pages' single COMPUTE_DTYPE switch
 * (aimarketly.com copy of the nanochat README, "Precision / dtype"):
 * NC_F32 stores and computes everything in fp32; NC_BF16 stores weights,
 * activations and logits in bf16 and accumulates every reduction in fp32. */
typedef enum { NC_F32 = 0, NC_BF16 = 1 } nc_dtype;

typedef struct nc_model nc_model;

typedef struct {
  int depth;      /* number of blocks L */
  int width;      /* C */
  int n_head;     /* query heads H = C / 128 */
  int head_dim;   /* 128 */
  int hidden;     /* MLP hidden width F = 4C */
  int vocab;      /* V */
  int seq;        /* longest T accepted */
  int dtype;      /* nc_dtype */
  int64_t n_params;
} nc_dims;

typedef struct {
  char name[24];    /* "wte", "h<l>.wq", ..., "lm_head", then the full block's extras */
  int64_t offset;   /* element offset in the flat weight / gradient buffer */
  int rows, cols;
} nc_param;

/* Create a model handle for the current CUDA device.  depth >= 1 sets every
 * shape (one dial); vocab >= 2; seq >= 1 is the longest sequence T accepted.
 * Builds the RoPE table (theta 10,000) for positions [0, seq) on the host in
 * float64, rounds it to fp32 once and uploads it.  Returns NC_EUNSUPPORTED on
 * a device that is not compute capability 10.x.  *out receives the handle. */
int nc_init(int depth, int vocab, int seq, int dtype, nc_model **out);

/* Shapes of the model. */
int nc_get_dims(const nc_model *m, nc_dims *out);

/* The full reference block's departures from the baseline decoder, all off
 * by default ("Nanochat: full-stack LLM training in 8,000 lines for $72",
 * section "A Llama-class transformer with ten modern departures";
 * "nanochat - full-stack ChatGPT in ~8k lines", section "0. The model"):
 *   window         > 0: sliding-window attention on the schedule "SSSL" --
 *                  layer l is "SSSL"[l % 4] and the last layer is "L"; an "S"
 *                  layer lets query i see keys j with 0 <= i - j < window
 *                  (the pages: 1,024), an "L" layer the plain causal context
 *   value_embeds   != 0: a gated value-embedding table [vocab, 128] on
 *                  layers 0, 2, 4, ...: v += g_l * ve_l[token] before
 *                  attention, g_l one learnable scalar per such layer (the
 *                  pages name the gate without its form: this scalar is a
 *                  reading)
 *   resid_scalars  != 0: at every block entry the stream becomes
 *                  resid_lambdas[l] * x + x0_lambdas[l] * x0, x0 the
 *                  normalised embedding (the pages' initial values: 1.0, 0.1)
 * The extra tensors follow lm_head in the layout, in this order: ve<l> for
 * each value-embedding layer, resid_lambdas [1, L], x0_lambdas [1, L],
 * ve_gates [1, number of value-embedding layers]. */
typedef struct {
  int window;
  int value_embeds;
  int resid_scalars;
} nc_block_opts;

/* nc_init with the full reference block's options (opts == NULL: none,
 * the same model as nc_init).  window < 0 is NC_EINVAL. */
int nc_init_ex(int depth, int vocab, int seq, int dtype, const nc_block_opts *opts, nc_model **out);

/* Keys a query of layer `layer` sees: the window of an "S" layer, or 0 for
 * the plain causal mask. */
int nc_layer_window(const nc_model *m, int layer, int *window);

/* Number of weight tensors: 2 + 6*depth, plus the full block's extras. */
int nc_param_count(const nc_model *m, int *count);

/* Name, offset and shape of weight tensor `index`, 0 <= index <
 * nc_param_count(), in storage order. */
int nc_param_layout(const nc_model *m, int index, nc_param *out);

/* Bytes of device workspace that nc_fwd_bwd / nc_fwd need for B rows of T
 * tokens.  The workspace holds every saved activation and scratch tensor. */
int nc_workspace_bytes(const nc_model *m, int B, int T, size_t *out);

/* One training step: loss and the gradient of the loss with respect to every
 * weight.
 *   weights    device, n_params elements of the model dtype, layout above
 *   tokens     device int32 [B,T], ids in [0, vocab)
 *   targets    device int32 [B,T], ids in [0, vocab)
 *   workspace  device, ws_bytes >= nc_workspace_bytes(B, T), 256-byte aligned
 *   loss       device fp32 [1]: mean over B*T positions of
 *              logsumexp(s_i) - s_i[target_i], s = 15 tanh(z/15)
 *   token_loss device fp32 [B,T] per-position losses, or NULL
 *   grads      device fp32 [n_params], overwritten
 * Out-of-range ids are clamped for addressing and flagged NC_ERANGE. */
int nc_fwd_bwd(nc_model *m, const void *weights, const int32_t *tokens,
               const int32_t *targets, int B, int T, void *workspace,
               size_t ws_bytes, float *loss, float *token_loss, float *grads,
               void *stream);

/* Flags of nc_fwd_bwd_ex. */
#define NC_ACCUMULATE 1  /* add this step's gradients to grads instead of writing over them */

/* nc_fwd_bwd with flags: NC_ACCUMULATE sums the gradients of several calls
 * into one buffer (gradient accumulation over micro-batches: scale the sum
 * yourself, each call's loss being the mean over its own B*T positions).
 * Unknown flag bits are NC_EINVAL. */
int nc_fwd_bwd_ex(nc_model *m, const void *weights, const int32_t *tokens,
                  const int32_t *targets, int B, int T, void *workspace,
                  size_t ws_bytes, float *loss, float *token_loss, float *grads,
                  int flags, void *stream);

/* Gradient buckets, for overlapping a reduction of the gradients (the
 * data-parallel all-reduce, "Nanochat: full-stack LLM training in 8,000
 * lines for $72", section "A Llama-class transformer with ten modern
 * departures": DistMuonAdamW / ZeRO-2 over 8 GPUs) with the rest of the
 * backward.  Bucket k is the contiguous range [offset, offset + count) of
 * grads, numbered in the order the backward finishes them: 0 lm_head, then
 * one bucket per block from the last block to the first (its six matrices),
 * then wte, then (full block) the extras after lm_head in the layout. */
int nc_grad_bucket_count(const nc_model *m, int *count);
int nc_grad_bucket(const nc_model *m, int k, int64_t *offset, int64_t *count);

/* Events (cudaEvent_t as void*, owned by the caller, n <= the bucket count,
 * NULL entries skipped) that every later nc_fwd_bwd(_ex) records on its
 * stream as soon as bucket k is final; another stream can wait on event k
 * and reduce bucket k while the backward goes on.  n = 0 turns them off. */
int nc_set_grad_events(nc_model *m, void *const *events, int n);

/* Forward only: softcapped logits s = 15 tanh(z/15) of every position.
 *   logits  device [B,T,vocab] in the model dtype (row-major, vocab fastest),
 *           16-byte aligned; a bf16 model needs vocab % 8 == 0 here (its
 *           rows are stored by TMA), else NC_EALIGN
 * Other arguments as nc_fwd_bwd. */
int nc_fwd(nc_model *m, const void *weights, const int32_t *tokens, int B,
           int T, void *workspace, size_t ws_bytes, void *logits, void *stream);

/* Inference with a KV cache ("nanochat - full-stack ChatGPT in ~8k lines",
 * section "6. Inference": a KV cache with int32 per-row sequence lengths;
 * energyai.berlin page, "KV caching").  With one shared KV head the cache
 * holds, per layer, K then V of every position seen, each [B, T_max, 128] in
 * the model dtype: nc_kv_cache_bytes() bytes of caller-owned device memory
 * (16-byte aligned).  seqlens: device int32 [B], the number of cached
 * positions of each row, owned by the caller and kept up to date by the
 * calls below.  T_max <= seq and T_max <= 32,768 (the decode kernel keeps one
 * score per cached key in shared memory), else NC_ESHAPE. */
int nc_kv_cache_bytes(const nc_model *m, int B, int T_max, size_t *out);

/* Runs the forward pass over tokens [B, T] (positions 0..T-1), writes every
 * layer's K and V into the cache, sets seqlens[b] = T and returns the
 * softcapped logits of each row's last position: logits device [B, vocab]
 * (model dtype; bf16 needs vocab % 8 == 0).  workspace as nc_fwd_bwd for
 * (B, T); T <= T_max. */
int nc_prefill(nc_model *m, const void *weights, const int32_t *tokens, int B, int T, void *cache,
               int T_max, int32_t *seqlens, void *workspace, size_t ws_bytes, void *logits,
               void *stream);

/* One decode step: token b (device int32 [B]) sits at position seqlens[b]
 * of its row; it attends to the cached positions 0..seqlens[b] (itself
 * included; the "S" layers of the full block to their last `window`),
 * its K and V are appended, seqlens[b] is incremented, and the softcapped
 * logits of the new token are written to logits [B, vocab].  workspace as
 * nc_fwd_bwd for (B, 1).  A position past T_max - 1 is clamped and reported
 * as NC_ERANGE by nc_sync_status. */
int nc_decode(nc_model *m, const void *weights, const int32_t *tokens, int B, void *cache, int T_max,
              int32_t *seqlens, void *workspace, size_t ws_bytes, void *logits, void *stream);

/* The optimizer step ("Nanochat: full-stack LLM training in 8,000 lines for
 * $72", section "A Llama-class transformer with ten modern departures": Muon
 * for the transformer's matrices, AdamW for the embeddings and scalars;
 * "nanochat - full-stack ChatGPT in ~8k lines", section "2. Pretrain").
 * Groups by tensor: "matrix" = wq, wk, wv, wo, w1, w2 of every block (Muon,
 * each matrix on its own); "embed" = wte and the value-embedding tables,
 * "head" = lm_head, "scalar" = resid_lambdas, x0_lambdas, ve_gates (AdamW).
 *   Muon:  buf = mu buf + g;  X = buf / |buf|_F;  ns_steps times
 *          X = 1.5 X - 0.5 X X^T X (cubic Newton-Schulz towards the polar
 *          factor of buf; the pages' "Polar Express" coefficients are not on
 *          them);  w -= lr_matrix (X + weight_decay w)
 *   AdamW: m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;
 *          w -= lr (m / (1-b1^t)) / (sqrt(v / (1-b2^t)) + eps) + lr weight_decay w
 * The learning-rate and momentum schedules (warm-up, warm-down; Muon's
 * momentum 0.85 -> 0.97 -> 0.90) are the caller's: pass each step's values. */
typedef struct {
  float lr_matrix, lr_embed, lr_head, lr_scalar;
  float weight_decay;   /* decoupled, every group */
  float muon_momentum;
  int ns_steps;         /* Newton-Schulz steps, 0..100 */
  float beta1, beta2, eps;
} nc_optim_opts;

/* State: fp32, 3 * n_params: the master copy of the weights, m (AdamW's first
 * moment or Muon's momentum) and v, each in the weight layout.  16-byte
 * aligned caller-owned device memory. */
int nc_optim_state_bytes(const nc_model *m, size_t *out);

/* Device scratch of nc_optim_step (256-byte aligned). */
int nc_optim_workspace_bytes(const nc_model *m, size_t *out);

/* master = weights (widened to fp32), m = v = 0. */
int nc_optim_init(nc_model *m, const void *weights, void *state, void *stream);

/* One step t >= 1 with gradients grads (fp32, weight layout): updates the
 * master copy, the moments, and weights (model dtype, rounded from the
 * master copy).  NC_EINVAL for t < 1, betas outside [0, 1), eps < 0 or
 * ns_steps outside 0..100; NC_ENOMEM for a short workspace. */
int nc_optim_step(nc_model *m, void *weights, const float *grads, void *state, int step,
                  const nc_optim_opts *opts, void *workspace, size_t ws_bytes, void *stream);

/* Wait at most timeout_ms for the work enqueued so far on `stream` to finish
 * (polling, never blocking longer), then read and clear the device status
 * word.  Returns NC_ETIMEOUT if the stream is still busy, else the first
 * device-side error recorded (NC_ERANGE, NC_ENONFINITE, NC_ETIMEOUT) or NC_OK. */
int nc_sync_status(nc_model *m, void *stream, int timeout_ms);

/* Per-kernel accounting of the work enqueued through one handle, for
 * measurement.  Launch counts and algorithmic work (flops: 2 per multiply-add
 * of the mathematical definition, causal attention counted over j <= i only;
 * bytes: the tensors a kernel must read and write once) are always summed.
 * With profiling on, every launch is also bracketed by two CUDA events on
 * the caller's stream and the device time between them is summed. */
typedef struct {
  char name[24];      /* kernel class: "gemm_tc", "gemm_simt", "attn_fwd", ... */
  int64_t launches;
  double ms;          /* summed device time; 0 unless profiling was on */
  double flops;
  double bytes;
} nc_kernel_stat;

/* Turn event timing of every launch on (enable != 0) or off. */
int nc_profile(nc_model *m, int enable);

/* Wait for the recorded events, write up to `max` per-class sums into `out`
 * (classes with no launch are skipped), set *count, and reset the sums. */
int nc_profile_read(nc_model *m, nc_kernel_stat *out, int max, int *count);

/* Static string for a status code. */
const char *nc_strerror(int code);

/* Free the handle and the memory it owns.  The caller must make sure no work
 * that uses it is still running. */
void nc_destroy(nc_model *m);

#ifdef __cplusplus
}
#endif

#endif /* NANOCHAT_B200_H */
