/*
 * nanochat_b200_ops.h -- op-level entry points of libnanochat_b200.so: the
 * dense contractions and the attention of the decoder step, exposed on their
 * own so each kernel can be checked and timed in isolation.  nc_fwd_bwd
 * (nanochat_b200.h) runs the same kernels.
 *
 * Same conventions as nanochat_b200.h: device pointers owned by the caller,
 * work enqueued on `stream` (a cudaStream_t as void*), no host sync, no
 * device allocation, nc_status return codes.
 */
#ifndef NANOCHAT_B200_OPS_H
#define NANOCHAT_B200_OPS_H

#include <stddef.h>
#include <stdint.h>

#include "nanochat_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogues fused into the GEMM (the element-wise steps that follow each
 * projection of the block, "A Llama-class transformer with ten modern
 * departures"):
 *   NC_EPI_STORE      D = acc                (D in dtype)
 *   NC_EPI_STORE_F32  D = acc                (D fp32)
 *   NC_EPI_ADD        D = D + acc            (residual add; D in dtype)
 *   NC_EPI_RELU2      D = relu(acc)^2        (relu^2 MLP activation)
 *   NC_EPI_DRELU2     D = acc * 2 sqrt(D)    (its backward: D holds relu(h)^2)
 *   NC_EPI_SOFTCAP    D = 15 tanh(acc / 15)  (logit softcap)
 *   NC_EPI_ACC_F32    D = D + acc            (D fp32: gradient accumulation) */
enum {
  NC_EPI_STORE = 0,
  NC_EPI_STORE_F32 = 1,
  NC_EPI_ADD = 2,
  NC_EPI_RELU2 = 3,
  NC_EPI_DRELU2 = 4,
  NC_EPI_SOFTCAP = 5,
  NC_EPI_ACC_F32 = 6
};

/* D[m,n] = epilogue(sum_k A(m,k) B(n,k)), fp32 accumulation.
 *   A(m,k) = A[m*lda + k] if a_mn == 0 (K-major) else A[k*lda + m] (MN-major)
 *   B(n,k) = B[n*ldb + k] if b_mn == 0 else B[k*ldb + n]
 *   D[m,n] = D[m*ldd + n]
 * dtype (nc_dtype) is the type of A, B and of D unless NC_EPI_STORE_F32 or
 * NC_EPI_ACC_F32.
 * engine: 0 = the path nc_fwd_bwd takes (bf16: tcgen05 tensor cores, pairs of
 * CTAs on 256 x 256 tiles when M >= 256, one CTA per 128 x 256 tile
 * otherwise; fp32: CUDA cores), 1 = the CUDA-core kernel (a test engine for
 * either dtype), 2 = tcgen05 with one CTA per tile.  The tensor-core engines
 * need 16-byte aligned pointers and strides that are multiples of 8 elements
 * (4 for an fp32 D): anything else returns NC_EALIGN before any work is
 * enqueued -- there is no silent slower path.
 * M, N, K >= 1.  Kernel-side problems (a wait that ran out of time) are
 * reported through nc_ops_status. */
int nc_gemm(const void *A, int64_t lda, int a_mn, const void *B, int64_t ldb, int b_mn, void *D,
            int64_t ldd, int M, int N, int K, int dtype, int epilogue, int engine, void *stream);

/* Causal multi-query attention forward (energyai.berlin page, "Multi-Query
 * Attention (MQA)": one key/value head shared by the H query heads).
 *   qkv     device [B*T, ld] rows [q (H*128) | k (128) | v (128)],
 *           128*(H+2) <= ld <= INT_MAX, else NC_ESHAPE
 *   O       device [B*T, H*128]: O_h = softmax(q_h k^T / sqrt(128) + mask) v
 *   lse     device fp32 [B, H, T]: log-sum-exp of each score row
 *   window  0: the causal mask (key j <= query i); > 0: a sliding window,
 *           0 <= i - j < window ("ten modern departures": the short-window
 *           layers of the SSSL schedule); < 0: NC_EINVAL
 * engine: 0 = the path nc_fwd_bwd takes (bf16: tcgen05 tensor cores, which
 * need 16-byte aligned qkv and O and ld % 8 == 0, else NC_EALIGN; fp32: CUDA
 * cores), 1 = the CUDA-core kernel (a test engine for either dtype), 2 = the
 * other tcgen05 forward kernel (bf16 only; the two differ in how the softmax
 * work is split between warps: one pair of warps per query row on every key
 * tile, or one thread per row with two warpgroups on alternating key tiles),
 * 3 = the model's kernel with one CTA per 128-query tile instead of one
 * persistent CTA per SM.  Engines 2 and 3 with fp32 run the CUDA-core kernel. */
int nc_attention_fwd(const void *qkv, int64_t ld, void *O, float *lse, int B, int T, int H, int window,
                     int dtype, int engine, void *stream);

/* Its backward.  dO [B*T, H*128] and O as above, lse from the forward.
 *   Drow  device fp32 [B, H, T] scratch, receives rowsum(dO * O)
 *   dqkv  device [B*T, ld]: dq per head; dk, dv summed over the query heads
 * window and errors as nc_attention_fwd (dO and dqkv 16-byte aligned too);
 * engine 0 or 1 (else NC_EINVAL). */
int nc_attention_bwd(const void *qkv, int64_t ld, const void *O, const void *dO, const float *lse,
                     float *Drow, void *dqkv, int B, int T, int H, int window, int dtype, int engine,
                     void *stream);

/* Scratch with which nc_attention_bwd_ex cuts the dK/dV work of the key tiles
 * with the most (head, query-tile) pairs into pieces that spread over every
 * SM of the current device: *out = the bytes needed (0 when no tile needs
 * cutting at this shape).  The tcgen05 dK/dV kernel otherwise gives each
 * 128-key tile of each row one CTA, which leaves SMs idle when B * T / 128
 * is small against the SM count or the earliest key tiles (which every later
 * query sees) carry most of the work. */
int nc_attention_bwd_scratch_bytes(int B, int T, int H, int window, size_t *out);

/* nc_attention_bwd with that scratch (device, 16-byte aligned, scratch_bytes
 * long).  With scratch_bytes >= nc_attention_bwd_scratch_bytes each cut key
 * tile's pieces leave fp32 partial sums there that a second kernel adds in
 * piece order: deterministic, and equal to the uncut result up to the order
 * of the fp32 sums.  scratch == NULL or smaller: no cut (nc_attention_bwd).
 * Only the bf16 tcgen05 engine cuts; the scratch is not read afterwards. */
int nc_attention_bwd_ex(const void *qkv, int64_t ld, const void *O, const void *dO, const float *lse,
                        float *Drow, void *scratch, size_t scratch_bytes, void *dqkv, int B, int T, int H,
                        int window, int dtype, int engine, void *stream);

/* Largest B*H*T that nc_attention_bwd_noalloc accepts: the number of fp32
 * entries of its fixed device scratch (4 MiB). */
#define NC_ATTN_BWD_NOALLOC_MAX_ROWS (1 << 20)

/* nc_attention_bwd for callers that cannot allocate device memory: the same
 * computation (causal mask, window 0) and arguments minus Drow and window.  No passage of the nanochat pages
 * corresponds to this entry point; it exists for the library's users.
 *
 * Who needs it: code that must not call cudaMalloc or any allocating routine
 * -- for example a process whose device memory is handed out once at start-up
 * by its own allocator and may not grow, or a latency-sensitive loop that
 * cannot afford the device-wide synchronisation cudaMalloc/cudaFree imply --
 * but still has to run the attention backward, which needs a B*H*T fp32
 * scratch for rowsum(dO * O).
 *
 * What it does instead: the scratch is a file-scope device array of
 * NC_ATTN_BWD_NOALLOC_MAX_ROWS floats inside the library, so every GPU that
 * loads the library holds those 4 MiB until the process exits.  The first
 * call in a CUDA context looks the array's device address up
 * (cudaGetSymbolAddress, with that context current) and caches it under the
 * context's unique id; make that first call before any stream capture.  A
 * context created later (after cudaDeviceReset, say) has a new id and gets a
 * fresh lookup on its first call.  The call itself allocates nothing.
 *
 * Limits and sharing: B*H*T > NC_ATTN_BWD_NOALLOC_MAX_ROWS returns NC_ENOMEM
 * before anything is enqueued.  Every call in a context uses the same array
 * and leaves its contents behind; each call overwrites every entry it reads,
 * so no clearing is needed between calls, but two calls that overlap on the
 * GPU (different streams, or different host threads) race on the array and
 * give wrong results: serialise them.  Kernel-side problems are reported
 * through nc_ops_status, like the other op-level calls. */
int nc_attention_bwd_noalloc(const void *qkv, int64_t ld, const void *O, const void *dO,
                             const float *lse, void *dqkv, int B, int T, int H, int dtype,
                             int engine, void *stream);

/* Logit softcap, log-sum-exp and token cross-entropy, forward and backward
 * in one pass over each row ("Nanochat: full-stack LLM training in 8,000
 * lines for $72", section "A Llama-class transformer with ten modern
 * departures": logits softcapped as 15 tanh(z/15), computed in fp32), in
 * place:
 *   z           device [M, ldz] (dtype), row i holds the V logits z_i;
 *               overwritten by dz_i = (softmax(s_i) - onehot(t_i)) (1 - (s_i/15)^2) g
 *               with s_i = 15 tanh(z_i / 15); entries past V are untouched
 *   targets     device int32 [M], ids in [0, V) (others are clamped and
 *               reported as NC_ERANGE by nc_ops_status)
 *   token_loss  device fp32 [M]: logsumexp(s_i) - s_i[t_i]
 *   grad_scale  g (1/M gives the gradient of the mean loss)
 * tanh and 1 - tanh^2 are formed to fp32 precision for both dtypes.  bf16
 * rows with V % 8 == 0, V <= 65,536, ldz % 8 == 0 and a 16-byte aligned z
 * take the persistent kernel the model step uses; other rows a general
 * kernel.  M, V >= 1, ldz >= V. */
int nc_softcap_ce(void *z, int64_t ldz, const int32_t *targets, float *token_loss, int M, int V,
                  float grad_scale, int dtype, void *stream);

/* Parameterless RMSNorm of M rows of C ("A Llama-class transformer with ten
 * modern departures": RMSNorm without learnable parameters):
 *   r[m] = 1 / sqrt(mean_c x[m,c]^2 + eps),  y[m,c] = x[m,c] r[m],  eps = 2^-23
 * x, y: [M, C] row-major in dtype (y may equal x); r: [M] fp32.  The kernel
 * the model's norms run.  8 <= C <= 4096 with C % 8 == 0 (else NC_ESHAPE);
 * x, y 16-byte aligned and r 4-byte aligned (else NC_EALIGN). */
int nc_rmsnorm(const void *x, void *y, float *r, int M, int C, int dtype, void *stream);

/* Its backward, with the residual-stream gradient it feeds:
 *   g[m,c] = r[m] (dy[m,c] - y[m,c] mean_c(dy[m,:] y[m,:]))
 *   dx = g (accumulate == 0) or dx + g (accumulate != 0), dx fp32 [M, C];
 *   dx_t = the new dx in dtype (the next GEMM's operand).
 * y, r: the outputs of nc_rmsnorm.  Shapes and alignment as nc_rmsnorm (dx,
 * dx_t 16-byte aligned). */
int nc_rmsnorm_bwd(const void *dy, const void *y, const float *r, float *dx, void *dx_t, int M, int C,
                   int accumulate, int dtype, void *stream);

/* RoPE (theta 10,000, dims i and i+64 of each head rotated by the angle
 * pos * 10000^(-i/64), pos = row index mod T) then QK-norm (parameterless
 * RMSNorm over each head's 128 dims), in place on the m->H query heads and the
 * shared key head of the fused rows qkv [B*T, ld] = [q | k | v] ("ten modern
 * departures": rotary embeddings, QK normalisation after them).  rq [B*T, H]
 * and rk [B*T] receive the heads' reciprocal rms.  The model's RoPE tables
 * are used, so T <= the model's seq (else NC_ESHAPE); ld >= 128 (H + 2)
 * elements; qkv 16-byte aligned with 16-byte rows (else NC_EALIGN). */
int nc_rope_qknorm(const nc_model *m, void *qkv, int64_t ld, float *rq, float *rk, int B, int T, void *stream);

/* Backward of nc_rope_qknorm, in place on the q and k parts of dqkv [B*T, ld]
 * (the v part is left as it is): qkv, rq, rk are nc_rope_qknorm's outputs.
 *   g = r (dy - y mean(dy y)) per head, then the rotation by -angle. */
int nc_rope_qknorm_bwd(const nc_model *m, void *dqkv, const void *qkv, int64_t ld, const float *rq,
                       const float *rk, int B, int T, void *stream);

/* Cap on the CTAs of the persistent attention kernels (the forward and the
 * dQ kernel of the backward, in nc_fwd_bwd and the op-level calls): 0 (the
 * default) = one CTA per SM; n > 0 = at most n CTAs, each then taking more
 * 128-query tiles (fewer CTAs leave SMs to other streams, e.g. gradient
 * all-reduces).  Process-wide, for launches that follow; < 0: NC_EINVAL. */
int nc_set_attention_ctas(int ctas);

/* Status of the op-level calls above (nc_gemm, nc_attention_*, and the
 * calls below), which have no model handle: waits at most timeout_ms for the
 * work enqueued so far on `stream` (polling), then reads and clears the
 * library's op status word of the current CUDA context.  Returns
 * NC_ETIMEOUT if the stream is still busy or a kernel wait ran out of time
 * (its output is then not valid), else NC_OK.  The word is one per context,
 * shared by every stream: read it after the calls whose outcome you need. */
int nc_ops_status(void *stream, int timeout_ms);

/* Self-check of the wait-expiry path: enqueues one thread that waits on a
 * barrier nothing completes, gives up after wait_us microseconds
 * (0 <= wait_us <= 1,000,000, else NC_EINVAL) and records a timeout in the op
 * status word, exactly as a kernel whose partner never arrives does.  The
 * next nc_ops_status then returns NC_ETIMEOUT.  No passage of the nanochat
 * pages corresponds to it; it lets a caller check that expired waits reach
 * the host without faulting or hanging the GPU. */
int nc_check_wait_expiry(int wait_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NANOCHAT_B200_OPS_H */
