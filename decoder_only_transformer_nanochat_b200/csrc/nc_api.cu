// C ABI of the nanochat decoder step: argument checks, workspace carving and
// the forward / backward launch sequence on the caller's stream.
//
// Model ("Nanochat: full-stack LLM training in 8,000 lines for $72", sections
// "One dial controls everything" and "A Llama-class transformer with ten
// modern departures"; energyai.berlin page, "Multi-Query Attention"):
//   x = norm(wte[tok])
//   per block l: xn = norm(x); [q|k|v] = xn [Wq;Wk;Wv]^T; q,k = norm(rope(q,k));
//                O = causal attention; x += O Wo^T;
//                xn2 = norm(x); a = relu(xn2 W1^T)^2; x += a W2^T
//   xf = norm(x); z = xf Wout^T; s = 15 tanh(z/15); loss = mean CE(s, target)
#include <limits.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <chrono>
#include <mutex>
#include <thread>
#include <vector>

#include "../../include/nanochat_b200.h"
#include "../../include/nanochat_b200_ops.h"
#include "attn_simt.cuh"
#include "ce.cuh"
#include "elementwise.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "optim.cuh"
#include "token_sort.cuh"

using namespace nc;

// kernel classes of the per-launch accounting
enum KernelClass {
  K_GEMM_TC, K_GEMM_SIMT, K_ATTN_FWD, K_ATTN_BWD, K_EMBED, K_RMSNORM, K_ROPE_QKNORM, K_CE,
  K_LOSS_MEAN, K_RMSNORM_BWD, K_ROWDOT, K_ROPE_QKNORM_BWD, K_EMBED_BWD, K_TOKEN_SORT, K_SEG_FIXUP,
  K_VE_BWD, K_OPTIM, K_NUM_CLASSES
};
static const char *kClassName[K_NUM_CLASSES] = {
    "gemm_tc", "gemm_simt", "attn_fwd", "attn_bwd", "embed_norm", "rmsnorm", "rope_qknorm",
    "ce_fused", "loss_mean", "rmsnorm_bwd", "attn_rowdot", "rope_qknorm_bwd", "embed_bwd",
    "token_sort", "seg_fixup", "block_extras_bwd", "optimizer"};

struct nc_model {
  int depth, C, H, F, V, seq, dtype;
  int64_t n_params;
  // full reference block (nc_init_ex): short window of the "S" layers (0:
  // none), value embeddings, residual scalars
  int window = 0;
  bool ve = false, scalars = false;
  std::vector<int> layer_window;  // per layer: keys a query sees (0: plain causal)
  std::vector<int> ve_param;      // per layer: param index of its value-embedding table, or -1
  std::vector<int> ve_slot;       // per layer: its entry of ve_gates, or -1
  int p_resid = -1, p_x0 = -1, p_gates = -1;
  // gradient buckets in the order the backward completes them, and the
  // caller's events recorded when each one is final (nc_set_grad_events)
  std::vector<std::pair<int64_t, int64_t>> buckets;  // (offset, count) in elements
  std::vector<cudaEvent_t> grad_events;
  int device;
  int num_sms;
  float *rope_cos;  // [seq, 64] fp32
  float *rope_sin;
  int *status;      // device status word
  std::vector<nc_param> params;
  // accounting (see nc_profile)
  bool prof = false;
  std::vector<cudaEvent_t> events;
  size_t events_used = 0;
  std::vector<std::pair<int, size_t>> records;  // (class, index of the start event)
  int64_t launches[K_NUM_CLASSES] = {};
  double flops[K_NUM_CLASSES] = {};
  double bytes[K_NUM_CLASSES] = {};
};

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

template <typename T>
struct Work {
  std::vector<T *> xn, qkv, O, xn2, a;
  std::vector<float *> r1, rq, rk, lse, r2;
  T *x, *xf, *z, *dxb, *dO, *dqkv, *dy;
  float *r0, *rf, *tok_loss, *dx, *Drow;
  float *attn_part = nullptr;  // partial dK/dV sums of key tiles cut into pieces
  size_t attn_part_bytes = 0;
  int64_t ldz;
  TokenSort sort;                   // positions grouped by token (embedding gradient)
  float *seg_head, *seg_tail;       // [chunks, C] partial sums of segments cut by chunks
  int *seg_flags;                   // [chunks]
  // residual scalars: the stream entering each block kept ([0] = x0 =
  // norm(wte[tok])), the gradient reaching x0 through the mixing, and
  // per-block partial sums of the scalars' gradients [2][L][blocks]
  std::vector<T *> xs;
  float *dx0 = nullptr, *scal_part = nullptr;
  float *ve_part = nullptr;         // value-embedding gate gradient partials [blocks of 64 rows]
};

// Lay the workspace out (base == nullptr only measures it).
template <typename T>
size_t carve(const nc_model *m, int B, int T_len, char *base, Work<T> *w) {
  const size_t M = (size_t)B * T_len;
  const int C = m->C, H = m->H, F = m->F, L = m->depth;
  const int64_t ldqkv = C + 2 * kHeadDim;
  const int64_t ldz = ((int64_t)m->V + 63) / 64 * 64;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char * {
    char *p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  const size_t es = sizeof(T);
  if (w) {
    w->xn.resize(L); w->qkv.resize(L); w->O.resize(L); w->xn2.resize(L); w->a.resize(L);
    w->r1.resize(L); w->rq.resize(L); w->rk.resize(L); w->lse.resize(L); w->r2.resize(L);
  }
  for (int l = 0; l < L; ++l) {
    T *xn = (T *)take(M * C * es);
    float *r1 = (float *)take(M * 4);
    T *qkv = (T *)take(M * ldqkv * es);
    float *rq = (float *)take(M * H * 4);
    float *rk = (float *)take(M * 4);
    T *O = (T *)take(M * C * es);
    float *lse = (float *)take(M * H * 4);
    T *xn2 = (T *)take(M * C * es);
    float *r2 = (float *)take(M * 4);
    T *a = (T *)take(M * F * es);
    if (w) {
      w->xn[l] = xn; w->r1[l] = r1; w->qkv[l] = qkv; w->rq[l] = rq; w->rk[l] = rk;
      w->O[l] = O; w->lse[l] = lse; w->xn2[l] = xn2; w->r2[l] = r2; w->a[l] = a;
    }
  }
  T *x = (T *)take(M * C * es);
  float *r0 = (float *)take(M * 4);
  T *xf = (T *)take(M * C * es);
  float *rf = (float *)take(M * 4);
  T *z = (T *)take(M * ldz * es);
  float *tok_loss = (float *)take(M * 4);
  float *dx = (float *)take(M * C * 4);
  T *dxb = (T *)take(M * C * es);
  T *dy = (T *)take(M * C * es);
  T *dO = (T *)take(M * C * es);
  T *dqkv = (T *)take(M * ldqkv * es);
  float *Drow = (float *)take(M * H * 4);
  size_t part_bytes = 0;
  if (sizeof(T) == 2)
    for (int l = 0; l < L; ++l)
      part_bytes = std::max(part_bytes, fatc::dkdv_scratch_bytes(B, T_len, H, m->layer_window[l], m->num_sms));
  float *attn_part = part_bytes ? (float *)take(part_bytes) : nullptr;
  int32_t *sk0 = (int32_t *)take(M * 4), *sk1 = (int32_t *)take(M * 4);
  int32_t *sv0 = (int32_t *)take(M * 4), *sv1 = (int32_t *)take(M * 4);
  int *hist = (int *)take((size_t)256 * sort_tiles((int)M) * 4);
  const size_t nch = (size_t)seg_chunks((int)M);
  float *seg_head = (float *)take(nch * C * 4), *seg_tail = (float *)take(nch * C * 4);
  int *seg_flags = (int *)take(nch * 4);
  std::vector<T *> xs;
  float *dx0 = nullptr, *scal_part = nullptr, *ve_part = nullptr;
  if (m->scalars) {
    for (int l = 1; l <= L; ++l) xs.push_back((T *)take(M * C * es));
    dx0 = (float *)take(M * C * 4);
    scal_part = (float *)take((size_t)2 * L * ((M + 7) / 8) * 4);
  }
  if (m->ve) ve_part = (float *)take(((M + 63) / 64) * 4);
  if (w) {
    w->xs.clear();
    if (m->scalars) {
      w->xs.push_back(x);  // x0: the embedding output is the stream entering block 0
      for (T *p : xs) w->xs.push_back(p);
    }
    w->dx0 = dx0; w->scal_part = scal_part; w->ve_part = ve_part;
    w->sort.keys[0] = sk0; w->sort.keys[1] = sk1; w->sort.vals[0] = sv0; w->sort.vals[1] = sv1;
    w->sort.hist = hist; w->sort.skey = nullptr; w->sort.spos = nullptr;
    w->seg_head = seg_head; w->seg_tail = seg_tail; w->seg_flags = seg_flags;
  }
  if (w) {
    w->x = x; w->r0 = r0; w->xf = xf; w->rf = rf; w->z = z; w->ldz = ldz;
    w->tok_loss = tok_loss; w->dx = dx; w->dxb = dxb; w->dy = dy; w->dO = dO;
    w->dqkv = dqkv; w->Drow = Drow;
    w->attn_part = attn_part; w->attn_part_bytes = part_bytes;
  }
  return off;
}

// Weight pointers of the flat buffer, layout order of nc_param_layout.
template <typename T>
struct Weights {
  const T *wte, *lm_head;
  std::vector<const T *> wqkv, wo, w1, w2;  // wq, wk, wv are contiguous: [C+256, C]
  std::vector<const T *> ve;                // per layer: value-embedding table [V, 128] or null
  const T *resid = nullptr, *x0l = nullptr, *gates = nullptr;  // [L], [L], [n_ve]
};

template <typename T>
Weights<T> weight_ptrs(const nc_model *m, const void *weights) {
  const T *base = (const T *)weights;
  Weights<T> w;
  w.wte = base + m->params[0].offset;
  for (int l = 0; l < m->depth; ++l) {
    w.wqkv.push_back(base + m->params[1 + 6 * l].offset);
    w.wo.push_back(base + m->params[1 + 6 * l + 3].offset);
    w.w1.push_back(base + m->params[1 + 6 * l + 4].offset);
    w.w2.push_back(base + m->params[1 + 6 * l + 5].offset);
    w.ve.push_back(m->ve_param[l] >= 0 ? base + m->params[m->ve_param[l]].offset : nullptr);
  }
  w.lm_head = base + m->params[1 + 6 * m->depth].offset;
  if (m->p_resid >= 0) w.resid = base + m->params[m->p_resid].offset;
  if (m->p_x0 >= 0) w.x0l = base + m->params[m->p_x0].offset;
  if (m->p_gates >= 0) w.gates = base + m->params[m->p_gates].offset;
  return w;
}

#define NC_CHECK_LAUNCH()                              \
  do {                                                 \
    cudaError_t e_ = cudaGetLastError();               \
    if (e_ != cudaSuccess) {                           \
      fprintf(stderr, "nanochat_b200: %s at %s:%d\n",  \
              cudaGetErrorString(e_), __FILE__, __LINE__); \
      return NC_ECUDA;                                 \
    }                                                  \
  } while (0)

// Start event of one launch when profiling is on; -1 otherwise.
long prof_begin(nc_model *m, cudaStream_t st) {
  if (!m->prof) return -1;
  while (m->events.size() < m->events_used + 2) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return -1;
    m->events.push_back(e);
  }
  const size_t i = m->events_used;
  if (cudaEventRecord(m->events[i], st) != cudaSuccess) return -1;
  m->events_used += 2;
  return (long)i;
}

void prof_end(nc_model *m, cudaStream_t st, long ev, int cls, double flops, double bytes) {
  m->launches[cls] += 1;
  m->flops[cls] += flops;
  m->bytes[cls] += bytes;
  if (ev >= 0 && cudaEventRecord(m->events[ev + 1], st) == cudaSuccess)
    m->records.push_back({cls, (size_t)ev});
}

// Launch one kernel with its accounting: class, algorithmic flops and bytes.
#define NC_RUN(cls, fl, by, LAUNCH)                                  \
  do {                                                               \
    const long ev_ = prof_begin(m, st);                              \
    LAUNCH;                                                          \
    NC_CHECK_LAUNCH();                                               \
    prof_end(m, st, ev_, (cls), (double)(fl), (double)(by));         \
  } while (0)

template <typename T>
int gemm(nc_model *m, const GemmProblem &p, cudaStream_t st) {
  if (p.M <= 0 || p.N <= 0) return NC_OK;
  cudaError_t e;
  // bf16 runs on the tensor cores only: operands they cannot take are an
  // error, not a slower path
  const bool tcp = sizeof(T) == 2;
  if (tcp && !tc_gemm_aligned(p)) return NC_EALIGN;
  const long ev = prof_begin(m, st);
  if (tcp) e = launch_gemm_tc(p, m->num_sms, m->status, st);
  else e = launch_gemm_simt<T>(p, st);
  if (e != cudaSuccess) {
    fprintf(stderr, "nanochat_b200: gemm launch: %s\n", cudaGetErrorString(e));
    return NC_ECUDA;
  }
  prof_end(m, st, ev, tcp ? K_GEMM_TC : K_GEMM_SIMT, 2.0 * p.M * (double)p.N * p.K, 0.0);
  return NC_OK;
}

inline GemmProblem gp(int M, int N, int K, const void *A, int64_t lda, int a_mn, const void *B,
                      int64_t ldb, int b_mn, void *D, int64_t ldd, int epi) {
  GemmProblem p;
  p.M = M; p.N = N; p.K = K; p.A = A; p.lda = lda; p.a_mn = a_mn; p.B = B; p.ldb = ldb;
  p.b_mn = b_mn; p.D = D; p.ldd = ldd; p.epi = epi;
  return p;
}

inline unsigned rows_grid(size_t rows, int rows_per_block) {
  return (unsigned)((rows + rows_per_block - 1) / rows_per_block);
}

#define NC_TRY(x)              \
  do {                         \
    int rc_ = (x);             \
    if (rc_ != NC_OK) return rc_; \
  } while (0)

// Keys summed over the queries of one row of T tokens: causal (window 0 or
// >= T) or sliding window.
inline double attn_keys(int T, int window) {
  if (window <= 0 || window >= T) return 0.5 * T * (T + 1.0);
  return 0.5 * window * (window + 1.0) + (double)(T - window) * window;
}

// Inference context of forward_body: the KV cache (per layer K then V, each
// [B, tmax, 128]) that the RoPE kernel fills, and for a decode step the
// per-row positions of the new tokens (attention then reads the cache).
template <typename T>
struct Infer {
  T *cache = nullptr;
  int tmax = 0;
  const int32_t *positions = nullptr;  // decode only
  KvCacheOut<T> layer(int l, int B, int *status) const {
    KvCacheOut<T> o;
    o.kc = cache + (size_t)l * 2 * B * tmax * kHeadDim;
    o.vc = o.kc + (size_t)B * tmax * kHeadDim;
    o.cstride = (int64_t)tmax * kHeadDim;
    o.positions = positions;
    o.tmax = tmax;
    o.status = status;
    return o;
  }
};

// Forward through the blocks and the final norm; leaves xf, rf in the workspace.
template <typename T>
int forward_body(nc_model *m, const Weights<T> &W, const int32_t *tokens, int B, int T_len,
                 Work<T> &w, cudaStream_t st, const Infer<T> *inf = nullptr) {
  const int M = B * T_len, C = m->C, H = m->H, F = m->F;
  const int ldqkv = C + 2 * kHeadDim;
  const double es = sizeof(T);
  NC_RUN(K_EMBED, 0, M * (8.0 + 2.0 * C * es),
         NC_DISPATCH_NV(C, (embed_norm_kernel<T, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                               tokens, W.wte, w.x, w.r0, M, C, m->V, m->status))));
  T *x = w.x;  // the stream the block's residual adds go into
  for (int l = 0; l < m->depth; ++l) {
    const double attn_flops = 4.0 * B * H * (double)kHeadDim * attn_keys(T_len, m->layer_window[l]);
    if (m->scalars) {
      // block entry: x_in = lam_r x + lam_0 x0 into the next stream buffer, xn = norm(x_in)
      x = w.xs[l + 1];
      NC_RUN(K_RMSNORM, 0, M * (4.0 + 4.0 * C * es),
             NC_DISPATCH_NV(C, (mix_rmsnorm_kernel<T, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                                   w.xs[l], w.xs[0], W.resid + l, W.x0l + l, x, w.xn[l], w.r1[l], M, C))));
    } else {
      NC_RUN(K_RMSNORM, 0, M * (4.0 + 2.0 * C * es),
             NC_DISPATCH_NV(C, (rmsnorm_kernel<T, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                                   x, w.xn[l], w.r1[l], M, C))));
    }
    NC_TRY(gemm<T>(m, gp(M, ldqkv, C, w.xn[l], C, 0, W.wqkv[l], C, 0, w.qkv[l], ldqkv, EPI_STORE), st));
    const bool ve = W.ve[l] != nullptr;
    const KvCacheOut<T> kvo = inf ? inf->layer(l, B, m->status) : KvCacheOut<T>();
    NC_RUN(K_ROPE_QKNORM, 0, M * (2.0 * (C + kHeadDim) * es + 4.0 * (H + 1) + (ve ? 3.0 * kHeadDim * es : 0.0)),
           (rope_qknorm_kernel<T><<<rows_grid((size_t)M, 8), 256, 0, st>>>(
               w.qkv[l], ldqkv, w.rq[l], w.rk[l], m->rope_cos, m->rope_sin, M, T_len, H, tokens, W.ve[l],
               ve ? W.gates + m->ve_slot[l] : nullptr, m->V, kvo)));
    if (inf && inf->positions) {
      // decode: the new token's queries against the cached keys of its row
      NC_RUN(K_ATTN_FWD, 0, 0,
             if (launch_attn_decode<T>(w.qkv[l], ldqkv, kvo.kc, kvo.vc, kvo.cstride, inf->positions, inf->tmax, B, H,
                                       m->layer_window[l], w.O[l], st) != cudaSuccess) return NC_ECUDA);
    } else {
      NC_RUN(K_ATTN_FWD, attn_flops, 0,
             if (launch_attn_fwd<T>(w.qkv[l], ldqkv, w.O[l], w.lse[l], B, T_len, H, m->layer_window[l], 0,
                                    m->status, st, m->num_sms) != cudaSuccess) return NC_ECUDA);
    }
    NC_TRY(gemm<T>(m, gp(M, C, C, w.O[l], C, 0, W.wo[l], C, 0, x, C, EPI_ADD), st));
    NC_RUN(K_RMSNORM, 0, M * (4.0 + 2.0 * C * es),
           NC_DISPATCH_NV(C, (rmsnorm_kernel<T, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                                 x, w.xn2[l], w.r2[l], M, C))));
    NC_TRY(gemm<T>(m, gp(M, F, C, w.xn2[l], C, 0, W.w1[l], C, 0, w.a[l], F, EPI_RELU2), st));
    NC_TRY(gemm<T>(m, gp(M, C, F, w.a[l], F, 0, W.w2[l], F, 0, x, C, EPI_ADD), st));
  }
  NC_RUN(K_RMSNORM, 0, M * (4.0 + 2.0 * C * es),
         NC_DISPATCH_NV(C, (rmsnorm_kernel<T, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                               x, w.xf, w.rf, M, C))));
  return NC_OK;
}

// Record the caller's event of gradient bucket k (if set) on the step's stream.
inline int bucket_done(nc_model *m, int k, cudaStream_t st) {
  if (k < (int)m->grad_events.size() && m->grad_events[k] &&
      cudaEventRecord(m->grad_events[k], st) != cudaSuccess)
    return NC_ECUDA;
  return NC_OK;
}

template <typename T>
int fwd_bwd_impl(nc_model *m, const void *weights, const int32_t *tokens, const int32_t *targets,
                 int B, int T_len, void *workspace, float *loss, float *token_loss, float *grads,
                 int flags, cudaStream_t st) {
  // accumulate: every gradient is added to grads instead of written over it
  const int acc = (flags & NC_ACCUMULATE) ? 1 : 0;
  const int wg = acc ? EPI_ACC_F32 : EPI_STORE_F32;
  Work<T> w;
  carve<T>(m, B, T_len, (char *)workspace, &w);
  const Weights<T> W = weight_ptrs<T>(m, weights);
  const int M = B * T_len, C = m->C, H = m->H, F = m->F, V = m->V;
  const int ldqkv = C + 2 * kHeadDim;
  const double es = sizeof(T);
  NC_TRY(forward_body<T>(m, W, tokens, B, T_len, w, st));

  // head: z = xf Wout^T, then softcap + CE forward and backward in place
  NC_TRY(gemm<T>(m, gp(M, V, C, w.xf, C, 0, W.lm_head, C, 0, w.z, w.ldz, EPI_STORE), st));
  float *tl = token_loss ? token_loss : w.tok_loss;
  const float inv_M = 1.f / (float)M;
  NC_RUN(K_CE, 0, M * (2.0 * V * es + 8.0),
         if (launch_ce<T>(w.z, w.ldz, targets, tl, M, V, inv_M, m->num_sms, m->status, st) != cudaSuccess)
             return NC_ECUDA);
  NC_RUN(K_LOSS_MEAN, 0, M * 4.0, (loss_mean_kernel<<<1, 1024, 0, st>>>(tl, M, loss, m->status)));

  // gradient pointers (fp32, same layout as the weights)
  auto G = [&](int idx) { return grads + m->params[idx].offset; };
  const int last = 1 + 6 * m->depth;  // lm_head
  const double nbwd = M * (8.0 * C + 3.0 * C * es + 4.0);  // dx_old, dx in fp32; dy, y, dx_t in T
  // dWout = dz^T xf ;  dxf = dz Wout
  NC_TRY(gemm<T>(m, gp(V, C, M, w.z, w.ldz, 1, w.xf, C, 1, G(last), C, wg), st));
  NC_TRY(bucket_done(m, 0, st));
  NC_TRY(gemm<T>(m, gp(M, C, V, w.z, w.ldz, 0, W.lm_head, C, 1, w.dy, C, EPI_STORE), st));
  NC_RUN(K_RMSNORM_BWD, 0, nbwd - M * 4.0 * C,
         NC_DISPATCH_NV(C, (rmsnorm_bwd_kernel<T, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                               w.dy, w.xf, w.rf, w.dx, w.dxb, M, C, 0))));

  // positions grouped by token: the embedding's and the value embeddings'
  // table gradients are summed per token in this fixed order
  NC_RUN(K_TOKEN_SORT, 0, M * 16.0 * sort_passes(V), sort_tokens(tokens, M, V, w.sort, st));
  m->launches[K_TOKEN_SORT] += 3 * sort_passes(V) - 1;  // one accounting entry, three launches per pass
  const int nch = seg_chunks(M);
  const unsigned nblk8 = rows_grid(M, 8);

  for (int l = m->depth - 1; l >= 0; --l) {
    const int pi = 1 + 6 * l;
    const double attn_bwd_flops = 8.0 * B * H * (double)kHeadDim * attn_keys(T_len, m->layer_window[l]);
    // MLP: x += a W2^T, a = relu(h)^2, h = xn2 W1^T
    NC_TRY(gemm<T>(m, gp(C, F, M, w.dxb, C, 1, w.a[l], F, 1, G(pi + 5), F, wg), st));
    NC_TRY(gemm<T>(m, gp(M, F, C, w.dxb, C, 0, W.w2[l], F, 1, w.a[l], F, EPI_DRELU2), st));
    NC_TRY(gemm<T>(m, gp(F, C, M, w.a[l], F, 1, w.xn2[l], C, 1, G(pi + 4), C, wg), st));
    NC_TRY(gemm<T>(m, gp(M, C, F, w.a[l], F, 0, W.w1[l], C, 1, w.dy, C, EPI_STORE), st));
    NC_RUN(K_RMSNORM_BWD, 0, nbwd,
           NC_DISPATCH_NV(C, (rmsnorm_bwd_kernel<T, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                                 w.dy, w.xn2[l], w.r2[l], w.dx, w.dxb, M, C, 1))));
    // attention: x += O Wo^T
    NC_TRY(gemm<T>(m, gp(C, C, M, w.dxb, C, 1, w.O[l], C, 1, G(pi + 3), C, wg), st));
    NC_TRY(gemm<T>(m, gp(M, C, C, w.dxb, C, 0, W.wo[l], C, 1, w.dO, C, EPI_STORE), st));
    int attn_launched = 1;
    NC_RUN(K_ATTN_BWD, attn_bwd_flops, 0,
           if (launch_attn_bwd<T>(w.qkv[l], ldqkv, w.O[l], w.dO, w.lse[l], w.Drow, w.dqkv, B, T_len, H,
                                  m->layer_window[l], 0, m->status, st, w.attn_part, w.attn_part_bytes,
                                  m->num_sms, &attn_launched) != cudaSuccess) return NC_ECUDA);
    m->launches[K_ATTN_BWD] += attn_launched - 1;  // one accounting entry, two or three kernels
    if (W.ve[l]) {
      // v += g ve[tok]:  dg = sum_i dv_i . ve[tok_i];  dve[v] = g sum_{tok_i = v} dv_i
      const T *dv = w.dqkv + (size_t)(H + 1) * kHeadDim;
      const int nb = (M + 63) / 64;
      float *gv = G(m->ve_param[l]);
      NC_RUN(K_VE_BWD, 0, M * 2.0 * kHeadDim * es,
             (ve_gate_partial_kernel<T><<<nb, 256, 0, st>>>(dv, ldqkv, tokens, W.ve[l], V, M, w.ve_part)));
      NC_RUN(K_VE_BWD, 0, nb * 4.0,
             (ordered_sum_kernel<<<1, 1024, 0, st>>>(w.ve_part, nb, 1.f, G(m->p_gates) + m->ve_slot[l], acc)));
      if (!acc && cudaMemsetAsync(gv, 0, sizeof(float) * (size_t)V * kHeadDim, st) != cudaSuccess) return NC_ECUDA;
      ValueEmbedRows<T> src{dv, ldqkv, W.gates + m->ve_slot[l]};
      NC_RUN(K_VE_BWD, 0, M * (kHeadDim * es + 8.0),
             (segsum_kernel<ValueEmbedRows<T>, 1><<<(nch + 7) / 8, 256, 0, st>>>(
                 src, w.sort.skey, w.sort.spos, M, kHeadDim, gv, w.seg_head, w.seg_tail, w.seg_flags, acc)));
      NC_RUN(K_SEG_FIXUP, 0, 0,
             (seg_fixup_kernel<<<nch, 256, 0, st>>>(w.sort.skey, M, kHeadDim, w.seg_head, w.seg_tail, w.seg_flags,
                                                    nch, gv, acc)));
    }
    NC_RUN(K_ROPE_QKNORM_BWD, 0, M * (3.0 * (C + kHeadDim) * es + 4.0 * (H + 1)),
           (rope_qknorm_bwd_kernel<T><<<rows_grid((size_t)M, 8), 256, 0, st>>>(
               w.dqkv, w.qkv[l], ldqkv, w.rq[l], w.rk[l], m->rope_cos, m->rope_sin, M, T_len, H)));
    // [q|k|v] = xn [Wq;Wk;Wv]^T
    NC_TRY(gemm<T>(m, gp(ldqkv, C, M, w.dqkv, ldqkv, 1, w.xn[l], C, 1, G(pi), C, wg), st));
    NC_TRY(bucket_done(m, 1 + (m->depth - 1 - l), st));  // the block's six matrices are final
    NC_TRY(gemm<T>(m, gp(M, C, ldqkv, w.dqkv, ldqkv, 0, W.wqkv[l], C, 1, w.dy, C, EPI_STORE), st));
    if (m->scalars) {
      // block entry: dx_in = dx + norm bwd;  dx = lam_r dx_in;  dx0 += lam_0 dx_in
      float *pr = w.scal_part + (size_t)l * nblk8, *p0 = w.scal_part + (size_t)(m->depth + l) * nblk8;
      NC_RUN(K_RMSNORM_BWD, 0, nbwd + M * (8.0 * C + 2.0 * C * es),
             NC_DISPATCH_NV(C, (rmsnorm_bwd_mix_kernel<T, NV><<<nblk8, 256, 0, st>>>(
                                   w.dy, w.xn[l], w.r1[l], w.dx, w.dxb, w.xs[l], w.xs[0], W.resid + l, W.x0l + l,
                                   w.dx0, l == m->depth - 1, pr, p0, M, C))));
    } else {
      NC_RUN(K_RMSNORM_BWD, 0, nbwd,
             NC_DISPATCH_NV(C, (rmsnorm_bwd_kernel<T, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                                   w.dy, w.xn[l], w.r1[l], w.dx, w.dxb, M, C, 1))));
    }
  }
  if (m->scalars) {
    // resid_lambdas and x0_lambdas are adjacent in the layout: 2L sums
    NC_RUN(K_VE_BWD, 0, 2.0 * m->depth * nblk8 * 4.0,
           (ordered_sum_rows_kernel<<<2 * m->depth, 256, 0, st>>>(w.scal_part, (int)nblk8, G(m->p_resid), 1,
                                                                   acc)));
  }
  // embedding: through the first norm, summed per token over its positions
  // in a fixed order (positions sorted by token; no floating-point atomics)
  // (with residual scalars the gradient reaching x0 through the mixing, dx0, adds to dx)
  if (!acc && cudaMemsetAsync(G(0), 0, sizeof(float) * (size_t)V * C, st) != cudaSuccess) return NC_ECUDA;
  NC_RUN(K_EMBED_BWD, 0, M * (4.0 * C + C * es + 12.0) + (m->scalars ? M * 4.0 * C : 0.0),
         NC_DISPATCH_NV(C, (segsum_kernel<EmbedRows<T, NV>, NV><<<(nch + 7) / 8, 256, 0, st>>>(
                               EmbedRows<T, NV>{w.dx, m->scalars ? w.dx0 : nullptr, W.wte, w.r0, C}, w.sort.skey,
                               w.sort.spos, M, C, G(0), w.seg_head, w.seg_tail, w.seg_flags, acc))));
  NC_RUN(K_SEG_FIXUP, 0, 0,
         (seg_fixup_kernel<<<nch, 256, 0, st>>>(w.sort.skey, M, C, w.seg_head, w.seg_tail, w.seg_flags, nch, G(0),
                                                acc)));
  NC_TRY(bucket_done(m, m->depth + 1, st));
  if ((int)m->buckets.size() > m->depth + 2) NC_TRY(bucket_done(m, m->depth + 2, st));  // the extras
  return NC_OK;
}

template <typename T>
int fwd_impl(nc_model *m, const void *weights, const int32_t *tokens, int B, int T_len,
             void *workspace, void *logits, cudaStream_t st) {
  Work<T> w;
  carve<T>(m, B, T_len, (char *)workspace, &w);
  const Weights<T> W = weight_ptrs<T>(m, weights);
  const int M = B * T_len;
  NC_TRY(forward_body<T>(m, W, tokens, B, T_len, w, st));
  return gemm<T>(m, gp(M, m->V, m->C, w.xf, m->C, 0, W.lm_head, m->C, 0, logits, m->V, EPI_SOFTCAP), st);
}

int check_step_args(const nc_model *m, const void *weights, const int32_t *tokens, int B, int T,
                    void *workspace, size_t ws_bytes) {
  if (!m || !weights || !tokens || !workspace) return NC_EINVAL;
  if (B < 1 || T < 1 || T > m->seq) return NC_ESHAPE;
  if ((int64_t)B * T > (int64_t)1 << 30) return NC_ESHAPE;
  size_t need = 0;
  need = m->dtype == NC_F32 ? carve<float>(m, B, T, nullptr, nullptr)
                            : carve<bf16>(m, B, T, nullptr, nullptr);
  if (ws_bytes < need) return NC_ENOMEM;
  if (((uintptr_t)weights & 15) || ((uintptr_t)workspace & (kAlign - 1)) || ((uintptr_t)tokens & 3))
    return NC_EALIGN;
  return NC_OK;
}


// Wait at most timeout_ms for the work enqueued so far on `st` (polling),
// then read and clear a device status word.
int read_status_word(int *word_dev, cudaStream_t st, int timeout_ms) {
  cudaEvent_t ev;
  if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return NC_ECUDA;
  if (cudaEventRecord(ev, st) != cudaSuccess) {
    cudaEventDestroy(ev);
    return NC_ECUDA;
  }
  const auto t0 = std::chrono::steady_clock::now();
  cudaError_t q;
  while ((q = cudaEventQuery(ev)) == cudaErrorNotReady) {
    const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(
                        std::chrono::steady_clock::now() - t0).count();
    if (ms >= timeout_ms) {
      cudaEventDestroy(ev);
      return NC_ETIMEOUT;
    }
    std::this_thread::sleep_for(std::chrono::microseconds(100));
  }
  cudaEventDestroy(ev);
  if (q != cudaSuccess) return NC_ECUDA;
  int word = 0;
  if (cudaMemcpyAsync(&word, word_dev, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(word_dev, 0, sizeof(int), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return NC_ECUDA;
  if (word & kStatusRange) return NC_ERANGE;
  if (word & kStatusNonFinite) return NC_ENONFINITE;
  if (word & kStatusTimeout) return NC_ETIMEOUT;
  return NC_OK;
}

// File-scope device words of the op-level entry points, which have no model
// handle: the status word their kernels report to (read by nc_ops_status)
// and the fixed scratch of nc_attention_bwd_noalloc (rowsum(dO * O)).
static __device__ int g_ops_status;
static __device__ __align__(256) float g_attn_bwd_rowdot[NC_ATTN_BWD_NOALLOC_MAX_ROWS];

// In host code those names are host-side stand-ins, not device addresses.
// Their device addresses belong to the CUDA context (a module is loaded per
// context), so they are looked up with cudaGetSymbolAddress and cached per
// context, keyed by the context's unique id: a context created after a
// cudaDeviceReset gets a new id and a fresh lookup, never a stale address.
struct SymbolAddrs {
  unsigned long long ctx_id;
  int *ops_status;
  float *rowdot;
};
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
static std::mutex g_sym_mutex;
static std::vector<SymbolAddrs> g_sym_cache;

int context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_cur || !get_id) {
    void *f1 = nullptr, *f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
      return NC_ECUDA;
    get_cur = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return NC_ECUDA;
  return get_id(ctx, id) == CUDA_SUCCESS ? NC_OK : NC_ECUDA;
}

// Addresses of the file-scope device words in the current context; the first
// call in a context looks them up (and makes the runtime's primary context
// current if there is none yet).
int symbol_addrs(SymbolAddrs *out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NC_ECUDA;
  unsigned long long id = 0;
  if (context_id(&id) != NC_OK) {
    // no current context yet: a runtime call that needs one creates it
    void *probe = nullptr;
    if (cudaGetSymbolAddress(&probe, g_ops_status) != cudaSuccess || context_id(&id) != NC_OK) return NC_ECUDA;
  }
  std::lock_guard<std::mutex> lock(g_sym_mutex);
  for (const SymbolAddrs &e : g_sym_cache)
    if (e.ctx_id == id) {
      *out = e;
      return NC_OK;
    }
  SymbolAddrs e;
  e.ctx_id = id;
  void *p1 = nullptr, *p2 = nullptr;
  if (cudaGetSymbolAddress(&p1, g_ops_status) != cudaSuccess || !p1 ||
      cudaGetSymbolAddress(&p2, g_attn_bwd_rowdot) != cudaSuccess || !p2)
    return NC_ECUDA;
  e.ops_status = static_cast<int *>(p1);
  e.rowdot = static_cast<float *>(p2);
  g_sym_cache.push_back(e);
  *out = e;
  return NC_OK;
}

// Device set-up shared by the op-level entry points: SM count, kernel
// attributes, and the status word their kernels report to.
int op_setup(int *num_sms, int **status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NC_ECUDA;
  if (cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return NC_ECUDA;
  if (tc_init() != cudaSuccess || fatc::init() != cudaSuccess || ce_init() != cudaSuccess) return NC_ECUDA;
  SymbolAddrs a;
  if (symbol_addrs(&a) != NC_OK) return NC_ECUDA;
  *status = a.ops_status;
  return NC_OK;
}

// The attention ops take the row stride as int64 but the kernels index with
// 32 bits: strides beyond INT_MAX are a shape error, not a silent truncation.
inline bool attn_shape_ok(int B, int T, int H, int64_t ld) {
  return B >= 1 && T >= 1 && H >= 1 && ld >= (int64_t)kHeadDim * (H + 2) && ld <= INT32_MAX &&
         (int64_t)B * T * ld <= ((int64_t)1 << 40);
}

// A bounded wait on an mbarrier that nothing completes: it runs out after
// wait_ns and reports kStatusTimeout, the path every kernel wait takes when
// its partner never arrives.
__global__ void wait_expiry_kernel(uint64_t wait_ns, int *status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t a = tc::smem_u32(&bar);
  tc::mbar_init(a, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const uint64_t t0 = tc::globaltimer();
  for (uint32_t i = 0;; ++i) {
    if (tc::mbar_try(a, 0)) return;  // never: nothing arrives on the barrier
    if ((i & 63) == 0 && tc::globaltimer() - t0 > wait_ns) {
      set_status(status, kStatusTimeout);
      return;
    }
  }
}

// ---------------------------------------------------------------------------
// Inference with a KV cache

constexpr int kMaxCacheT = 32768;  // longest cache the decode kernel's shared memory holds

template <typename T>
int prefill_impl(nc_model *m, const void *weights, const int32_t *tokens, int B, int T_len, void *cache, int T_max,
                 int32_t *seqlens, void *workspace, void *logits, cudaStream_t st) {
  Work<T> w;
  carve<T>(m, B, T_len, (char *)workspace, &w);
  const Weights<T> W = weight_ptrs<T>(m, weights);
  Infer<T> inf;
  inf.cache = (T *)cache;
  inf.tmax = T_max;
  NC_TRY(forward_body<T>(m, W, tokens, B, T_len, w, st, &inf));
  seqlens_kernel<<<(B + 255) / 256, 256, 0, st>>>(seqlens, B, T_len);
  NC_CHECK_LAUNCH();
  // logits of each row's last position: rows b*T + T-1 of xf (row stride T*C)
  const int64_t C = m->C;
  return gemm<T>(m, gp(B, m->V, m->C, w.xf + (T_len - 1) * C, T_len * C, 0, W.lm_head, C, 0, logits, m->V,
                       EPI_SOFTCAP), st);
}

template <typename T>
int decode_impl(nc_model *m, const void *weights, const int32_t *tokens, int B, void *cache, int T_max,
                int32_t *seqlens, void *workspace, void *logits, cudaStream_t st) {
  Work<T> w;
  carve<T>(m, B, 1, (char *)workspace, &w);
  const Weights<T> W = weight_ptrs<T>(m, weights);
  Infer<T> inf;
  inf.cache = (T *)cache;
  inf.tmax = T_max;
  inf.positions = seqlens;
  NC_TRY(forward_body<T>(m, W, tokens, B, 1, w, st, &inf));
  NC_TRY(gemm<T>(m, gp(B, m->V, m->C, w.xf, m->C, 0, W.lm_head, m->C, 0, logits, m->V, EPI_SOFTCAP), st));
  seqlens_kernel<<<(B + 255) / 256, 256, 0, st>>>(seqlens, B, -1);
  NC_CHECK_LAUNCH();
  return NC_OK;
}

int check_infer_args(const nc_model *m, void *cache, int T_max, int32_t *seqlens, void *logits, int B) {
  if (!cache || !seqlens || !logits) return NC_EINVAL;
  if (T_max < 1 || T_max > m->seq || T_max > kMaxCacheT) return NC_ESHAPE;
  if (((uintptr_t)cache & 15) || ((uintptr_t)logits & 15) || ((uintptr_t)seqlens & 3)) return NC_EALIGN;
  if (m->dtype == NC_BF16 && (m->V % 8)) return NC_EALIGN;  // logit rows leave the GEMM by TMA
  (void)B;
  return NC_OK;
}

// ---------------------------------------------------------------------------
// Optimizer step (Muon for the block matrices, AdamW for the rest)

enum ParamGroup { G_MATRIX, G_EMBED, G_HEAD, G_SCALAR };

ParamGroup param_group(const char *name) {
  if (!strcmp(name, "lm_head")) return G_HEAD;
  if (!strcmp(name, "wte") || (name[0] == 'v' && name[1] == 'e' && name[2] >= '0' && name[2] <= '9')) return G_EMBED;
  if (!strcmp(name, "resid_lambdas") || !strcmp(name, "x0_lambdas") || !strcmp(name, "ve_gates")) return G_SCALAR;
  return G_MATRIX;
}

// Newton-Schulz scratch: two X buffers of the largest matrix, the Gram matrix
// of the largest shorter side (fp32) and its coefficient matrix, the norm's
// partial sums.
struct OptimWork {
  char *x0, *x1, *bm;
  float *gram, *partial;
};

size_t optim_carve(const nc_model *m, char *base, OptimWork *w) {
  int64_t big = 0, small = 0;
  for (const nc_param &p : m->params)
    if (param_group(p.name) == G_MATRIX) {
      big = std::max<int64_t>(big, (int64_t)p.rows * p.cols);
      small = std::max<int64_t>(small, std::min(p.rows, p.cols));
    }
  const size_t es = m->dtype == NC_F32 ? 4 : 2;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char * {
    char *q = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return q;
  };
  char *x0 = take(big * es), *x1 = take(big * es), *bm = take(small * small * es);
  float *gram = (float *)take(small * small * 4), *partial = (float *)take((kOptBlocks + 1) * 4);
  if (w) *w = OptimWork{x0, x1, bm, gram, partial};
  return off;
}

template <typename T>
int optim_step_impl(nc_model *m, T *weights, const float *grads, float *state, int step, const nc_optim_opts &o,
                    void *workspace, cudaStream_t st) {
  OptimWork ow;
  optim_carve(m, (char *)workspace, &ow);
  const int64_t N = m->n_params;
  float *master = state, *mom = state + N, *vel = state + 2 * N;
  const float bc1 = 1.f / (1.f - powf(o.beta1, (float)step)), bc2 = 1.f / (1.f - powf(o.beta2, (float)step));
  const double es = sizeof(T);
  for (const nc_param &p : m->params) {
    const int64_t off = p.offset, n = (int64_t)p.rows * p.cols;
    const ParamGroup grp = param_group(p.name);
    if (grp != G_MATRIX) {
      const float lr = grp == G_EMBED ? o.lr_embed : grp == G_HEAD ? o.lr_head : o.lr_scalar;
      NC_RUN(K_OPTIM, 0, n * (20.0 + es),
             (adamw_kernel<T><<<ew_grid(n, m->num_sms), 256, 0, st>>>(weights + off, master + off, grads + off,
                                                                       mom + off, vel + off, n, lr, o.beta1, o.beta2,
                                                                       o.eps, o.weight_decay, bc1, bc2)));
      continue;
    }
    T *X = (T *)ow.x0, *Y = (T *)ow.x1, *Bm = (T *)ow.bm;
    NC_RUN(K_OPTIM, 0, n * 12.0,
           (muon_momentum_kernel<<<kOptBlocks, 256, 0, st>>>(grads + off, mom + off, n, o.muon_momentum,
                                                             ow.partial)));
    NC_RUN(K_OPTIM, 0, 0, (ordered_sum_kernel<<<1, 1024, 0, st>>>(ow.partial, kOptBlocks, 1.f,
                                                                  ow.partial + kOptBlocks, 0)));
    NC_RUN(K_OPTIM, 0, n * (4.0 + es),
           (muon_scale_kernel<T><<<ew_grid(n, m->num_sms), 256, 0, st>>>(mom + off, n, ow.partial + kOptBlocks, X)));
    const int r = p.rows, c = p.cols;
    for (int k = 0; k < o.ns_steps; ++k) {
      if (r >= c) {  // X (1.5 I - 0.5 X^T X): the Gram matrix of the columns
        NC_TRY(gemm<T>(m, gp(c, c, r, X, c, 1, X, c, 1, ow.gram, c, EPI_STORE_F32), st));
        NC_RUN(K_OPTIM, 0, (double)c * c * (4.0 + es),
               (ns_coeff_kernel<T><<<ew_grid((int64_t)c * c, m->num_sms), 256, 0, st>>>(ow.gram, c, Bm)));
        NC_TRY(gemm<T>(m, gp(r, c, c, X, c, 0, Bm, c, 1, Y, c, EPI_STORE), st));
      } else {       // (1.5 I - 0.5 X X^T) X: the Gram matrix of the rows
        NC_TRY(gemm<T>(m, gp(r, r, c, X, c, 0, X, c, 0, ow.gram, r, EPI_STORE_F32), st));
        NC_RUN(K_OPTIM, 0, (double)r * r * (4.0 + es),
               (ns_coeff_kernel<T><<<ew_grid((int64_t)r * r, m->num_sms), 256, 0, st>>>(ow.gram, r, Bm)));
        NC_TRY(gemm<T>(m, gp(r, c, r, Bm, r, 0, X, c, 1, Y, c, EPI_STORE), st));
      }
      std::swap(X, Y);
    }
    NC_RUN(K_OPTIM, 0, n * (8.0 + 2.0 * es),
           (muon_apply_kernel<T><<<ew_grid(n, m->num_sms), 256, 0, st>>>(master + off, X, weights + off, n,
                                                                          o.lr_matrix, o.weight_decay)));
  }
  return NC_OK;
}

}  // namespace

extern "C" {

int nc_init(int depth, int vocab, int seq, int dtype, nc_model **out) {
  return nc_init_ex(depth, vocab, seq, dtype, nullptr, out);
}

int nc_init_ex(int depth, int vocab, int seq, int dtype, const nc_block_opts *opts, nc_model **out) {
  if (!out) return NC_EINVAL;
  *out = nullptr;
  if (depth < 1 || vocab < 2 || seq < 1) return NC_EINVAL;
  if (opts && opts->window < 0) return NC_EINVAL;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  const int C = kHeadDim * ((64 * depth + kHeadDim - 1) / kHeadDim);
  if (C > 32 * kMaxVecPerLane * 8) return NC_EINVAL;  // widest row the row kernels hold
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NC_ECUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return NC_ECUDA;
  if (prop.major != 10) return NC_EUNSUPPORTED;

  nc_model *m = new nc_model();
  m->depth = depth; m->C = C; m->H = C / kHeadDim; m->F = 4 * C; m->V = vocab; m->seq = seq;
  m->dtype = dtype; m->device = dev; m->num_sms = prop.multiProcessorCount;
  int64_t off = 0;
  auto add = [&](const char *name, int rows, int cols) {
    nc_param p;
    memset(&p, 0, sizeof(p));
    snprintf(p.name, sizeof(p.name), "%s", name);
    p.offset = off; p.rows = rows; p.cols = cols;
    off += (int64_t)rows * cols;
    m->params.push_back(p);
  };
  add("wte", vocab, C);
  char nm[24];
  for (int l = 0; l < depth; ++l) {
    snprintf(nm, sizeof(nm), "h%d.wq", l); add(nm, C, C);
    snprintf(nm, sizeof(nm), "h%d.wk", l); add(nm, kHeadDim, C);
    snprintf(nm, sizeof(nm), "h%d.wv", l); add(nm, kHeadDim, C);
    snprintf(nm, sizeof(nm), "h%d.wo", l); add(nm, C, C);
    snprintf(nm, sizeof(nm), "h%d.w1", l); add(nm, 4 * C, C);
    snprintf(nm, sizeof(nm), "h%d.w2", l); add(nm, C, 4 * C);
  }
  add("lm_head", vocab, C);
  // full reference block: the "SSSL" window schedule (last layer always
  // full), value-embedding tables on layers 0, 2, ..., then the scalars
  m->window = opts ? opts->window : 0;
  m->ve = opts && opts->value_embeds;
  m->scalars = opts && opts->resid_scalars;
  m->layer_window.assign(depth, 0);
  m->ve_param.assign(depth, -1);
  m->ve_slot.assign(depth, -1);
  for (int l = 0; l < depth; ++l) {
    const char kind = l == depth - 1 ? 'L' : "SSSL"[l % 4];
    if (kind == 'S') m->layer_window[l] = m->window;
  }
  int n_ve = 0;
  if (m->ve)
    for (int l = 0; l < depth; l += 2) {
      snprintf(nm, sizeof(nm), "ve%d", l);
      m->ve_param[l] = (int)m->params.size();
      m->ve_slot[l] = n_ve++;
      add(nm, vocab, kHeadDim);
    }
  if (m->scalars) {
    m->p_resid = (int)m->params.size();
    add("resid_lambdas", 1, depth);
    m->p_x0 = (int)m->params.size();
    add("x0_lambdas", 1, depth);
  }
  if (m->ve) {
    m->p_gates = (int)m->params.size();
    add("ve_gates", 1, n_ve);
  }
  m->n_params = off;
  // gradient buckets, completion order: lm_head, blocks L-1 .. 0, wte, extras
  const int first_extra = 2 + 6 * depth;
  m->buckets.push_back({m->params[1 + 6 * depth].offset, (int64_t)vocab * C});
  for (int l = depth - 1; l >= 0; --l) {
    const nc_param &a = m->params[1 + 6 * l], &z = m->params[6 + 6 * l];
    m->buckets.push_back({a.offset, z.offset + (int64_t)z.rows * z.cols - a.offset});
  }
  m->buckets.push_back({0, (int64_t)vocab * C});
  if ((int)m->params.size() > first_extra)
    m->buckets.push_back({m->params[first_extra].offset, off - m->params[first_extra].offset});

  // RoPE table: angle = pos * 10000^(-i/64), built in float64, rounded once.
  std::vector<float> hc((size_t)seq * 64), hs((size_t)seq * 64);
  for (int p = 0; p < seq; ++p)
    for (int i = 0; i < 64; ++i) {
      const double ang = (double)p * pow(10000.0, -(double)i / 64.0);
      hc[(size_t)p * 64 + i] = (float)cos(ang);
      hs[(size_t)p * 64 + i] = (float)sin(ang);
    }
  bool ok = cudaMalloc(&m->rope_cos, hc.size() * 4) == cudaSuccess &&
            cudaMalloc(&m->rope_sin, hs.size() * 4) == cudaSuccess &&
            cudaMalloc(&m->status, 256) == cudaSuccess &&
            cudaMemcpy(m->rope_cos, hc.data(), hc.size() * 4, cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(m->rope_sin, hs.data(), hs.size() * 4, cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemset(m->status, 0, 256) == cudaSuccess;
  if (ok)
    ok = cudaFuncSetAttribute(attn_decode_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)attn_decode_smem(kMaxCacheT)) == cudaSuccess &&
         cudaFuncSetAttribute(attn_decode_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)attn_decode_smem(kMaxCacheT)) == cudaSuccess;
  if (!ok || tc_init() != cudaSuccess || fatc::init() != cudaSuccess || ce_init() != cudaSuccess) {
    nc_destroy(m);
    return NC_ECUDA;
  }
  *out = m;
  return NC_OK;
}

int nc_get_dims(const nc_model *m, nc_dims *out) {
  if (!m || !out) return NC_EINVAL;
  out->depth = m->depth; out->width = m->C; out->n_head = m->H; out->head_dim = kHeadDim;
  out->hidden = m->F; out->vocab = m->V; out->seq = m->seq; out->dtype = m->dtype;
  out->n_params = m->n_params;
  return NC_OK;
}

int nc_grad_bucket_count(const nc_model *m, int *count) {
  if (!m || !count) return NC_EINVAL;
  *count = (int)m->buckets.size();
  return NC_OK;
}

int nc_grad_bucket(const nc_model *m, int k, int64_t *offset, int64_t *count) {
  if (!m || !offset || !count || k < 0 || k >= (int)m->buckets.size()) return NC_EINVAL;
  *offset = m->buckets[k].first;
  *count = m->buckets[k].second;
  return NC_OK;
}

int nc_set_grad_events(nc_model *m, void *const *events, int n) {
  if (!m || n < 0 || (n > 0 && !events) || n > (int)m->buckets.size()) return NC_EINVAL;
  m->grad_events.assign(n, nullptr);
  for (int i = 0; i < n; ++i) m->grad_events[i] = (cudaEvent_t)events[i];
  return NC_OK;
}

int nc_layer_window(const nc_model *m, int layer, int *window) {
  if (!m || !window || layer < 0 || layer >= m->depth) return NC_EINVAL;
  *window = m->layer_window[layer];
  return NC_OK;
}

int nc_param_count(const nc_model *m, int *count) {
  if (!m || !count) return NC_EINVAL;
  *count = (int)m->params.size();
  return NC_OK;
}

int nc_param_layout(const nc_model *m, int index, nc_param *out) {
  if (!m || !out || index < 0 || index >= (int)m->params.size()) return NC_EINVAL;
  *out = m->params[index];
  return NC_OK;
}

int nc_workspace_bytes(const nc_model *m, int B, int T, size_t *out) {
  if (!m || !out) return NC_EINVAL;
  if (B < 1 || T < 1 || T > m->seq) return NC_ESHAPE;
  *out = m->dtype == NC_F32 ? carve<float>(m, B, T, nullptr, nullptr)
                            : carve<bf16>(m, B, T, nullptr, nullptr);
  return NC_OK;
}

int nc_fwd_bwd(nc_model *m, const void *weights, const int32_t *tokens, const int32_t *targets,
               int B, int T, void *workspace, size_t ws_bytes, float *loss, float *token_loss,
               float *grads, void *stream) {
  return nc_fwd_bwd_ex(m, weights, tokens, targets, B, T, workspace, ws_bytes, loss, token_loss, grads, 0,
                       stream);
}

int nc_fwd_bwd_ex(nc_model *m, const void *weights, const int32_t *tokens, const int32_t *targets,
                  int B, int T, void *workspace, size_t ws_bytes, float *loss, float *token_loss,
                  float *grads, int flags, void *stream) {
  if (flags & ~NC_ACCUMULATE) return NC_EINVAL;
  int rc = check_step_args(m, weights, tokens, B, T, workspace, ws_bytes);
  if (rc != NC_OK) return rc;
  if (!targets || !loss || !grads) return NC_EINVAL;
  if (((uintptr_t)grads & 15) || ((uintptr_t)targets & 3) || ((uintptr_t)loss & 3)) return NC_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (m->dtype == NC_F32)
    return fwd_bwd_impl<float>(m, weights, tokens, targets, B, T, workspace, loss, token_loss, grads, flags, st);
  return fwd_bwd_impl<bf16>(m, weights, tokens, targets, B, T, workspace, loss, token_loss, grads, flags, st);
}

int nc_fwd(nc_model *m, const void *weights, const int32_t *tokens, int B, int T, void *workspace,
           size_t ws_bytes, void *logits, void *stream) {
  int rc = check_step_args(m, weights, tokens, B, T, workspace, ws_bytes);
  if (rc != NC_OK) return rc;
  if (!logits) return NC_EINVAL;
  if ((uintptr_t)logits & 15) return NC_EALIGN;
  // bf16 logit rows leave the tensor-core GEMM by TMA: 16-byte row strides
  if (m->dtype == NC_BF16 && (m->V % 8)) return NC_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (m->dtype == NC_F32) return fwd_impl<float>(m, weights, tokens, B, T, workspace, logits, st);
  return fwd_impl<bf16>(m, weights, tokens, B, T, workspace, logits, st);
}

int nc_kv_cache_bytes(const nc_model *m, int B, int T_max, size_t *out) {
  if (!m || !out) return NC_EINVAL;
  if (B < 1 || T_max < 1 || T_max > m->seq || T_max > kMaxCacheT) return NC_ESHAPE;
  *out = (size_t)m->depth * 2 * B * T_max * kHeadDim * (m->dtype == NC_F32 ? 4 : 2);
  return NC_OK;
}

int nc_prefill(nc_model *m, const void *weights, const int32_t *tokens, int B, int T, void *cache, int T_max,
               int32_t *seqlens, void *workspace, size_t ws_bytes, void *logits, void *stream) {
  int rc = check_step_args(m, weights, tokens, B, T, workspace, ws_bytes);
  if (rc != NC_OK) return rc;
  if ((rc = check_infer_args(m, cache, T_max, seqlens, logits, B)) != NC_OK) return rc;
  if (T > T_max) return NC_ESHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  if (m->dtype == NC_F32) return prefill_impl<float>(m, weights, tokens, B, T, cache, T_max, seqlens, workspace, logits, st);
  return prefill_impl<bf16>(m, weights, tokens, B, T, cache, T_max, seqlens, workspace, logits, st);
}

int nc_decode(nc_model *m, const void *weights, const int32_t *tokens, int B, void *cache, int T_max,
              int32_t *seqlens, void *workspace, size_t ws_bytes, void *logits, void *stream) {
  int rc = check_step_args(m, weights, tokens, B, 1, workspace, ws_bytes);
  if (rc != NC_OK) return rc;
  if ((rc = check_infer_args(m, cache, T_max, seqlens, logits, B)) != NC_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if (m->dtype == NC_F32) return decode_impl<float>(m, weights, tokens, B, cache, T_max, seqlens, workspace, logits, st);
  return decode_impl<bf16>(m, weights, tokens, B, cache, T_max, seqlens, workspace, logits, st);
}

int nc_optim_state_bytes(const nc_model *m, size_t *out) {
  if (!m || !out) return NC_EINVAL;
  *out = (size_t)3 * m->n_params * sizeof(float);
  return NC_OK;
}

int nc_optim_workspace_bytes(const nc_model *m, size_t *out) {
  if (!m || !out) return NC_EINVAL;
  *out = optim_carve(m, nullptr, nullptr);
  return NC_OK;
}

int nc_optim_init(nc_model *m, const void *weights, void *state, void *stream) {
  if (!m || !weights || !state) return NC_EINVAL;
  if (((uintptr_t)weights & 15) || ((uintptr_t)state & 15)) return NC_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t N = m->n_params;
  float *master = (float *)state;
  if (m->dtype == NC_F32)
    optim_init_kernel<float><<<ew_grid(N, m->num_sms), 256, 0, st>>>((const float *)weights, master, master + N,
                                                                      master + 2 * N, N);
  else
    optim_init_kernel<bf16><<<ew_grid(N, m->num_sms), 256, 0, st>>>((const bf16 *)weights, master, master + N,
                                                                     master + 2 * N, N);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ECUDA;
}

int nc_optim_step(nc_model *m, void *weights, const float *grads, void *state, int step, const nc_optim_opts *o,
                  void *workspace, size_t ws_bytes, void *stream) {
  if (!m || !weights || !grads || !state || !o || !workspace) return NC_EINVAL;
  if (step < 1 || o->ns_steps < 0 || o->ns_steps > 100 || !(o->beta1 >= 0.f && o->beta1 < 1.f) ||
      !(o->beta2 >= 0.f && o->beta2 < 1.f) || !(o->eps >= 0.f))
    return NC_EINVAL;
  if (ws_bytes < optim_carve(m, nullptr, nullptr)) return NC_ENOMEM;
  if (((uintptr_t)weights & 15) || ((uintptr_t)grads & 15) || ((uintptr_t)state & 15) ||
      ((uintptr_t)workspace & (kAlign - 1)))
    return NC_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (m->dtype == NC_F32)
    return optim_step_impl<float>(m, (float *)weights, grads, (float *)state, step, *o, workspace, st);
  return optim_step_impl<bf16>(m, (bf16 *)weights, grads, (float *)state, step, *o, workspace, st);
}

int nc_sync_status(nc_model *m, void *stream, int timeout_ms) {
  if (!m) return NC_EINVAL;
  return read_status_word(m->status, (cudaStream_t)stream, timeout_ms);
}

int nc_profile(nc_model *m, int enable) {
  if (!m) return NC_EINVAL;
  m->prof = enable != 0;
  return NC_OK;
}

int nc_profile_read(nc_model *m, nc_kernel_stat *out, int max, int *count) {
  if (!m || (!out && max > 0) || !count) return NC_EINVAL;
  double ms[K_NUM_CLASSES] = {};
  int rc = NC_OK;
  if (!m->records.empty()) {
    if (cudaEventSynchronize(m->events[m->records.back().second + 1]) != cudaSuccess) rc = NC_ECUDA;
    for (const auto &r : m->records) {
      float t = 0.f;
      if (rc == NC_OK && cudaEventElapsedTime(&t, m->events[r.second], m->events[r.second + 1]) == cudaSuccess)
        ms[r.first] += t;
    }
  }
  int n = 0;
  for (int c = 0; c < K_NUM_CLASSES; ++c) {
    if (!m->launches[c]) continue;
    if (n < max) {
      memset(&out[n], 0, sizeof(nc_kernel_stat));
      snprintf(out[n].name, sizeof(out[n].name), "%s", kClassName[c]);
      out[n].launches = m->launches[c];
      out[n].ms = ms[c];
      out[n].flops = m->flops[c];
      out[n].bytes = m->bytes[c];
    }
    ++n;
  }
  *count = n < max ? n : max;
  m->records.clear();
  m->events_used = 0;
  for (int c = 0; c < K_NUM_CLASSES; ++c) { m->launches[c] = 0; m->flops[c] = 0; m->bytes[c] = 0; }
  return rc;
}

const char *nc_strerror(int code) {
  switch (code) {
    case NC_OK: return "ok";
    case NC_EINVAL: return "invalid argument";
    case NC_ESHAPE: return "invalid shape (B < 1, T < 1 or T > seq)";
    case NC_ENOMEM: return "workspace too small";
    case NC_EUNSUPPORTED: return "unsupported device or dtype (needs sm_100)";
    case NC_ECUDA: return "CUDA runtime error";
    case NC_ERANGE: return "token or target id outside [0, vocab)";
    case NC_ENONFINITE: return "non-finite loss";
    case NC_ETIMEOUT: return "timed out";
    case NC_EALIGN: return "misaligned device pointer";
    default: return "unknown status";
  }
}

void nc_destroy(nc_model *m) {
  if (!m) return;
  for (cudaEvent_t e : m->events) cudaEventDestroy(e);
  if (m->rope_cos) cudaFree(m->rope_cos);
  if (m->rope_sin) cudaFree(m->rope_sin);
  if (m->status) cudaFree(m->status);
  delete m;
}


int nc_gemm(const void *A, int64_t lda, int a_mn, const void *B, int64_t ldb, int b_mn, void *D,
            int64_t ldd, int M, int N, int K, int dtype, int epilogue, int engine, void *stream) {
  if (!A || !B || !D) return NC_EINVAL;
  if (M < 1 || N < 1 || K < 1) return NC_ESHAPE;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  if (epilogue < NC_EPI_STORE || epilogue > NC_EPI_ACC_F32 || (a_mn | b_mn) & ~1) return NC_EINVAL;
  if (engine < 0 || engine > 2) return NC_EINVAL;
  const GemmProblem p = gp(M, N, K, A, lda, a_mn, B, ldb, b_mn, D, ldd, epilogue);
  const bool tensor = dtype == NC_BF16 && engine != 1;
  if (tensor && !tc_gemm_aligned(p)) return NC_EALIGN;
  int num_sms = 0, *status = nullptr;
  if (op_setup(&num_sms, &status) != NC_OK) return NC_ECUDA;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (tensor) e = launch_gemm_tc(p, num_sms, status, st, engine == 0 ? 1 : 0);
  else if (dtype == NC_BF16) e = launch_gemm_simt<bf16>(p, st);
  else e = launch_gemm_simt<float>(p, st);
  return e == cudaSuccess ? NC_OK : NC_ECUDA;
}

int nc_attention_fwd(const void *qkv, int64_t ld, void *O, float *lse, int B, int T, int H, int window,
                     int dtype, int engine, void *stream) {
  if (!qkv || !O || !lse) return NC_EINVAL;
  if (!attn_shape_ok(B, T, H, ld)) return NC_ESHAPE;
  if (window < 0) return NC_EINVAL;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  if (engine < 0 || engine > 3) return NC_EINVAL;
  if (dtype == NC_BF16 && engine != 1 && !fatc::aligned(qkv, ld, O)) return NC_EALIGN;
  int num_sms = 0, *status = nullptr;
  if (op_setup(&num_sms, &status) != NC_OK) return NC_ECUDA;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (dtype == NC_BF16)
    e = launch_attn_fwd<bf16>((const bf16 *)qkv, (int)ld, (bf16 *)O, lse, B, T, H, window, engine, status, st,
                              num_sms);
  else
    e = launch_attn_fwd<float>((const float *)qkv, (int)ld, (float *)O, lse, B, T, H, window, engine, status, st);
  return e == cudaSuccess ? NC_OK : NC_ECUDA;
}

static int attention_bwd_common(const void *qkv, int64_t ld, const void *O, const void *dO, const float *lse,
                                float *Drow, void *dqkv, int B, int T, int H, int window, int dtype, int engine,
                                int *status, cudaStream_t st, void *scratch = nullptr, size_t scratch_bytes = 0,
                                int num_sms = 148) {
  cudaError_t e;
  if (dtype == NC_BF16) {
    e = launch_attn_bwd<bf16>((const bf16 *)qkv, (int)ld, (const bf16 *)O, (const bf16 *)dO, lse, Drow,
                              (bf16 *)dqkv, B, T, H, window, engine, status, st, (float *)scratch, scratch_bytes,
                              num_sms);
  } else {
    e = launch_attn_bwd<float>((const float *)qkv, (int)ld, (const float *)O, (const float *)dO, lse, Drow,
                               (float *)dqkv, B, T, H, window, engine, status, st);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? NC_OK : NC_ECUDA;
}

int nc_attention_bwd(const void *qkv, int64_t ld, const void *O, const void *dO, const float *lse,
                     float *Drow, void *dqkv, int B, int T, int H, int window, int dtype, int engine,
                     void *stream) {
  if (!qkv || !O || !dO || !lse || !Drow || !dqkv) return NC_EINVAL;
  if (!attn_shape_ok(B, T, H, ld)) return NC_ESHAPE;
  if (window < 0) return NC_EINVAL;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  if (engine < 0 || engine > 1) return NC_EINVAL;
  if (dtype == NC_BF16 && engine == 0 && !fatc::aligned_bwd(qkv, ld, O, dO, dqkv)) return NC_EALIGN;
  int num_sms = 0, *status = nullptr;
  if (op_setup(&num_sms, &status) != NC_OK) return NC_ECUDA;
  return attention_bwd_common(qkv, ld, O, dO, lse, Drow, dqkv, B, T, H, window, dtype, engine, status,
                              (cudaStream_t)stream, nullptr, 0, num_sms);
}

int nc_attention_bwd_scratch_bytes(int B, int T, int H, int window, size_t *out) {
  if (!out) return NC_EINVAL;
  if (B < 1 || T < 1 || H < 1) return NC_ESHAPE;
  if (window < 0) return NC_EINVAL;
  int dev = 0, num_sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return NC_ECUDA;
  *out = fatc::dkdv_scratch_bytes(B, T, H, window, num_sms);
  return NC_OK;
}

int nc_attention_bwd_ex(const void *qkv, int64_t ld, const void *O, const void *dO, const float *lse,
                        float *Drow, void *scratch, size_t scratch_bytes, void *dqkv, int B, int T, int H,
                        int window, int dtype, int engine, void *stream) {
  if (!qkv || !O || !dO || !lse || !Drow || !dqkv) return NC_EINVAL;
  if (!attn_shape_ok(B, T, H, ld)) return NC_ESHAPE;
  if (window < 0) return NC_EINVAL;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  if (engine < 0 || engine > 1) return NC_EINVAL;
  if (dtype == NC_BF16 && engine == 0 && !fatc::aligned_bwd(qkv, ld, O, dO, dqkv)) return NC_EALIGN;
  if (scratch && ((uintptr_t)scratch & 15)) return NC_EALIGN;
  int num_sms = 0, *status = nullptr;
  if (op_setup(&num_sms, &status) != NC_OK) return NC_ECUDA;
  return attention_bwd_common(qkv, ld, O, dO, lse, Drow, dqkv, B, T, H, window, dtype, engine, status,
                              (cudaStream_t)stream, scratch, scratch ? scratch_bytes : 0, num_sms);
}

int nc_attention_bwd_noalloc(const void *qkv, int64_t ld, const void *O, const void *dO,
                             const float *lse, void *dqkv, int B, int T, int H, int dtype,
                             int engine, void *stream) {
  if (!qkv || !O || !dO || !lse || !dqkv) return NC_EINVAL;
  if (!attn_shape_ok(B, T, H, ld)) return NC_ESHAPE;
  if ((int64_t)B * H * T > NC_ATTN_BWD_NOALLOC_MAX_ROWS) return NC_ENOMEM;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  if (engine < 0 || engine > 1) return NC_EINVAL;
  if (dtype == NC_BF16 && engine == 0 && !fatc::aligned_bwd(qkv, ld, O, dO, dqkv)) return NC_EALIGN;
  int num_sms = 0, *status = nullptr;
  if (op_setup(&num_sms, &status) != NC_OK) return NC_ECUDA;
  SymbolAddrs a;
  if (symbol_addrs(&a) != NC_OK) return NC_ECUDA;
  return attention_bwd_common(qkv, ld, O, dO, lse, a.rowdot, dqkv, B, T, H, 0, dtype, engine, status,
                              (cudaStream_t)stream, nullptr, 0, num_sms);
}

int nc_softcap_ce(void *z, int64_t ldz, const int32_t *targets, float *token_loss, int M, int V,
                  float grad_scale, int dtype, void *stream) {
  if (!z || !targets || !token_loss) return NC_EINVAL;
  if (M < 1 || V < 1 || ldz < V) return NC_ESHAPE;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  if (((uintptr_t)targets & 3) || ((uintptr_t)token_loss & 3) ||
      ((uintptr_t)z & (dtype == NC_BF16 ? 1 : 3)))
    return NC_EALIGN;
  int num_sms = 0, *status = nullptr;
  if (op_setup(&num_sms, &status) != NC_OK) return NC_ECUDA;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = dtype == NC_BF16
                      ? launch_ce<bf16>((bf16 *)z, ldz, targets, token_loss, M, V, grad_scale, num_sms, status, st)
                      : launch_ce<float>((float *)z, ldz, targets, token_loss, M, V, grad_scale, num_sms, status, st);
  return e == cudaSuccess ? NC_OK : NC_ECUDA;
}

static bool rows_ok(int M, int C, const void *a, const void *b, const void *c) {
  return M >= 1 && C >= 8 && C % 8 == 0 && C <= 32 * kMaxVecPerLane * 8 &&
         !(((uintptr_t)a | (uintptr_t)b | (uintptr_t)c) & 15);
}

int nc_rmsnorm(const void *x, void *y, float *r, int M, int C, int dtype, void *stream) {
  if (!x || !y || !r) return NC_EINVAL;
  if (M < 1 || C < 8 || C % 8 || C > 32 * kMaxVecPerLane * 8) return NC_ESHAPE;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  if (!rows_ok(M, C, x, y, nullptr) || ((uintptr_t)r & 3)) return NC_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == NC_BF16)
    NC_DISPATCH_NV(C, (rmsnorm_kernel<bf16, NV><<<rows_grid(M, 8), 256, 0, st>>>((const bf16 *)x, (bf16 *)y, r,
                                                                                 M, C)));
  else
    NC_DISPATCH_NV(C, (rmsnorm_kernel<float, NV><<<rows_grid(M, 8), 256, 0, st>>>((const float *)x, (float *)y,
                                                                                  r, M, C)));
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ECUDA;
}

int nc_rmsnorm_bwd(const void *dy, const void *y, const float *r, float *dx, void *dx_t, int M, int C,
                   int accumulate, int dtype, void *stream) {
  if (!dy || !y || !r || !dx || !dx_t) return NC_EINVAL;
  if (M < 1 || C < 8 || C % 8 || C > 32 * kMaxVecPerLane * 8) return NC_ESHAPE;
  if (dtype != NC_F32 && dtype != NC_BF16) return NC_EUNSUPPORTED;
  if (!rows_ok(M, C, dy, y, dx) || ((uintptr_t)dx_t & 15) || ((uintptr_t)r & 3)) return NC_EALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  const int acc = accumulate ? 1 : 0;
  if (dtype == NC_BF16)
    NC_DISPATCH_NV(C, (rmsnorm_bwd_kernel<bf16, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                          (const bf16 *)dy, (const bf16 *)y, r, dx, (bf16 *)dx_t, M, C, acc)));
  else
    NC_DISPATCH_NV(C, (rmsnorm_bwd_kernel<float, NV><<<rows_grid(M, 8), 256, 0, st>>>(
                          (const float *)dy, (const float *)y, r, dx, (float *)dx_t, M, C, acc)));
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ECUDA;
}

static int rope_args_ok(const nc_model *m, const void *a, const void *b, int64_t ld, int B, int T) {
  if (B < 1 || T < 1 || T > m->seq || ld < (int64_t)kHeadDim * (m->H + 2) || ld > INT32_MAX ||
      (int64_t)B * T * ld > ((int64_t)1 << 40))
    return NC_ESHAPE;
  const int es = m->dtype == NC_BF16 ? 2 : 4;
  if ((((uintptr_t)a | (uintptr_t)b) & 15) || (ld * es) % 16) return NC_EALIGN;
  return NC_OK;
}

int nc_rope_qknorm(const nc_model *m, void *qkv, int64_t ld, float *rq, float *rk, int B, int T, void *stream) {
  if (!m || !qkv || !rq || !rk) return NC_EINVAL;
  const int rc = rope_args_ok(m, qkv, nullptr, ld, B, T);
  if (rc != NC_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const int M = B * T;
  if (m->dtype == NC_BF16)
    rope_qknorm_kernel<bf16><<<rows_grid((size_t)M, 8), 256, 0, st>>>((bf16 *)qkv, (int)ld, rq, rk, m->rope_cos,
                                                                      m->rope_sin, M, T, m->H);
  else
    rope_qknorm_kernel<float><<<rows_grid((size_t)M, 8), 256, 0, st>>>((float *)qkv, (int)ld, rq, rk, m->rope_cos,
                                                                       m->rope_sin, M, T, m->H);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ECUDA;
}

int nc_rope_qknorm_bwd(const nc_model *m, void *dqkv, const void *qkv, int64_t ld, const float *rq,
                       const float *rk, int B, int T, void *stream) {
  if (!m || !dqkv || !qkv || !rq || !rk) return NC_EINVAL;
  const int rc = rope_args_ok(m, dqkv, qkv, ld, B, T);
  if (rc != NC_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const int M = B * T;
  if (m->dtype == NC_BF16)
    rope_qknorm_bwd_kernel<bf16><<<rows_grid((size_t)M, 8), 256, 0, st>>>(
        (bf16 *)dqkv, (const bf16 *)qkv, (int)ld, rq, rk, m->rope_cos, m->rope_sin, M, T, m->H);
  else
    rope_qknorm_bwd_kernel<float><<<rows_grid((size_t)M, 8), 256, 0, st>>>(
        (float *)dqkv, (const float *)qkv, (int)ld, rq, rk, m->rope_cos, m->rope_sin, M, T, m->H);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ECUDA;
}

int nc_set_attention_ctas(int ctas) {
  if (ctas < 0) return NC_EINVAL;
  fatc::persistent_cap().store(ctas);
  return NC_OK;
}

int nc_ops_status(void *stream, int timeout_ms) {
  SymbolAddrs a;
  if (symbol_addrs(&a) != NC_OK) return NC_ECUDA;
  return read_status_word(a.ops_status, (cudaStream_t)stream, timeout_ms);
}

int nc_check_wait_expiry(int wait_us, void *stream) {
  if (wait_us < 0 || wait_us > 1000000) return NC_EINVAL;
  SymbolAddrs a;
  if (symbol_addrs(&a) != NC_OK) return NC_ECUDA;
  wait_expiry_kernel<<<1, 1, 0, (cudaStream_t)stream>>>((uint64_t)wait_us * 1000ull, a.ops_status);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ECUDA;
}

}  // extern "C"
