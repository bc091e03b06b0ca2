// Positions grouped by token id, and gradients summed per token without
// floating-point atomics: the embedding table's gradient (and any other
// table indexed by the tokens) gets sum_{i : tok_i = v} g_i in an order
// fixed by the inputs, so it is the same, bit for bit, on every run.
//
// 1. Stable LSD radix sort of the positions by token id (8-bit digits, as
//    many passes as the vocabulary needs: two for V = 65,536).  Each pass:
//    per-tile digit histograms, one exclusive scan in digit-major order,
//    then a scatter in which a warp ranks equal digits with match_any and
//    warps are ordered by a scan in shared memory -- stable, so every
//    token's positions come out in increasing order.
// 2. Segmented sum over the sorted positions: a warp owns a chunk of S
//    consecutive sorted positions and sums each run of equal tokens in it;
//    a run that is a whole segment (all of a token's positions) is written
//    straight to its row, a run cut by a chunk boundary leaves a partial,
//    and a fix-up kernel adds a segment's partials in chunk order.
#pragma once

#include "common.cuh"

namespace nc {

constexpr int kSortTile = 1024;     // elements per CTA of a radix pass
constexpr int kSortThreads = 256;   // 8 warps x 128 consecutive elements (4 rounds of 32)
constexpr int kSegChunk = 16;       // sorted positions per warp in the segmented sum

__device__ __forceinline__ int clamp_token(int t, int V) { return t < 0 ? 0 : (t >= V ? V - 1 : t); }

inline int sort_tiles(int M) { return (M + kSortTile - 1) / kSortTile; }
inline int sort_passes(int V) {
  int bits = 0;
  while (bits < 31 && (1 << bits) < V) ++bits;
  return bits <= 8 ? 1 : (bits + 7) / 8;
}
inline int seg_chunks(int M) { return (M + kSegChunk - 1) / kSegChunk; }

// hist[d * ntiles + tile] = count of digit d in the tile
__global__ void __launch_bounds__(kSortThreads) radix_hist_kernel(const int32_t *__restrict__ keys, int M, int V,
                                                                  int shift, int *__restrict__ hist, int ntiles) {
  __shared__ int cnt[256];
  cnt[threadIdx.x] = 0;
  __syncthreads();
  const int base = blockIdx.x * kSortTile;
  for (int i = threadIdx.x; i < kSortTile; i += kSortThreads) {
    const int e = base + i;
    if (e < M) atomicAdd(&cnt[(clamp_token(keys[e], V) >> shift) & 255], 1);
  }
  __syncthreads();
  hist[threadIdx.x * ntiles + blockIdx.x] = cnt[threadIdx.x];
}

// In-place exclusive prefix sum of n ints by one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) exclusive_scan_kernel(int *__restrict__ a, int n) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 4096) {
    const int i0 = base + threadIdx.x * 4;
    int v[4], s = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[k] = i0 + k < n ? a[i0 + k] : 0;
      s += v[k];
    }
    int x = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int t = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[lane] = t;
    }
    __syncthreads();
    int ex = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + x - s;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (i0 + k < n) a[i0 + k] = ex;
      ex += v[k];
    }
    __syncthreads();
    if (threadIdx.x == 1023) carry = ex;
    __syncthreads();
  }
}

// One stable pass: element e of the tile goes to
// base[digit][tile] + (same digits in earlier warps of the tile) + (in earlier rounds / lanes of its warp).
// vals_in == nullptr: the values are the positions themselves.
__global__ void __launch_bounds__(kSortThreads) radix_scatter_kernel(
    const int32_t *__restrict__ keys_in, const int32_t *__restrict__ vals_in, int32_t *__restrict__ keys_out,
    int32_t *__restrict__ vals_out, int M, int V, int shift, const int *__restrict__ base, int ntiles) {
  __shared__ int cnt[kSortThreads / 32][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (kSortThreads / 32) * 256; i += kSortThreads) (&cnt[0][0])[i] = 0;
  __syncthreads();
  const int e0 = blockIdx.x * kSortTile + warp * 128;
  const unsigned lt = (1u << lane) - 1u;
  int dg[4], rk[4], key[4], val[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int e = e0 + r * 32 + lane;
    const bool valid = e < M;
    key[r] = valid ? clamp_token(keys_in[e], V) : 0;
    val[r] = valid ? (vals_in ? vals_in[e] : e) : 0;
    const int d = valid ? ((key[r] >> shift) & 255) : 256;  // 256: no digit (past the end)
    dg[r] = d;
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    const int before = d < 256 ? cnt[warp][d] : 0;
    rk[r] = before + __popc(peers & lt);
    __syncwarp();
    if (d < 256 && lane == __ffs(peers) - 1) cnt[warp][d] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  {  // exclusive scan over the warps, per digit
    const int d = threadIdx.x;
    int run = 0;
#pragma unroll
    for (int w = 0; w < kSortThreads / 32; ++w) {
      const int t = cnt[w][d];
      cnt[w][d] = run;
      run += t;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int d = dg[r];
    if (d < 256) {
      const int pos = base[d * ntiles + blockIdx.x] + cnt[warp][d] + rk[r];
      keys_out[pos] = key[r];
      vals_out[pos] = val[r];
    }
  }
}

// Sort scratch: two key and two value buffers of M ints, 256 * ntiles ints of histogram.
struct TokenSort {
  int32_t *keys[2];
  int32_t *vals[2];
  int *hist;
  // results after sort_tokens(): sorted token ids and their positions
  const int32_t *skey;
  const int32_t *spos;
};

// Launch the radix passes; returns the number of launches.
inline int sort_tokens(const int32_t *tokens, int M, int V, TokenSort &s, cudaStream_t st) {
  const int ntiles = sort_tiles(M), passes = sort_passes(V);
  const int32_t *kin = tokens, *vin = nullptr;
  int launches = 0;
  for (int p = 0; p < passes; ++p) {
    const int shift = 8 * p;
    radix_hist_kernel<<<ntiles, kSortThreads, 0, st>>>(kin, M, V, shift, s.hist, ntiles);
    exclusive_scan_kernel<<<1, 1024, 0, st>>>(s.hist, 256 * ntiles);
    radix_scatter_kernel<<<ntiles, kSortThreads, 0, st>>>(kin, vin, s.keys[p & 1], s.vals[p & 1], M, V, shift,
                                                          s.hist, ntiles);
    kin = s.keys[p & 1];
    vin = s.vals[p & 1];
    launches += 3;
  }
  s.skey = kin;
  s.spos = vin;
  return launches;
}

// ---------------------------------------------------------------------------
// Segmented sum.  flags per chunk: bit 0 the chunk's first run continues a
// segment from the previous chunk (its sum is in head[chunk]), bit 1 that
// run also ends its segment in this chunk, bit 2 the chunk's last run starts
// here and continues into the next chunk (its sum is in tail[chunk]).
constexpr int kSegHead = 1, kSegHeadEnds = 2, kSegTail = 4;

// Store (add != 0: add) the 8*NV-per-lane row sum `acc` (C values) to dst.
template <int NV>
__device__ __forceinline__ void seg_store_row(float *dst, const float (&acc)[NV][8], int C, int lane, int add = 0) {
  const int nv = C >> 3;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = lane + 32 * i;
    if (c < nv) {
      if (add) {
        float o[8];
        Vec8<float>::load(dst + c * 8, o);
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] += acc[i][j];
        Vec8<float>::store(dst + c * 8, o);
      } else {
        Vec8<float>::store(dst + c * 8, acc[i]);
      }
    }
  }
}

// Row sources of the segmented sum: load(row, tok, g, lane) leaves in g
// (8 values per 16-byte unit, units lane, lane + 32, ...) the row whose sum
// over a token's positions is that token's gradient row.
//
// Embedding: for position i with token v,
//   y = wte[v] r0_i,  g_i = r0_i (d_i - y mean(d_i y)),  d_i = dx_i (+ dx2_i)
// the backward of x0 = rmsnorm(wte[tok]) (dx2: a second gradient reaching
// x0, the residual-scalar mixing; may be null).
template <typename T, int NV>
struct EmbedRows {
  const float *dx, *dx2;
  const T *wte;
  const float *r0;
  int C;
  __device__ __forceinline__ void load(int row, int v, float (&g)[NV][8], int lane) const {
    const int nv = C >> 3;
    const float r = r0[row];
    float y[NV][8], dot = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = lane + 32 * i;
#pragma unroll
      for (int j = 0; j < 8; ++j) g[i][j] = y[i][j] = 0.f;
      if (c < nv) {
        Vec8<float>::load(dx + (size_t)row * C + c * 8, g[i]);
        if (dx2) {
          float e[8];
          Vec8<float>::load(dx2 + (size_t)row * C + c * 8, e);
#pragma unroll
          for (int j = 0; j < 8; ++j) g[i][j] += e[j];
        }
        Vec8<T>::load(wte + (size_t)v * C + c * 8, y[i]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          y[i][j] *= r;
          dot += g[i][j] * y[i][j];
        }
      }
    }
    dot = warp_sum(dot) / (float)C;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) g[i][j] = r * (g[i][j] - y[i][j] * dot);
  }
};

// Value embedding: v_i += gate ve[tok_i] in the forward, so the table's
// gradient row of token v is gate * sum of dv_i over its positions; dv_i is
// the 128-wide v part of row i of dqkv (stride ld).
template <typename T>
struct ValueEmbedRows {
  const T *dv;
  int64_t ld;
  const T *gate;
  __device__ __forceinline__ void load(int row, int, float (&g)[1][8], int lane) const {
    const float s = to_f(gate[0]);
#pragma unroll
    for (int j = 0; j < 8; ++j) g[0][j] = 0.f;
    if (lane < kHeadDim / 8) {
      Vec8<T>::load(dv + (size_t)row * ld + lane * 8, g[0]);
#pragma unroll
      for (int j = 0; j < 8; ++j) g[0][j] *= s;
    }
  }
};

// out[v] = sum over token v's positions of src rows (C wide), for every
// token that occurs (accumulate != 0: added to out[v]); rows of other tokens
// are left as they are (the caller zeroes the table first when not
// accumulating).
template <typename Src, int NV>
__global__ void __launch_bounds__(256) segsum_kernel(Src src, const int32_t *__restrict__ skey,
                                                     const int32_t *__restrict__ spos, int M, int C,
                                                     float *__restrict__ out, float *__restrict__ head,
                                                     float *__restrict__ tail, int *__restrict__ flags,
                                                     int accumulate) {
  const int lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int p0 = chunk * kSegChunk;
  if (p0 >= M) return;
  const int p1 = min(M, p0 + kSegChunk);
  float acc[NV][8];
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  int tok = skey[p0], run0 = p0, fl = 0;
  auto emit = [&](int a, int b) {
    const bool starts = a == 0 || skey[a - 1] != tok;
    const bool ends = b == M || skey[b] != tok;
    if (starts && ends) {
      seg_store_row<NV>(out + (size_t)tok * C, acc, C, lane, accumulate);
    } else if (!starts) {  // the chunk's first run, continuing a segment
      seg_store_row<NV>(head + (size_t)chunk * C, acc, C, lane);
      fl |= kSegHead | (ends ? kSegHeadEnds : 0);
    } else {               // the chunk's last run, continuing into the next chunk
      seg_store_row<NV>(tail + (size_t)chunk * C, acc, C, lane);
      fl |= kSegTail;
    }
  };
  for (int p = p0; p < p1; ++p) {
    const int v = skey[p];
    if (v != tok) {
      emit(run0, p);
#pragma unroll
      for (int i = 0; i < NV; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
      run0 = p;
      tok = v;
    }
    float g[NV][8];
    src.load(spos[p], v, g, lane);
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] += g[i][j];
  }
  emit(run0, p1);
  if (lane == 0) flags[chunk] = fl;
}

// A segment that starts in chunk c and continues: tail[c] + head[c+1] + ...
// up to the chunk whose head run ends it.  The 8 warps of the CTA each add
// every 8th head partial (warp w: chunks c+1+w, c+9+w, ... in order), then
// the partials meet in a fixed order (tail, warp 0, ..., warp 7): the same
// sum on every run, with a chain 8 times shorter than one warp's.
constexpr int kFixCols = 256;  // float4 columns per pass
__global__ void __launch_bounds__(256) seg_fixup_kernel(const int32_t *__restrict__ skey, int M, int C,
                                                        const float *__restrict__ head,
                                                        const float *__restrict__ tail,
                                                        const int *__restrict__ flags, int nchunks,
                                                        float *__restrict__ out, int accumulate) {
  __shared__ float4 part[8][kFixCols];
  const int c = blockIdx.x;
  if (!(flags[c] & kSegTail)) return;
  const int tok = skey[min(M, (c + 1) * kSegChunk) - 1];
  int last = c + 1;
  while (last < nchunks - 1 && !(flags[last] & kSegHeadEnds)) ++last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C4 = C / 4;
  for (int q0 = 0; q0 < C4; q0 += kFixCols) {
    float4 acc[kFixCols / 32];
#pragma unroll
    for (int i = 0; i < kFixCols / 32; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = c + 1 + warp; k <= last; k += 8) {
      const float4 *hk = reinterpret_cast<const float4 *>(head + (size_t)k * C) + q0;
#pragma unroll
      for (int i = 0; i < kFixCols / 32; ++i) {
        const int q = lane + 32 * i;
        if (q0 + q < C4) {
          const float4 h = hk[q];
          acc[i].x += h.x; acc[i].y += h.y; acc[i].z += h.z; acc[i].w += h.w;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kFixCols / 32; ++i) part[warp][lane + 32 * i] = acc[i];
    __syncthreads();
    const int q = q0 + (int)threadIdx.x;
    if (threadIdx.x < kFixCols && q < C4) {
      float4 a = reinterpret_cast<const float4 *>(tail + (size_t)c * C)[q];
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float4 h = part[w][threadIdx.x];
        a.x += h.x; a.y += h.y; a.z += h.z; a.w += h.w;
      }
      float4 *o = reinterpret_cast<float4 *>(out + (size_t)tok * C) + q;
      if (accumulate) {
        const float4 bb = *o;
        a.x += bb.x; a.y += bb.y; a.z += bb.z; a.w += bb.w;
      }
      *o = a;
    }
    __syncthreads();
  }
}

// Deterministic sum of n partial values by one CTA: each thread adds a
// fixed strided subset in order, then a fixed tree; *out = scale * sum
// (accumulate != 0: *out += scale * sum).
__global__ void __launch_bounds__(1024) ordered_sum_kernel(const float *__restrict__ partial, int n, float scale,
                                                           float *__restrict__ out, int accumulate) {
  __shared__ float sh[32];
  float s = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += partial[i];
  s = block_sum(s, sh);
  if (threadIdx.x == 0) *out = scale * s + (accumulate ? *out : 0.f);
}

}  // namespace nc
