// General-dimension CUDA-core kernels of the TurboQuant hot path.
//
// These handle every supported (d, b) with plain fp32 FFMA arithmetic and are
// the path for shapes the tensor-core kernels do not specialise.  They also
// serve the small, launch-bound cases (a few thousand vectors, one token per
// kv-head) where a tensor-core pipeline would not fill.
//
// Pages:
//   [ttakun]  "KV缓存52GB瞬间爆内存？TurboQuant随机旋转+标量量化如何把LLM长上下文推理成本
//             砍到1/16且失真逼近理论极限" (ttakun.com/news/45354)
//   [tmdm]    "谷歌悄悄扔下一颗“性能核弹”：KV缓存压缩6倍，推理提速8倍，还不用重训模型"
//   [tq.net]  turboquant.net/zh, "TurboQuant 最近的进展和外溢影响"
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cfloat>

#include "tq_internal.h"

namespace tqi {
namespace {

constexpr float kSqrtHalfPi = 1.2533141373155003f;  // sqrt(pi/2)

__device__ __forceinline__ float load_elem(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

// index of coordinate j in a packed code row (layout documented in tq.h)
__device__ __forceinline__ int code_at(const uint32_t* w, int bm, int j) {
  const int g = j >> 5, i = j & 31;
  const uint32_t* p = w + g * bm;
  switch (bm) {
    case 1:
      return (p[0] >> i) & 1u;
    case 2:
      return (p[i >> 4] >> (2 * (i & 15))) & 3u;
    case 3:
      if (i < 24) return (p[i >> 3] >> (4 * (i & 7))) & 7u;
      {
        const int s = 4 * (i - 24) + 3;
        return ((p[0] >> s) & 1u) | (((p[1] >> s) & 1u) << 1) | (((p[2] >> s) & 1u) << 2);
      }
    default:
      return (p[i >> 3] >> (4 * (i & 7))) & 15u;
  }
}

// word k of group g of a code row, from per-coordinate indices in shared memory
__device__ __forceinline__ uint32_t pack_word(const uint8_t* idx, int d, int bm, int g, int k) {
  const int base = 32 * g;
  auto at = [&](int i) -> uint32_t { return (base + i < d) ? idx[base + i] : 0u; };
  uint32_t w = 0;
  switch (bm) {
    case 1:
      for (int i = 0; i < 32; ++i) w |= at(i) << i;
      break;
    case 2:
      for (int j = 0; j < 16; ++j) w |= at(16 * k + j) << (2 * j);
      break;
    case 3:
      for (int j = 0; j < 8; ++j) w |= at(8 * k + j) << (4 * j);
      for (int j = 0; j < 8; ++j) w |= ((at(24 + j) >> k) & 1u) << (4 * j + 3);
      break;
    default:
      for (int j = 0; j < 8; ++j) w |= at(8 * k + j) << (4 * j);
      break;
  }
  return w;
}

__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
  return s;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = -FLT_MAX;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s = fmaxf(s, red[w]);
  return s;
}

struct QuantArgs {
  const void* x;
  const int32_t* channels;  // optional: coordinate i reads x[channels[i]]
  int64_t N, x_stride, out_stride;
  int d, bm, prod;
  const float* PiT;  // [i][j] = Pi[j][i]
  const float* TT;   // [i][j] = T[j][i], T = S Pi^T
  const float* centroids;
  const float* thresholds;
  uint32_t* codes;
  uint32_t* signs;
  float* norms;
  float* rnorms;
};

// One CTA per vector (grid-stride).  Shared: x[d], y[d], u[d], idx[d].
// Steps: n = ||x||; y = Pi x (fp32 FFMA); idx_j = #{k : y_j >= n t_k};
// pack; for prod: u = y/n - c[idx], v = T u, sign bits, rn = n ||u||.
template <typename TIn>
__global__ void __launch_bounds__(128) quant_simple_kernel(QuantArgs a) {
  extern __shared__ float sm[];
  const int d = a.d;
  float* xs = sm;
  float* ys = sm + d;
  float* us = sm + 2 * d;
  __shared__ float red[32];
  __shared__ float thr[16];
  uint8_t* sidx = reinterpret_cast<uint8_t*>(sm + 3 * d);
  const int K = 1 << a.bm;
  const int G = (d + 31) >> 5;
  const int words = G * a.bm;
  const TIn* x = static_cast<const TIn*>(a.x);
  for (int64_t v = blockIdx.x; v < a.N; v += gridDim.x) {
    float ss = 0.f;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      float e = load_elem(x, v * a.x_stride + (a.channels ? a.channels[i] : i));
      xs[i] = e;
      ss += e * e;
    }
    const float n = sqrtf(block_sum(ss, red));  // block_sum syncs: xs visible
    if (threadIdx.x < K - 1) thr[threadIdx.x] = n * a.thresholds[threadIdx.x];
    // the loads of Pi^T are independent of the FMA chain: a deep unroll keeps
    // many of them in flight (a small batch, e.g. one appended token per head,
    // is bound by their latency)
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
      float acc = 0.f;
#pragma unroll 16
      for (int i = 0; i < d; ++i) acc = fmaf(a.PiT[(int64_t)i * d + j], xs[i], acc);
      ys[j] = acc;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
      const float y = ys[j];
      int idx = 0;
      for (int k = 0; k < K - 1; ++k) idx += (y >= thr[k]) ? 1 : 0;
      sidx[j] = (uint8_t)idx;
      if (a.prod) us[j] = (n > 0.f) ? (y / n - a.centroids[idx]) : 0.f;
    }
    __syncthreads();
    const int64_t slot = v * a.out_stride;
    for (int w = threadIdx.x; w < words; w += blockDim.x)
      a.codes[slot * words + w] = pack_word(sidx, d, a.bm, w / a.bm, w % a.bm);
    if (threadIdx.x == 0) a.norms[slot] = n;
    if (a.prod) {
      float uu = 0.f;
      for (int j = threadIdx.x; j < d; j += blockDim.x) uu += us[j] * us[j];
      const float un = sqrtf(block_sum(uu, red));
      // reuse sidx as the sign-bit array
      __syncthreads();
      for (int j = threadIdx.x; j < d; j += blockDim.x) {
        float acc = 0.f;
#pragma unroll 16
        for (int i = 0; i < d; ++i) acc = fmaf(a.TT[(int64_t)i * d + j], us[i], acc);
        sidx[j] = (acc >= 0.f) ? 1 : 0;
      }
      __syncthreads();
      for (int w = threadIdx.x; w < G; w += blockDim.x)
        a.signs[slot * G + w] = pack_word(sidx, d, 1, w, 0);
      if (threadIdx.x == 0) a.rnorms[slot] = n * un;
    }
    __syncthreads();
  }
}

// Small batches (one arriving token per kv-head): one launch quantizes every
// channel group of every vector, CTA (vector, group), 256 threads.  Each
// mat-vec (Pi x, then T u) splits the input coordinates into 256 / d parts
// whose partial sums meet in shared memory, so a thread's dependent FMA chain
// is d^2 / 256 long instead of d; the norm is summed in float64.
struct SmallGroup {
  const float* PiT;          // [i][j] = Pi[j][i]
  const float* TT;           // [i][j] = T[j][i]
  const float* centroids;
  const float* thresholds;
  const int32_t* channels;   // [d] channels of the input row
  uint32_t* codes;
  uint32_t* signs;
  float* norms;
  float* rnorms;
  int d, bm, prod;
};

struct SmallArgs {
  const void* x;
  int64_t N, x_stride, out_stride;
  SmallGroup g[2];
};

template <typename TIn>
__global__ void __launch_bounds__(256) quant_small_kernel(SmallArgs a) {
  const SmallGroup& G = a.g[blockIdx.y];
  const int64_t v = blockIdx.x;
  const int d = G.d, t = threadIdx.x;
  __shared__ float xs[256], ys[256], us[256], part[256];
  __shared__ uint8_t sidx[256];
  __shared__ double redd[8];
  __shared__ float red[8];
  __shared__ float thr[16];
  const int parts = 256 / d;            // d <= 256
  const int j = t % d, p = t / d;       // output coordinate and input part of this thread
  const int i0 = p * d / parts, i1 = (p + 1) * d / parts;
  const TIn* x = static_cast<const TIn*>(a.x) + v * a.x_stride;
  double ss = 0.0;
  if (t < d) {
    const float e = load_elem(x, G.channels ? G.channels[t] : t);
    xs[t] = e;
    ss = (double)e * e;
  }
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((t & 31) == 0) redd[t >> 5] = ss;
  __syncthreads();
  double tot = 0.0;
  for (int w = 0; w < 8; ++w) tot += redd[w];
  const float n = (float)sqrt(tot);
  const int K = 1 << G.bm;
  if (t < K - 1) thr[t] = n * G.thresholds[t];
  // y = Pi x, split over the input coordinates
  float acc = 0.f;
  if (p < parts) {
#pragma unroll 8
    for (int i = i0; i < i1; ++i) acc = fmaf(G.PiT[(int64_t)i * d + j], xs[i], acc);
  }
  part[t] = acc;
  __syncthreads();
  const int64_t slot = v * a.out_stride;
  if (t < d) {
    float y = 0.f;
    for (int q = 0; q < parts; ++q) y += part[q * d + t];
    int idx = 0;
    for (int k = 0; k < K - 1; ++k) idx += (y >= thr[k]) ? 1 : 0;
    sidx[t] = (uint8_t)idx;
    us[t] = (G.prod && n > 0.f) ? (y / n - G.centroids[idx]) : 0.f;
  }
  __syncthreads();
  const int Gw = (d + 31) >> 5, words = Gw * G.bm;
  if (t < words) G.codes[slot * words + t] = pack_word(sidx, d, G.bm, t / G.bm, t % G.bm);
  if (t == 0) G.norms[slot] = n;
  if (!G.prod) return;
  float uu = t < d ? us[t] * us[t] : 0.f;
  for (int o = 16; o > 0; o >>= 1) uu += __shfl_xor_sync(0xffffffffu, uu, o);
  if ((t & 31) == 0) red[t >> 5] = uu;
  // V = T u, split the same way
  acc = 0.f;
  if (p < parts) {
#pragma unroll 8
    for (int i = i0; i < i1; ++i) acc = fmaf(G.TT[(int64_t)i * d + j], us[i], acc);
  }
  part[t] = acc;
  __syncthreads();
  if (t < d) {
    float vv = 0.f;
    for (int q = 0; q < parts; ++q) vv += part[q * d + t];
    sidx[t] = vv >= 0.f ? 1 : 0;
  }
  __syncthreads();
  if (t < Gw) G.signs[slot * Gw + t] = pack_word(sidx, d, 1, t, 0);
  if (t == 0) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += red[w];
    G.rnorms[slot] = n * sqrtf(s);
  }
}

// One CTA per vector: y_hat_j = c[idx_j] (shared), x_hat_i = n sum_j Pi[j][i] y_hat_j.
template <typename TOut>
__global__ void __launch_bounds__(128) dequant_simple_kernel(const uint32_t* codes, const float* norms,
                                                             int64_t N, int d, int bm,
                                                             const float* Pi, const float* centroids,
                                                             TOut* out) {
  extern __shared__ float yh[];
  const int words = ((d + 31) >> 5) * bm;
  for (int64_t v = blockIdx.x; v < N; v += gridDim.x) {
    const uint32_t* w = codes + v * words;
    for (int j = threadIdx.x; j < d; j += blockDim.x) yh[j] = centroids[code_at(w, bm, j)];
    __syncthreads();
    const float n = norms[v];
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      float acc = 0.f;
      for (int j = 0; j < d; ++j) acc = fmaf(Pi[(int64_t)j * d + i], yh[j], acc);
      if constexpr (sizeof(TOut) == 4)
        out[v * d + i] = n * acc;
      else
        out[v * d + i] = __float2bfloat16_rn(n * acc);
    }
    __syncthreads();
  }
}

// q' = Pi q and q'' = S q, one warp per output coordinate (coalesced row reads).
template <typename TIn>
__global__ void query_prep_kernel(const TIn* q, int64_t nq, int d, const float* Pi, const float* S,
                                  float* qrot, float* qproj) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t total = nq * d * (S ? 2 : 1);
  for (int64_t w = warp; w < total; w += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int which = (int)(w / (nq * d));
    const int64_t r = w % (nq * d);
    const int64_t qi = r / d;
    const int j = (int)(r % d);
    const float* M = which ? S : Pi;
    float acc = 0.f;
    for (int i = lane; i < d; i += 32) acc = fmaf(M[(int64_t)j * d + i], load_elem(q, qi * d + i), acc);
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) (which ? qproj : qrot)[qi * d + j] = acc;
  }
}

// One thread per (query, key): est = n <q', c[idx]> + rn sqrt(pi/2)/d <q'', sigma>.
// q' = Pi q and q'' = S q as a tiled fp32 product (d <= 256, d % 4 == 0): a
// block takes one matrix and one chunk of 128 output coordinates (blockIdx.y =
// matrix * chunks + chunk), keeps that chunk of M^T in shared memory and loops
// over tiles of 32 query rows; thread (ty, tx) accumulates rows 4 ty .. + 3 x
// outputs 4 tx .. + 3 of the chunk, summing over the input coordinate in order.
constexpr int kQpRows = 32;
constexpr int kQpLd = 132;   // padded row length (floats) of the transposed matrix chunk

inline int qp_smem_bytes(int d) { return (d * kQpLd + kQpRows * (d + 4)) * 4; }

template <typename TIn>
__global__ void __launch_bounds__(256) query_prep_tiled_kernel(const TIn* q, int64_t nq, int d, int chunks,
                                                               const float* Pi, const float* S, float* qrot,
                                                               float* qproj) {
  extern __shared__ __align__(16) float qp_smem[];
  const int ld = d + 4;                  // row length of the query tile
  float* mt = qp_smem;                   // [i][jj] = M[c0 + jj][i]
  float* qs = qp_smem + d * kQpLd;       // [row][i]
  const int which = (int)blockIdx.y / chunks, c0 = ((int)blockIdx.y % chunks) * 128;
  const float* M = which ? S : Pi;
  float* out = which ? qproj : qrot;
  for (int e = threadIdx.x; e < 128 * d; e += 256) {
    const int jj = e / d, i = e - jj * d;
    mt[i * kQpLd + jj] = c0 + jj < d ? M[(int64_t)(c0 + jj) * d + i] : 0.f;
  }
  const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
  const bool col_ok = c0 + 4 * tx < d;
  const int64_t tiles = (nq + kQpRows - 1) / kQpRows;
  for (int64_t rt = blockIdx.x; rt < tiles; rt += gridDim.x) {
    const int64_t r0 = rt * kQpRows;
    __syncthreads();
    for (int e = threadIdx.x; e < kQpRows * d; e += 256) {
      const int rr = e / d, i = e - rr * d;
      const int64_t row = r0 + rr;
      qs[rr * ld + i] = row < nq ? load_elem(q, row * d + i) : 0.f;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 2
    for (int i = 0; i < d; i += 4) {
      float4 xa[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) xa[r] = *reinterpret_cast<const float4*>(qs + (4 * ty + r) * ld + i);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 mb = *reinterpret_cast<const float4*>(mt + (i + k) * kQpLd + 4 * tx);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float x = k == 0 ? xa[r].x : k == 1 ? xa[r].y : k == 2 ? xa[r].z : xa[r].w;
          acc[r][0] = fmaf(mb.x, x, acc[r][0]);
          acc[r][1] = fmaf(mb.y, x, acc[r][1]);
          acc[r][2] = fmaf(mb.z, x, acc[r][2]);
          acc[r][3] = fmaf(mb.w, x, acc[r][3]);
        }
      }
    }
    if (col_ok)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int64_t row = r0 + 4 * ty + r;
        if (row < nq)
          *reinterpret_cast<float4*>(out + row * d + c0 + 4 * tx) =
              make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
      }
  }
}

__global__ void scores_simple_kernel(const float* qrot, const float* qproj, int64_t nq,
                                     const uint32_t* codes, const uint32_t* signs,
                                     const float* norms, const float* rnorms, int64_t N, int d,
                                     int bm, int prod, const float* centroids, float* scores) {
  const int words = ((d + 31) >> 5) * bm;
  const int G = (d + 31) >> 5;
  for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < nq * N;
       p += (int64_t)gridDim.x * blockDim.x) {
    const int64_t qi = p / N, k = p % N;
    const float* qr = qrot + qi * d;
    const uint32_t* w = codes + k * words;
    float mse = 0.f;
    for (int j = 0; j < d; ++j) mse = fmaf(qr[j], centroids[code_at(w, bm, j)], mse);
    float est = norms[k] * mse;
    if (prod) {
      const float* qp = qproj + qi * d;
      const uint32_t* s = signs + k * G;
      float qjl = 0.f;
      for (int j = 0; j < d; ++j) qjl += ((s[j >> 5] >> (j & 31)) & 1u) ? qp[j] : -qp[j];
      est = fmaf(rnorms[k] * (kSqrtHalfPi / d), qjl, est);
    }
    scores[qi * N + k] = est;
  }
}

// Top-k per query, one CTA per query: k rounds of a block-wide arg-max with
// exclusion of the winners so far (ties: lower index).  For modest N only.
__global__ void topk_simple_kernel(const float* scores, int64_t N, int k, int32_t* top_idx,
                                   float* top_val) {
  __shared__ float sv[32];
  __shared__ long long si[32];
  __shared__ long long chosen[TQ_MAX_TOPK];
  const int64_t qi = blockIdx.x;
  const float* s = scores + qi * N;
  for (int r = 0; r < k; ++r) {
    float best = -FLT_MAX;
    long long bi = LLONG_MAX;
    for (int64_t i = threadIdx.x; i < N; i += blockDim.x) {
      bool taken = false;
      for (int c = 0; c < r; ++c) taken |= (chosen[c] == i);
      if (taken) continue;
      float v = s[i];
      if (v > best || (v == best && i < bi)) best = v, bi = i;
    }
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, best, o);
      long long oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > best || (ov == best && oi < bi)) best = ov, bi = oi;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sv[warp] = best, si[warp] = bi;
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
        if (sv[w] > sv[0] || (sv[w] == sv[0] && si[w] < si[0])) sv[0] = sv[w], si[0] = si[w];
      chosen[r] = si[0];
      top_idx[qi * k + r] = (int32_t)si[0];
      top_val[qi * k + r] = sv[0];
    }
    __syncthreads();
  }
}

// Decode attention, split over the context.  CTA (split, q-head, batch):
// logits of a chunk of keys (one per thread), online max/sum, then the value
// sum acc_j += p_t n_t c_V[idx_tj] in the rotated frame (one coordinate per
// thread).  Writes partial (m, l, acc[d]) for the merge kernel.
struct DecodeArgs {
  const float* qrot;
  const float* qproj;
  int B, Hq, Hkv, d, bk, bv, splits;
  int64_t T, kv_stride;
  const uint32_t* kcodes;
  const uint32_t* ksigns;
  const float* knorms;
  const float* krnorms;
  const uint32_t* vcodes;
  const float* vnorms;
  const float* kcent;
  const float* vcent;
  float scale;
  float* partials;  // [B][Hq][splits][d + 2]
  PagedCache pg;    // page > 0: rows through the block table; rn16: fp16 residual norms
};

__device__ __forceinline__ int64_t dec_row(const DecodeArgs& a, int64_t bh, int64_t t) {
  if (a.pg.page == 0) return bh * a.kv_stride + t;
  return (int64_t)a.pg.block_table[bh * a.pg.max_pages + t / a.pg.page] * a.pg.page + t % a.pg.page;
}

__global__ void __launch_bounds__(128) decode_split_simple_kernel(DecodeArgs a) {
  extern __shared__ float sm[];
  const int d = a.d;
  float* qr = sm;            // [d]
  float* qp = sm + d;        // [d]
  float* pw = sm + 2 * d;    // [blockDim] weights p_t * n_t of the chunk
  __shared__ float red[32];
  __shared__ int64_t prow[128];  // cache rows of the chunk
  const int split = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int h = hq / (a.Hq / a.Hkv);
  const int64_t q_off = ((int64_t)b * a.Hq + hq) * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) qr[j] = a.qrot[q_off + j], qp[j] = a.qproj[q_off + j];
  const int64_t per = (a.T + a.splits - 1) / a.splits;
  const int64_t t0 = split * per, t1 = min(a.T, t0 + per);
  const int64_t bh = (int64_t)b * a.Hkv + h;
  const int kw = ((d + 31) >> 5) * a.bk, vw = ((d + 31) >> 5) * a.bv, G = (d + 31) >> 5;
  float m = -FLT_MAX, l = 0.f;
  float acc[TQ_MAX_DIM / 128];
  for (int r = 0; r < TQ_MAX_DIM / 128; ++r) acc[r] = 0.f;
  __syncthreads();
  for (int64_t c0 = t0; c0 < t1; c0 += blockDim.x) {
    const int64_t t = c0 + threadIdx.x;
    float logit = -FLT_MAX;
    const int64_t row = t < t1 ? dec_row(a, bh, t) : 0;
    if (t < t1) {
      const uint32_t* w = a.kcodes + row * kw;
      const uint32_t* s = a.ksigns + row * G;
      float mse = 0.f, qjl = 0.f;
      for (int j = 0; j < d; ++j) {
        mse = fmaf(qr[j], a.kcent[code_at(w, a.bk, j)], mse);
        qjl += ((s[j >> 5] >> (j & 31)) & 1u) ? qp[j] : -qp[j];
      }
      const float rn = a.pg.rn16 ? __half2float(reinterpret_cast<const __half*>(a.krnorms)[row]) : a.krnorms[row];
      logit = a.scale * (a.knorms[row] * mse + rn * (kSqrtHalfPi / d) * qjl);
    }
    const float cm = block_max(logit, red);
    const float mn = fmaxf(m, cm);
    const float p = (t < t1) ? __expf(logit - mn) : 0.f;
    const float cs = block_sum(p, red);
    const float corr = __expf(m - mn);
    l = l * corr + cs;
    m = mn;
    pw[threadIdx.x] = (t < t1) ? p * a.vnorms[row] : 0.f;
    if (t < t1) prow[threadIdx.x] = row;
    __syncthreads();
    const int cnt = (int)min((int64_t)blockDim.x, t1 - c0);
    for (int r = 0, j = threadIdx.x; j < d; ++r, j += blockDim.x) {
      float s = acc[r] * corr;
      for (int i = 0; i < cnt; ++i) {
        const uint32_t* w = a.vcodes + prow[i] * vw;
        s = fmaf(pw[i], a.vcent[code_at(w, a.bv, j)], s);
      }
      acc[r] = s;
    }
    __syncthreads();
  }
  float* out = a.partials + (((int64_t)b * a.Hq + hq) * a.splits + split) * (d + 2);
  for (int r = 0, j = threadIdx.x; j < d; ++r, j += blockDim.x) out[j] = acc[r];
  if (threadIdx.x == 0) out[d] = m, out[d + 1] = l;
}

// Merge the splits with the log-sum-exp rescale, divide by the sum, rotate back
// once: out = Pi_V^T (acc / l).  One CTA per (batch, q-head).  Split s of row
// bh is the (acc[d], m, l) record at partials + bh * row_stride + s * split_stride.
// With partial_out the merged record itself (sum_s acc_s e^(m_s - M), M,
// sum_s l_s e^(m_s - M)), still in the rotated frame, goes to out[bh][d + 2].
__global__ void __launch_bounds__(128) decode_merge_kernel(const float* partials, int splits, int64_t split_stride,
                                                           int64_t row_stride, int d, const float* PiV, float* out,
                                                           int partial_out) {
  extern __shared__ float orot[];
  const int64_t bh = blockIdx.x;
  const float* P = partials + bh * row_stride;
  float M = -FLT_MAX;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, P[s * split_stride + d]);
  float L = 0.f;
  for (int s = 0; s < splits; ++s) L += P[s * split_stride + d + 1] * __expf(P[s * split_stride + d] - M);
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < splits; ++s) a += P[s * split_stride + j] * __expf(P[s * split_stride + d] - M);
    orot[j] = partial_out ? a : a / L;
  }
  if (partial_out) {
    float* o = out + bh * (d + 2);
    for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = orot[j];
    if (threadIdx.x == 0) o[d] = M, o[d + 1] = L;
    return;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float a = 0.f;
    for (int j = 0; j < d; ++j) a = fmaf(PiV[(int64_t)j * d + i], orot[j], a);
    out[bh * d + i] = a;
  }
}

int grid_for(int64_t n, int cap) { return (int)((n < cap) ? (n > 0 ? n : 1) : cap); }

}  // namespace

int launch_quant_small(const tq_ctx* const* h, int ngroups, const void* x, int dtype, int64_t N, int64_t x_stride,
                       const int32_t* channels, uint32_t* const* codes, uint32_t* const* signs, float* const* norms,
                       float* const* rnorms, int64_t out_stride, void* stream) {
  SmallArgs a;
  a.x = x;
  a.N = N;
  a.x_stride = x_stride;
  a.out_stride = out_stride;
  int off = 0;
  for (int g = 0; g < ngroups; ++g) {
    const tq_ctx* hg = h[g];
    const bool prod = hg->variant == TQ_PROD;
    a.g[g] = SmallGroup{hg->dev.PiT, hg->dev.TT, hg->dev.centroids, hg->dev.thresholds,
                        channels ? channels + off : nullptr, codes[g], prod ? signs[g] : nullptr, norms[g],
                        prod ? rnorms[g] : nullptr, hg->d, hg->bm, prod ? 1 : 0};
    off += hg->d;
  }
  const dim3 grid((unsigned)N, (unsigned)ngroups);
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == TQ_BF16)
    quant_small_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a);
  else
    quant_small_kernel<float><<<grid, 256, 0, s>>>(a);
  return (int)cudaGetLastError();
}

int launch_quant_simple(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride,
                        uint32_t* codes, uint32_t* signs, float* norms, float* rnorms,
                        int64_t out_stride, void* stream, const int32_t* channels) {
  QuantArgs a{x, channels, N, x_stride, out_stride, h->d, h->bm, h->variant == TQ_PROD, h->dev.PiT,
              h->dev.TT, h->dev.centroids, h->dev.thresholds, codes, signs, norms, rnorms};
  const size_t smem = 3 * (size_t)h->d * sizeof(float) + h->d;
  const int grid = grid_for(N, h->sm_count * 16);
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == TQ_BF16)
    quant_simple_kernel<__nv_bfloat16><<<grid, 128, smem, s>>>(a);
  else
    quant_simple_kernel<float><<<grid, 128, smem, s>>>(a);
  return (int)cudaGetLastError();
}

int launch_dequant_simple(const tq_ctx* h, const uint32_t* codes, const float* norms, int64_t N,
                          void* out, int out_dtype, void* stream) {
  const int grid = grid_for(N, h->sm_count * 16);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t smem = (size_t)h->d * sizeof(float);
  if (out_dtype == TQ_BF16)
    dequant_simple_kernel<<<grid, 128, smem, s>>>(codes, norms, N, h->d, h->bm, h->dev.Pi,
                                                  h->dev.centroids, (__nv_bfloat16*)out);
  else
    dequant_simple_kernel<<<grid, 128, smem, s>>>(codes, norms, N, h->d, h->bm, h->dev.Pi,
                                                  h->dev.centroids, (float*)out);
  return (int)cudaGetLastError();
}

int launch_query_prep(const tq_ctx* h, const float* q, int q_dtype, int64_t nq, float* qrot,
                      float* qproj, void* stream) {
  const int64_t warps = nq * h->d * (qproj ? 2 : 1);
  const int grid = grid_for((warps * 32 + 255) / 256, h->sm_count * 32);
  const float* S = qproj ? h->dev.S : nullptr;
  cudaStream_t s = (cudaStream_t)stream;
  const bool out16 = ((reinterpret_cast<uintptr_t>(qrot) | reinterpret_cast<uintptr_t>(qproj)) & 15u) == 0;
  // the tiled product pays a copy of the matrix into shared memory per block; a few hundred query rows (a decode
  // step) finish sooner one warp per output
  if (h->d <= 256 && h->d % 4 == 0 && nq >= 1024 && out16) {
    const void* kern = q_dtype == TQ_BF16 ? (const void*)query_prep_tiled_kernel<__nv_bfloat16>
                                          : (const void*)query_prep_tiled_kernel<float>;
    const int smem = qp_smem_bytes(h->d);
    if (int e = ensure_dyn_smem(kern, smem)) return e;
    const int chunks = (h->d + 127) / 128;
    const int ys = chunks * (qproj ? 2 : 1);
    const int64_t tiles = (nq + kQpRows - 1) / kQpRows;
    const int64_t xs = std::max<int64_t>(1, std::min<int64_t>(tiles, 2 * (int64_t)h->sm_count / ys));
    const dim3 grid2((unsigned)xs, (unsigned)ys);
    if (q_dtype == TQ_BF16)
      query_prep_tiled_kernel<<<grid2, 256, smem, s>>>((const __nv_bfloat16*)q, nq, h->d, chunks, h->dev.Pi, S,
                                                       qrot, qproj);
    else
      query_prep_tiled_kernel<<<grid2, 256, smem, s>>>(q, nq, h->d, chunks, h->dev.Pi, S, qrot, qproj);
    return (int)cudaGetLastError();
  }
  if (q_dtype == TQ_BF16)
    query_prep_kernel<<<grid, 256, 0, s>>>((const __nv_bfloat16*)q, nq, h->d, h->dev.Pi, S, qrot, qproj);
  else
    query_prep_kernel<<<grid, 256, 0, s>>>(q, nq, h->d, h->dev.Pi, S, qrot, qproj);
  return (int)cudaGetLastError();
}

int launch_scores_simple(const tq_ctx* h, const float* qrot, const float* qproj, int64_t nq,
                         const uint32_t* codes, const uint32_t* signs, const float* norms,
                         const float* rnorms, int64_t N, float* scores, void* stream) {
  const int grid = grid_for((nq * N + 255) / 256, h->sm_count * 32);
  scores_simple_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(
      qrot, qproj, nq, codes, signs, norms, rnorms, N, h->d, h->bm, h->variant == TQ_PROD,
      h->dev.centroids, scores);
  return (int)cudaGetLastError();
}

int launch_topk_simple(const float* scores, int64_t nq, int64_t N, int k, int32_t* top_idx,
                       float* top_val, void* stream) {
  topk_simple_kernel<<<(unsigned)nq, 256, 0, (cudaStream_t)stream>>>(scores, N, k, top_idx, top_val);
  return (int)cudaGetLastError();
}

int launch_decode_simple(const tq_ctx* hk, const tq_ctx* hv, const float* qrot,
                         const float* qproj, int B, int Hq, int Hkv, int64_t T, int64_t kv_stride,
                         const uint32_t* kcodes, const uint32_t* ksigns, const float* knorms,
                         const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                         float scale, int splits, float* partials, float* out, void* stream, int partial_out,
                         PagedCache pg) {
  DecodeArgs a{qrot, qproj, B, Hq, Hkv, hk->d, hk->bm, hv->bm, splits, T, kv_stride, kcodes,
               ksigns, knorms, krnorms, vcodes, vnorms, hk->dev.centroids, hv->dev.centroids,
               scale, partials, pg};
  cudaStream_t s = (cudaStream_t)stream;
  const size_t smem = (2 * (size_t)hk->d + 128) * sizeof(float);
  decode_split_simple_kernel<<<dim3(splits, Hq, B), 128, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  return launch_decode_merge(partials, (int64_t)B * Hq, splits, hv, out, stream, hv->d + 2,
                             (int64_t)splits * (hv->d + 2), partial_out);
}

int launch_decode_merge(const float* partials, int64_t BH, int splits, const tq_ctx* hv, float* out, void* stream,
                        int64_t split_stride, int64_t row_stride, int partial_out) {
  decode_merge_kernel<<<(unsigned)BH, 128, hv->d * sizeof(float), (cudaStream_t)stream>>>(
      partials, splits, split_stride, row_stride, hv->d, hv->dev.Pi, out, partial_out);
  return (int)cudaGetLastError();
}

}  // namespace tqi
