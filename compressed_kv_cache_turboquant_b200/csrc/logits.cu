// Attention logits over a TurboQuant_prod key cache split into channel groups,
// and channel-gathered quantization for appending tokens to such a cache.
//
// Pages: turboquant.net/zh ("TurboQuant 最近的进展和外溢影响"): ordinary channels at
// very low bit width, outlier channels kept separately at higher precision;
// ttakun.com/news/45354 ("KV缓存52GB瞬间爆内存？…", 为什么TurboQuant…): 3.5 bits per
// channel, and quantizing each token as it arrives ("来一个token压一个token").
//
// A key is stored as independent TurboQuant_prod instances over disjoint
// channel groups (for example 64 outlier channels at 4 bits and 64 channels at
// 3 bits).  Its estimated inner product with a query is the sum of the groups'
// estimates, each group scoring the query restricted to its channels.
//
// logits_kernel: one thread per token, 4 query heads per kv-head (grouped-query
// attention).  Per group and coordinate: the index is cut out of the packed
// word, its centroid comes from a small shared table, and the four heads'
// rotated query values come as one broadcast 16-byte shared load.  The QJL part
// sums the projected query over the set sign bits: <q'', s> = 2 sum_{bit=1} q'' - sum q''.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tq_internal.h"

namespace tqi {
namespace {

constexpr float kSqrtHalfPi = 1.2533141373155003f;

template <int BM>
__device__ __forceinline__ uint32_t idx_at(const uint32_t* w, int j) {
  const int g = j >> 5, i = j & 31;
  const uint32_t* p = w + g * BM;
  if constexpr (BM == 1) return (p[0] >> i) & 1u;
  else if constexpr (BM == 2) return (p[i >> 4] >> (2 * (i & 15))) & 3u;
  else if constexpr (BM == 4) return (p[i >> 3] >> (4 * (i & 7))) & 15u;
  else {
    if (i < 24) return (p[i >> 3] >> (4 * (i & 7))) & 7u;
    const int s = 4 * (i - 24) + 3;
    return ((p[0] >> s) & 1u) | (((p[1] >> s) & 1u) << 1) | (((p[2] >> s) & 1u) << 2);
  }
}

struct GroupPtrs {
  const uint32_t* codes;
  const uint32_t* signs;
  const float* norms;
  const float* rnorms;
  const float* qrot;   // [B*Hq][d_g]
  const float* qproj;  // [B*Hq][d_g]
  const float* cent;   // [2^bm]
};

struct LogitsArgs {
  GroupPtrs g[2];
  int B, Hq, Hkv;
  int64_t T, kv_stride;
  float scale;
  float* logits;  // [B][Hq][T]
};

template <int D, int BM>
__device__ __forceinline__ void group_scores(const GroupPtrs& gp, int64_t row, const float4* qm, const float4* qq,
                                             const float* ct, const float4& qtot, float (&est)[4]) {
  constexpr int W = (D / 32) * BM, SW = D / 32;
  uint32_t w[W], s[SW];
#pragma unroll
  for (int k = 0; k < W; ++k) w[k] = gp.codes[row * W + k];
#pragma unroll
  for (int k = 0; k < SW; ++k) s[k] = gp.signs[row * SW + k];
  float am[4] = {0.f, 0.f, 0.f, 0.f}, aq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < D; ++j) {
    const float c = ct[idx_at<BM>(w, j)];
    const float4 q = qm[j];
    am[0] = fmaf(c, q.x, am[0]);
    am[1] = fmaf(c, q.y, am[1]);
    am[2] = fmaf(c, q.z, am[2]);
    am[3] = fmaf(c, q.w, am[3]);
    if ((s[j >> 5] >> (j & 31)) & 1u) {
      const float4 p = qq[j];
      aq[0] += p.x, aq[1] += p.y, aq[2] += p.z, aq[3] += p.w;
    }
  }
  const float n = gp.norms[row], rn = gp.rnorms[row];
  est[0] += n * am[0] + rn * (2.f * aq[0] - qtot.x);
  est[1] += n * am[1] + rn * (2.f * aq[1] - qtot.y);
  est[2] += n * am[2] + rn * (2.f * aq[2] - qtot.z);
  est[3] += n * am[3] + rn * (2.f * aq[3] - qtot.w);
}

// queries of the 4 heads of kv-head h as float4 per coordinate; the projected
// copy carries sqrt(pi/2)/d; qtot = sum of the projected copy
template <int D>
__device__ void load_group_queries(const GroupPtrs& gp, int64_t q0, float4* qm, float4* qq, float* cent_s, int K,
                                   float4* qtot, float* red) {
  const float coef = kSqrtHalfPi / D;
  for (int j = threadIdx.x; j < D; j += blockDim.x) {
    qm[j] = make_float4(gp.qrot[(q0 + 0) * D + j], gp.qrot[(q0 + 1) * D + j], gp.qrot[(q0 + 2) * D + j],
                        gp.qrot[(q0 + 3) * D + j]);
    qq[j] = make_float4(gp.qproj[(q0 + 0) * D + j] * coef, gp.qproj[(q0 + 1) * D + j] * coef,
                        gp.qproj[(q0 + 2) * D + j] * coef, gp.qproj[(q0 + 3) * D + j] * coef);
  }
  if (threadIdx.x < K) cent_s[threadIdx.x] = gp.cent[threadIdx.x];
  __syncthreads();
  if (threadIdx.x < 4) {
    float t = 0.f;
    for (int j = 0; j < D; ++j) t += reinterpret_cast<const float*>(&qq[j])[threadIdx.x];
    red[threadIdx.x] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) *qtot = make_float4(red[0], red[1], red[2], red[3]);
  __syncthreads();
}

template <int D0, int BM0, int D1, int BM1>
__global__ void __launch_bounds__(128) logits_kernel(LogitsArgs a) {
  __shared__ float4 qm0[D0], qq0[D0], qm1[D1 > 0 ? D1 : 1], qq1[D1 > 0 ? D1 : 1];
  __shared__ float c0[16], c1[16], red[4];
  __shared__ float4 tot[2];
  const int64_t bh = blockIdx.y;
  const int64_t b = bh / a.Hkv, h = bh % a.Hkv;
  const int64_t q0 = b * a.Hq + h * 4;
  load_group_queries<D0>(a.g[0], q0, qm0, qq0, c0, 1 << BM0, &tot[0], red);
  if constexpr (D1 > 0) load_group_queries<D1>(a.g[1], q0, qm1, qq1, c1, 1 << BM1, &tot[1], red);
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= a.T) return;
  const int64_t row = bh * a.kv_stride + t;
  float est[4] = {0.f, 0.f, 0.f, 0.f};
  group_scores<D0, BM0>(a.g[0], row, qm0, qq0, c0, tot[0], est);
  if constexpr (D1 > 0) group_scores<D1, BM1>(a.g[1], row, qm1, qq1, c1, tot[1], est);
#pragma unroll
  for (int hd = 0; hd < 4; ++hd) a.logits[(q0 + hd) * a.T + t] = a.scale * est[hd];
}

// q'_g = Pi_g q[channels_g], q''_g = S_g q[channels_g]: one warp per output value
template <typename TIn>
__global__ void query_prep_gather_kernel(const TIn* q, int64_t nq, int dq, const int32_t* channels, int d,
                                         const float* Pi, const float* S, float* qrot, float* qproj) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t total = nq * d * 2;
  for (int64_t w = warp; w < total; w += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int which = (int)(w / (nq * d));
    const int64_t r = w % (nq * d);
    const int64_t qi = r / d;
    const int j = (int)(r % d);
    const float* M = which ? S : Pi;
    float acc = 0.f;
    for (int i = lane; i < d; i += 32) {
      const int ch = channels ? channels[i] : i;
      float v;
      if constexpr (sizeof(TIn) == 4) v = q[qi * dq + ch];
      else v = __bfloat162float(q[qi * dq + ch]);
      acc = fmaf(M[(int64_t)j * d + i], v, acc);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) (which ? qproj : qrot)[qi * d + j] = acc;
  }
}

}  // namespace

int launch_query_prep_gather(const tq_ctx* h, const void* q, int q_dtype, int64_t nq, int dq,
                             const int32_t* channels, float* qrot, float* qproj, void* stream) {
  const int64_t warps = nq * h->d * 2;
  int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks > h->sm_count * 32) blocks = h->sm_count * 32;
  if (blocks < 1) blocks = 1;
  cudaStream_t s = (cudaStream_t)stream;
  if (q_dtype == TQ_BF16)
    query_prep_gather_kernel<<<(unsigned)blocks, 256, 0, s>>>((const __nv_bfloat16*)q, nq, dq, channels, h->d,
                                                             h->dev.Pi, h->dev.S, qrot, qproj);
  else
    query_prep_gather_kernel<<<(unsigned)blocks, 256, 0, s>>>((const float*)q, nq, dq, channels, h->d, h->dev.Pi,
                                                             h->dev.S, qrot, qproj);
  return (int)cudaGetLastError();
}

bool logits_supported(const tq_ctx* const* hk, int ngroups) {
  auto one = [](const tq_ctx* h) {
    return (h->d == 64 || h->d == 128) && h->bm >= 1 && h->bm <= 3;
  };
  if (ngroups == 1) return one(hk[0]);
  return ngroups == 2 && one(hk[0]) && one(hk[1]) && hk[0]->d == 64 && hk[1]->d == 64;
}

int launch_logits(const tq_ctx* const* hk, int ngroups, const float* const* qrot, const float* const* qproj, int B,
                  int Hq, int Hkv, int64_t T, int64_t kv_stride, const uint32_t* const* kcodes,
                  const uint32_t* const* ksigns, const float* const* knorms, const float* const* krnorms,
                  float scale, float* logits, void* stream) {
  LogitsArgs a{};
  for (int g = 0; g < ngroups; ++g)
    a.g[g] = GroupPtrs{kcodes[g], ksigns[g], knorms[g], krnorms[g], qrot[g], qproj[g], hk[g]->dev.centroids};
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.T = T;
  a.kv_stride = kv_stride;
  a.scale = scale;
  a.logits = logits;
  dim3 grid((unsigned)((T + 127) / 128), (unsigned)(B * Hkv));
  cudaStream_t s = (cudaStream_t)stream;
  const int d0 = hk[0]->d, b0 = hk[0]->bm;
#define TQ_LOGITS_CASE(D0_, B0_, D1_, B1_) logits_kernel<D0_, B0_, D1_, B1_><<<grid, 128, 0, s>>>(a)
  if (ngroups == 2) {
    const int b1 = hk[1]->bm;
    if (b0 == 3 && b1 == 2) TQ_LOGITS_CASE(64, 3, 64, 2);
    else if (b0 == 2 && b1 == 3) TQ_LOGITS_CASE(64, 2, 64, 3);
    else if (b0 == 3 && b1 == 3) TQ_LOGITS_CASE(64, 3, 64, 3);
    else if (b0 == 2 && b1 == 2) TQ_LOGITS_CASE(64, 2, 64, 2);
    else if (b0 == 1 && b1 == 1) TQ_LOGITS_CASE(64, 1, 64, 1);
    else if (b0 == 2 && b1 == 1) TQ_LOGITS_CASE(64, 2, 64, 1);
    else if (b0 == 3 && b1 == 1) TQ_LOGITS_CASE(64, 3, 64, 1);
    else return (int)cudaErrorNotSupported;
  } else if (d0 == 128) {
    if (b0 == 3) TQ_LOGITS_CASE(128, 3, 0, 0);
    else if (b0 == 2) TQ_LOGITS_CASE(128, 2, 0, 0);
    else TQ_LOGITS_CASE(128, 1, 0, 0);
  } else {
    if (b0 == 3) TQ_LOGITS_CASE(64, 3, 0, 0);
    else if (b0 == 2) TQ_LOGITS_CASE(64, 2, 0, 0);
    else TQ_LOGITS_CASE(64, 1, 0, 0);
  }
#undef TQ_LOGITS_CASE
  return (int)cudaGetLastError();
}

}  // namespace tqi
