// Decode and search over a cache split across devices: the per-slice calls
// and the merges that combine the slices' results.
//
// Decode (turboquant.net/zh, "实现步骤草图", 集成到 attention: attention over a
// TurboQuant K/V cache): when the context of every (batch, kv-head) is split
// into slices held by different devices, each device runs the decode step over
// its slice and keeps the softmax state (m = max logit, l = sum e^(logit - m),
// acc = sum e^(logit - m) n_t c_V[idx_t] in the rotated value frame); the
// states are exchanged (an all-gather of [B*Hq][d + 2] floats per device) and
// combined with the log-sum-exp rescale, and Pi_V^T is applied once.
//
// Search (m.admirer.cn report, "內存價格能下來嗎？": nearest-neighbour search over
// TurboQuant codes): each device scores its slice of the database keys and
// keeps its own top-k; the candidates are exchanged and merged into the global
// top-k (ties to the lower global index).
#include <cuda_runtime.h>

#include <cfloat>
#include <cmath>

#include "tq_internal.h"

namespace tqi {
namespace {

constexpr int kMaxShards = TQ_MAX_SHARDS;

// the state of an empty slice: acc = 0, m = -FLT_MAX, l = 0 (it adds nothing to a merge)
__global__ void empty_partial_kernel(float* partial, int64_t rows, int d) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * (d + 2)) return;
  const int64_t c = i % (d + 2);
  partial[i] = c == d ? -FLT_MAX : 0.f;
}

struct ShardOffsets {
  int64_t off[kMaxShards];
};

// One thread per query: the k best of R lists of k candidates each, by value
// descending, ties to the lower global index (the local index plus the
// slice's first key); candidates with a local index of INT32_MAX are empty.
__global__ void topk_shards_kernel(const float* val, const int32_t* idx, int R, int64_t nq, int k, ShardOffsets so,
                                   int32_t* out_idx, float* out_val) {
  const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= nq) return;
  float bv[TQ_MAX_TOPK];
  int64_t bi[TQ_MAX_TOPK];
  for (int j = 0; j < k; ++j) bv[j] = -FLT_MAX, bi[j] = INT64_MAX;
  for (int r = 0; r < R; ++r) {
    const float* v = val + ((int64_t)r * nq + q) * k;
    const int32_t* ix = idx + ((int64_t)r * nq + q) * k;
    for (int j = 0; j < k; ++j) {
      if (ix[j] == INT32_MAX) continue;
      float cv = v[j];
      int64_t ci = (int64_t)ix[j] + so.off[r];
      for (int t = 0; t < k; ++t) {
        if (cv > bv[t] || (cv == bv[t] && ci < bi[t])) {
          const float tv = bv[t];
          const int64_t ti = bi[t];
          bv[t] = cv, bi[t] = ci;
          cv = tv, ci = ti;
        }
      }
    }
  }
  for (int j = 0; j < k; ++j) {
    out_val[q * k + j] = bv[j];
    out_idx[q * k + j] = bi[j] == INT64_MAX ? INT32_MAX : (int32_t)bi[j];
  }
}

}  // namespace
}  // namespace tqi

using namespace tqi;

extern "C" size_t tq_attn_decode_partial_workspace(tq_handle hk, int B, int Hq, int Hkv, int64_t T) {
  return tq_attn_decode_workspace(hk, B, Hq, Hkv, T > 0 ? T : 1);
}

extern "C" int tq_attn_decode_partial(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
                                      int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                                      const float* knorms, const float* krnorms, const uint32_t* vcodes,
                                      const float* vnorms, float scale, float* partial, void* workspace,
                                      size_t ws_bytes, void* stream) {
  TQ_TRACE("tq_attn_decode_partial");
  const char* fn = "tq_attn_decode_partial";
  if (!hk || !hv) return set_error(TQ_EINVAL, "%s: NULL handle", fn);
  if (hk->variant != TQ_PROD || hv->variant != TQ_MSE)
    return set_error(TQ_EINVAL, "%s: need a TQ_PROD key handle and a TQ_MSE value handle", fn);
  if (hk->d != hv->d) return set_error(TQ_EINVAL, "%s: key and value d differ", fn);
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return set_error(TQ_EUNSUPPORTED, "%s: q_dtype %d", fn, q_dtype);
  if (B < 0 || Hq < 0 || Hkv <= 0 || (Hq % Hkv) != 0 || T < 0 || kv_stride < T)
    return set_error(TQ_EINVAL, "%s: bad shape (B=%d Hq=%d Hkv=%d T=%lld stride=%lld)", fn, B, Hq, Hkv,
                     (long long)T, (long long)kv_stride);
  if (!std::isfinite(scale)) return set_error(TQ_EINVAL, "%s: scale is not finite", fn);
  if (B == 0 || Hq == 0) return clear_error();
  if (!partial) return set_error(TQ_EINVAL, "%s: NULL partial", fn);
  if (reinterpret_cast<uintptr_t>(partial) & 15u) return set_error(TQ_EALIGN, "%s: partial is not 16-byte aligned", fn);
  const int64_t rows = (int64_t)B * Hq;
  if (T == 0) {
    const int64_t n = rows * (hv->d + 2);
    empty_partial_kernel<<<(unsigned)((n + 255) / 256), 256, 0, (cudaStream_t)stream>>>(partial, rows, hv->d);
    const int e = (int)cudaGetLastError();
    return e ? set_error(TQ_ECUDA, "%s: %s", fn, cudaGetErrorString((cudaError_t)e)) : clear_error();
  }
  if (!q || !kcodes || !ksigns || !knorms || !krnorms || !vcodes || !vnorms)
    return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  for (const void* p : {(const void*)q, (const void*)kcodes, (const void*)ksigns, (const void*)knorms,
                        (const void*)krnorms, (const void*)vcodes, (const void*)vnorms, (const void*)workspace})
    if (reinterpret_cast<uintptr_t>(p) & 15u) return set_error(TQ_EALIGN, "%s: a device pointer is not 16-byte aligned", fn);
  const size_t need = tq_attn_decode_workspace(hk, B, Hq, Hkv, T);
  if (!workspace || ws_bytes < need) return set_error(TQ_EWORKSPACE, "%s: workspace %zu < %zu bytes", fn, ws_bytes, need);
  const int e = decode_dispatch(hk, hv, q, q_dtype, B, Hq, Hkv, T, kv_stride, kcodes, ksigns, knorms, krnorms, vcodes,
                                vnorms, scale, partial, workspace, stream, 1);
  return e ? set_error(TQ_ECUDA, "%s: %s", fn, cudaGetErrorString((cudaError_t)e)) : clear_error();
}

extern "C" int tq_attn_merge(tq_handle hv, const float* partials, int R, int64_t rows, float* out, void* stream) {
  TQ_TRACE("tq_attn_merge");
  const char* fn = "tq_attn_merge";
  if (!hv) return set_error(TQ_EINVAL, "%s: NULL handle", fn);
  if (hv->variant != TQ_MSE) return set_error(TQ_EINVAL, "%s: need the TQ_MSE value handle", fn);
  if (R < 1 || rows < 0) return set_error(TQ_EINVAL, "%s: R = %d, rows = %lld", fn, R, (long long)rows);
  if (rows == 0) return clear_error();
  if (!partials || !out) return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  if ((reinterpret_cast<uintptr_t>(partials) | reinterpret_cast<uintptr_t>(out)) & 15u)
    return set_error(TQ_EALIGN, "%s: a device pointer is not 16-byte aligned", fn);
  const int d = hv->d;
  const int e = launch_decode_merge(partials, rows, R, hv, out, stream, rows * (d + 2), d + 2, 0);
  return e ? set_error(TQ_ECUDA, "%s: %s", fn, cudaGetErrorString((cudaError_t)e)) : clear_error();
}

extern "C" int tq_topk_merge(const float* val, const int32_t* idx, int R, int64_t nq, int k, const int64_t* offsets,
                             int32_t* out_idx, float* out_val, void* stream) {
  TQ_TRACE("tq_topk_merge");
  const char* fn = "tq_topk_merge";
  if (R < 1 || R > TQ_MAX_SHARDS) return set_error(TQ_EINVAL, "%s: R = %d (need 1..%d)", fn, R, TQ_MAX_SHARDS);
  if (nq < 0 || k < 1 || k > TQ_MAX_TOPK) return set_error(TQ_EINVAL, "%s: nq = %lld, k = %d", fn, (long long)nq, k);
  if (!offsets) return set_error(TQ_EINVAL, "%s: NULL offsets", fn);
  ShardOffsets so;
  for (int r = 0; r < R; ++r) {
    if (offsets[r] < 0) return set_error(TQ_EINVAL, "%s: negative offset", fn);
    so.off[r] = offsets[r];
  }
  if (nq == 0) return clear_error();
  if (!val || !idx || !out_idx || !out_val) return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  for (const void* p : {(const void*)val, (const void*)idx, (const void*)out_idx, (const void*)out_val})
    if (reinterpret_cast<uintptr_t>(p) & 3u) return set_error(TQ_EALIGN, "%s: a device pointer is not 4-byte aligned", fn);
  topk_shards_kernel<<<(unsigned)((nq + 127) / 128), 128, 0, (cudaStream_t)stream>>>(val, idx, R, nq, k, so, out_idx,
                                                                                     out_val);
  const int e = (int)cudaGetLastError();
  return e ? set_error(TQ_ECUDA, "%s: %s", fn, cudaGetErrorString((cudaError_t)e)) : clear_error();
}
