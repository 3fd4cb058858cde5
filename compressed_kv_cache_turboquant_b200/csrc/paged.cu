// A paged TurboQuant K/V cache: quantize-on-write through a slot mapping, and
// decode attention that reads the cache through a block table.
//
// turboquant.net/zh, "工程风险与应对", 残差范数存储: the residual norm costs one
// extra FP16 scalar per vector; tmdm.cn ("谷歌悄悄扔下一颗“性能核弹”…", 实测数据):
// only the store and load of the KV cache are replaced; ttakun.com/news/45354
// (新旧量化方案深度权衡矩阵): each token is compressed as it arrives.  The paging
// itself is the serving layout these calls plug into: a sequence's tokens live
// in fixed-size pages of every cache array, located through a block table.
#include <cuda_runtime.h>

#include <cmath>

#include "tq_internal.h"

using namespace tqi;

extern "C" int tq_quant_paged(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                              const int32_t* channels, const int64_t* slots, uint32_t* codes, uint32_t* signs,
                              float* norms, void* rnorms, int rn_dtype, void* stream) {
  TQ_TRACE("tq_quant_paged");
  const char* fn = "tq_quant_paged";
  if (!h) return set_error(TQ_EINVAL, "%s: NULL handle", fn);
  if (h->variant == TQ_POLAR) return set_error(TQ_EINVAL, "%s: a TQ_POLAR handle", fn);
  if (N < 0) return set_error(TQ_EINVAL, "%s: N < 0", fn);
  if (dtype != TQ_F32 && dtype != TQ_BF16) return set_error(TQ_EUNSUPPORTED, "%s: dtype %d", fn, dtype);
  if (rn_dtype != TQ_F32 && rn_dtype != TQ_F16) return set_error(TQ_EUNSUPPORTED, "%s: rn_dtype %d", fn, rn_dtype);
  if (!quant_fused_supported(h))
    return set_error(TQ_EUNSUPPORTED, "%s: d = %d (the paged writer takes d <= 256)", fn, h->d);
  if (channels ? x_stride < 1 : (x_stride < h->d || x_stride % 8 != 0))
    return set_error(TQ_EINVAL, "%s: x_stride %lld", fn, (long long)x_stride);
  const bool prod = h->variant == TQ_PROD;
  if (N == 0) return clear_error();
  if (!x || !slots || !codes || !norms || (prod && (!signs || !rnorms))) return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  for (const void* p : {(const void*)x, (const void*)channels, (const void*)slots, (const void*)codes,
                        (const void*)signs, (const void*)norms, (const void*)rnorms})
    if (reinterpret_cast<uintptr_t>(p) & (p == x || p == slots ? 15u : 3u))
      return set_error(TQ_EALIGN, "%s: a device pointer is not aligned", fn);
  const int e = launch_quant_fused(h, x, dtype, N, x_stride, codes, prod ? signs : nullptr, norms,
                                   prod ? rnorms : nullptr, 1, stream, channels, slots, rn_dtype == TQ_F16 ? 1 : 0);
  return e ? set_error(TQ_ECUDA, "%s: %s", fn, cudaGetErrorString((cudaError_t)e)) : clear_error();
}

extern "C" int tq_attn_decode_paged(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
                                    int64_t T, const int32_t* block_table, int max_pages, int page_size,
                                    const uint32_t* kcodes, const uint32_t* ksigns, const float* knorms,
                                    const void* krnorms, int rn_dtype, const uint32_t* vcodes, const float* vnorms,
                                    float scale, float* out, void* workspace, size_t ws_bytes, void* stream) {
  TQ_TRACE("tq_attn_decode_paged");
  const char* fn = "tq_attn_decode_paged";
  if (!hk || !hv) return set_error(TQ_EINVAL, "%s: NULL handle", fn);
  if (hk->variant != TQ_PROD || hv->variant != TQ_MSE)
    return set_error(TQ_EINVAL, "%s: need a TQ_PROD key handle and a TQ_MSE value handle", fn);
  if (hk->d != hv->d) return set_error(TQ_EINVAL, "%s: key and value d differ", fn);
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return set_error(TQ_EUNSUPPORTED, "%s: q_dtype %d", fn, q_dtype);
  if (rn_dtype != TQ_F32 && rn_dtype != TQ_F16) return set_error(TQ_EUNSUPPORTED, "%s: rn_dtype %d", fn, rn_dtype);
  if (B < 0 || Hq < 0 || Hkv <= 0 || (Hq % Hkv) != 0 || T < 1)
    return set_error(TQ_EINVAL, "%s: bad shape (B=%d Hq=%d Hkv=%d T=%lld)", fn, B, Hq, Hkv, (long long)T);
  if (page_size < 8 || page_size % 8 != 0 || max_pages < 1 || (int64_t)max_pages * page_size < T)
    return set_error(TQ_EINVAL, "%s: page_size %d (need a multiple of 8) and max_pages %d must cover T", fn,
                     page_size, max_pages);
  if (!std::isfinite(scale)) return set_error(TQ_EINVAL, "%s: scale is not finite", fn);
  if (B == 0 || Hq == 0) return clear_error();
  if (!q || !block_table || !kcodes || !ksigns || !knorms || !krnorms || !vcodes || !vnorms || !out)
    return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  for (const void* p : {(const void*)q, (const void*)kcodes, (const void*)ksigns, (const void*)knorms, krnorms,
                        (const void*)vcodes, (const void*)vnorms, (const void*)out, (const void*)workspace,
                        (const void*)block_table})
    if (reinterpret_cast<uintptr_t>(p) & 15u) return set_error(TQ_EALIGN, "%s: a device pointer is not 16-byte aligned", fn);
  const size_t need = tq_attn_decode_workspace(hk, B, Hq, Hkv, T);
  if (!workspace || ws_bytes < need) return set_error(TQ_EWORKSPACE, "%s: workspace %zu < %zu bytes", fn, ws_bytes, need);
  PagedCache pg;
  pg.block_table = block_table;
  pg.max_pages = max_pages;
  pg.page = page_size;
  pg.rn16 = rn_dtype == TQ_F16 ? 1 : 0;
  const int e = decode_dispatch(hk, hv, q, q_dtype, B, Hq, Hkv, T, T, kcodes, ksigns, knorms,
                                static_cast<const float*>(krnorms), vcodes, vnorms, scale, out, workspace, stream, 0, pg);
  return e ? set_error(TQ_ECUDA, "%s: %s", fn, cudaGetErrorString((cudaError_t)e)) : clear_error();
}
