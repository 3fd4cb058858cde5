// tq_attn_decode_static: the decode-attention step of tq_attn_decode with its
// scratch memory held in a fixed device array inside this library, so the
// caller passes no workspace and the call allocates nothing.
//
// Who needs this: a caller that may not allocate device memory while it runs
// -- for example a plugin whose host application owns the whole device memory
// budget through its own pool and offers the plugin no allocation hook, or a
// service that must keep its device footprint fixed after start-up.  Such a
// caller cannot obtain the workspace tq_attn_decode asks for.
//
// The scratch is one file-scope __device__ array of TQ_DECODE_STATIC_SCRATCH
// bytes.  It exists on every GPU that loads this library, for as long as the
// process lives.  All calls on a device share it.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "tq_internal.h"

namespace tqi {
namespace {

// The scratch array.  In host code this name is only a stand-in for the
// symbol: the device address must be obtained with cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_decode_scratch[TQ_DECODE_STATIC_SCRATCH];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once
// per device (the first call on a device does this set-up).
int scratch_address(void** out) {
  int dev = 0;
  int e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return (int)cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return (int)cudaSuccess;
}

}  // namespace
}  // namespace tqi

using namespace tqi;

extern "C" int tq_attn_decode_static(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B,
                                     int Hq, int Hkv, int64_t T, int64_t kv_stride,
                                     const uint32_t* kcodes, const uint32_t* ksigns,
                                     const float* knorms, const float* krnorms,
                                     const uint32_t* vcodes, const float* vnorms, float scale,
                                     float* out, void* stream) {
  TQ_TRACE("tq_attn_decode_static");
  if (!hk || !hv) return set_error(TQ_EINVAL, "tq_attn_decode_static: NULL handle");
  if (hk->variant != TQ_PROD || hv->variant != TQ_MSE)
    return set_error(TQ_EINVAL,
                     "tq_attn_decode_static: need a TQ_PROD key handle and a TQ_MSE value handle");
  if (hk->d != hv->d) return set_error(TQ_EINVAL, "tq_attn_decode_static: key and value d differ");
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16)
    return set_error(TQ_EUNSUPPORTED, "tq_attn_decode_static: q_dtype %d", q_dtype);
  if (B < 0 || Hq < 0 || Hkv <= 0 || (Hq % Hkv) != 0 || T < 1 || kv_stride < T)
    return set_error(TQ_EINVAL, "tq_attn_decode_static: bad shape (B=%d Hq=%d Hkv=%d T=%lld stride=%lld)",
                     B, Hq, Hkv, (long long)T, (long long)kv_stride);
  if (!std::isfinite(scale)) return set_error(TQ_EINVAL, "tq_attn_decode_static: scale is not finite");
  if (B == 0 || Hq == 0) return clear_error();
  if (!q || !kcodes || !ksigns || !knorms || !krnorms || !vcodes || !vnorms || !out)
    return set_error(TQ_EINVAL, "tq_attn_decode_static: NULL pointer");
  for (const void* p : {(const void*)q, (const void*)kcodes, (const void*)ksigns, (const void*)knorms,
                        (const void*)krnorms, (const void*)vcodes, (const void*)vnorms, (const void*)out})
    if (reinterpret_cast<uintptr_t>(p) & 15u)
      return set_error(TQ_EALIGN, "tq_attn_decode_static: a device pointer is not 16-byte aligned");
  const size_t need = tq_attn_decode_workspace(hk, B, Hq, Hkv, T);
  if (need > (size_t)TQ_DECODE_STATIC_SCRATCH)
    return set_error(TQ_EWORKSPACE,
                     "tq_attn_decode_static: this shape needs %zu bytes of scratch, more than the %d "
                     "bytes built into the library; use tq_attn_decode with a workspace",
                     need, TQ_DECODE_STATIC_SCRATCH);
  void* ws = nullptr;
  int e = scratch_address(&ws);
  if (e != cudaSuccess)
    return set_error(TQ_ECUDA, "tq_attn_decode_static: scratch set-up: %s",
                     cudaGetErrorString((cudaError_t)e));
  // same kernels and the same partition of the scratch as tq_attn_decode uses
  // for its workspace; every byte read is written earlier in the same call, so
  // nothing has to be cleared between calls
  e = decode_dispatch(hk, hv, q, q_dtype, B, Hq, Hkv, T, kv_stride, kcodes, ksigns, knorms, krnorms, vcodes,
                      vnorms, scale, out, ws, stream);
  if (e)
    return set_error(TQ_ECUDA, "tq_attn_decode_static: %s", cudaGetErrorString((cudaError_t)e));
  return clear_error();
}
