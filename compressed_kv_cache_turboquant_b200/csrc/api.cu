// C ABI of the TurboQuant hot path: argument checks, handle management and
// dispatch to the kernels.  The operations are defined in include/tq.h.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <set>
#include <tuple>
#include <vector>

#include "tq_internal.h"

namespace tqi {

static thread_local char g_err[512] = "";

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int clear_error() {
  g_err[0] = '\0';
  return TQ_OK;
}

// The attribute is one value per (kernel, device), the largest dynamic window a
// launch may ask for; it is raised once to the device's opt-in maximum, so
// launches of one kernel with different window sizes (one per d) never lower it.
int ensure_dyn_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return (int)cudaSuccess;
  int maxb = 0;
  e = cudaDeviceGetAttribute(&maxb, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return (int)e;
  if (bytes > maxb) return (int)cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, maxb);
  if (e == cudaSuccess) done.insert({kernel, dev});
  return (int)e;
}

static int cuda_error(const char* where, int e) {
  return set_error(TQ_ECUDA, "%s: %s", where, cudaGetErrorString((cudaError_t)e));
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define TQ_CHECK_ALIGN(p, name)                                                        \
  do {                                                                                 \
    if ((p) && !aligned16(p)) return set_error(TQ_EALIGN, "%s is not 16-byte aligned", name); \
  } while (0)

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// round to the nearest bfloat16 (ties to even, via float32); returns the bits
// and stores the value it represents
static uint16_t to_bf16(double v, double* represented) {
  float f = (float)v;
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  const uint16_t b = (uint16_t)(u >> 16);
  const uint32_t back = (uint32_t)b << 16;
  float r;
  std::memcpy(&r, &back, 4);
  *represented = (double)r;
  return b;
}

// Pi = hi + mid + lo in bf16, arranged for the tensor-core kernels (see DevConsts::pi_tc)
static void split_rotation_bf16(const double* Pi, int d, std::vector<uint16_t>& out) {
  const int slabs = d / 64;
  const size_t piece = (size_t)d * d;
  out.assign(3 * piece, 0);
  for (int j = 0; j < d; ++j)
    for (int i = 0; i < d; ++i) {
      double rem = Pi[(size_t)j * d + i];
      const int slab = i / 64, c = (i % 64) / 8, e = i % 8;
      const size_t off = (size_t)slab * d * 64 + (size_t)j * 64 + (size_t)((c ^ (j & 7)) * 8 + e);
      for (int p = 0; p < 3; ++p) {
        double rep;
        out[p * piece + off] = to_bf16(rem, &rep);
        rem -= rep;
      }
    }
  (void)slabs;
}

static uint16_t half_bits(double v) {
  __half h = __double2half(v);
  uint16_t b;
  std::memcpy(&b, &h, 2);
  return b;
}

static double half_value(uint16_t b) {
  __half h;
  std::memcpy(&h, &b, 2);
  return (double)__half2float(h);
}

// A common scale alpha in [1, 2) (20 fractional bits) for which every scaled
// centroid alpha c[k] is closest to an fp16 value, relative to its size.  With
// the scale divided out again in fp32, the fp16 table carries the codebook to
// about 2e-5 relative for 8 levels and 1e-6 or better for 4 or fewer, instead
// of the 2^-11 of a plain fp16 rounding.
static void scaled_half_codebook(tq_ctx* h) {
  const int K = 1 << h->bm;
  double mags[8];
  int nm = 0;
  for (int k = K / 2; k < K && nm < 8; ++k) mags[nm++] = std::fabs(h->host_centroids[k]);
  double best = 1e300, best_a = 1.0;
  for (int i = 0; i < (1 << 20); ++i) {
    const double a = 1.0 + std::ldexp((double)i, -20);
    double e = 0.0;
    for (int m = 0; m < nm && e < best; ++m) {
      const double v = a * mags[m];
      if (v == 0.0) continue;
      e = std::fmax(e, std::fabs(half_value(half_bits(v)) - v) / v);
    }
    if (e < best) best = e, best_a = a;
  }
  for (int k = 0; k < K; ++k) h->sc_tab[k] = half_bits(best_a * h->host_centroids[k]);
  h->sc_inv_alpha = (float)(1.0 / best_a);
  h->sc_rel_err = best;
}

// Pi^T as fp16 pieces (hi, (Pi - hi) * 2^11) in the swizzled K-major layout:
// B[i][j] = Pi[j][i], row i, K index j
static void split_rotation_t_f16(const double* Pi, int d, std::vector<uint16_t>& out) {
  const size_t piece = (size_t)d * d;
  out.assign(2 * piece, 0);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) {
      const double v = Pi[(size_t)j * d + i];
      const int slab = j / 64, c = (j % 64) / 8, e = j % 8;
      const size_t off = (size_t)slab * d * 64 + (size_t)i * 64 + (size_t)((c ^ (i & 7)) * 8 + e);
      const uint16_t hi = half_bits(v);
      out[off] = hi;
      out[piece + off] = half_bits((v - half_value(hi)) * 2048.0);
    }
}

// decode attention: context splits per (batch, q-head)
int decode_splits(int B, int Hq, int64_t T, int sm_count) {
  // enough CTAs to fill the machine a few times, each split >= 512 tokens
  int64_t want = (int64_t)sm_count * 4 / std::max(1, B * Hq);
  int64_t cap = (T + 511) / 512;
  int64_t s = std::max<int64_t>(1, std::min<int64_t>(want > 0 ? want : 1, cap));
  return (int)std::min<int64_t>(s, 256);
}

}  // namespace tqi

using namespace tqi;

extern "C" const char* tq_last_error(void) { return g_err; }
extern "C" const char* tq_version(void) { return "tq-b200 0.1 (sm_100a)"; }

extern "C" int tq_create(tq_handle* out, int d, int b, int variant, const double* Pi,
                         const double* S, const double* centroids) {
  TQ_TRACE("tq_create");
  if (!out || !Pi) return set_error(TQ_EINVAL, "tq_create: NULL handle or rotation");
  *out = nullptr;
  if (variant != TQ_MSE && variant != TQ_PROD)
    return set_error(TQ_EUNSUPPORTED, "tq_create: unknown variant %d", variant);
  if (d < 8 || d > TQ_MAX_DIM || d % 8 != 0)
    return set_error(TQ_EUNSUPPORTED, "tq_create: d = %d (need 8 <= d <= %d, d %% 8 == 0)", d,
                     TQ_MAX_DIM);
  const int bm = (variant == TQ_MSE) ? b : b - 1;
  if (bm < 1 || bm > kMaxMseBits)
    return set_error(TQ_EUNSUPPORTED, "tq_create: b = %d unsupported for this variant", b);
  if (variant == TQ_PROD && !S) return set_error(TQ_EINVAL, "tq_create: TQ_PROD needs S");

  tq_ctx* h = new (std::nothrow) tq_ctx();
  if (!h) return set_error(TQ_ENOMEM, "tq_create: out of host memory");
  h->d = d;
  h->b = b;
  h->variant = variant;
  h->bm = bm;
  const int K = 1 << bm;
  if (centroids) {
    for (int k = 0; k < K; ++k) h->host_centroids[k] = centroids[k];
    for (int k = 0; k + 1 < K; ++k) {
      if (!(centroids[k] < centroids[k + 1])) {
        delete h;
        return set_error(TQ_EINVAL, "tq_create: centroids must be strictly ascending");
      }
      h->host_thresholds[k] = 0.5 * (centroids[k] + centroids[k + 1]);
    }
  } else {
    int rc = tq_make_codebook(bm, d, h->host_centroids, h->host_thresholds);
    if (rc != TQ_OK) {
      delete h;
      return rc;
    }
  }
  if (bm <= 3) scaled_half_codebook(h);
  int e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, h->device);
  if (e != cudaSuccess) {
    delete h;
    return cuda_error("tq_create", e);
  }

  // host staging of every constant (float32), then one upload
  const size_t dd = (size_t)d * d;
  std::vector<float> Pf(dd), PTf(dd), Sf, TTf;
  std::vector<double> Td;
  for (int j = 0; j < d; ++j)
    for (int i = 0; i < d; ++i) {
      Pf[(size_t)j * d + i] = (float)Pi[(size_t)j * d + i];
      PTf[(size_t)i * d + j] = (float)Pi[(size_t)j * d + i];
    }
  if (variant == TQ_PROD) {
    Sf.resize(dd);
    TTf.resize(dd);
    for (size_t k = 0; k < dd; ++k) Sf[k] = (float)S[k];
    // T = S Pi^T in float64: T[j][i] = sum_k S[j][k] Pi[i][k]; stored as TT[i][j]
    Td.resize(dd);
    for (int j = 0; j < d; ++j)
      for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        const double* s = S + (size_t)j * d;
        const double* p = Pi + (size_t)i * d;
        for (int k = 0; k < d; ++k) acc += s[k] * p[k];
        Td[(size_t)j * d + i] = acc;
        TTf[(size_t)i * d + j] = (float)acc;
      }
  }
  // general-d quantizer pieces (hi, lo * 2^11) of Pi and of [S | T]
  const int dp = (d + 127) / 128 * 128;
  h->gen_d_pad = dp;
  std::vector<uint16_t> gpi((size_t)2 * dp * dp, 0), gst;
  auto split_into = [&](double v, uint16_t* hi, uint16_t* lo) {
    const uint16_t hb = half_bits(v);
    *hi = hb;
    *lo = half_bits((v - half_value(hb)) * 2048.0);
  };
  for (int n = 0; n < d; ++n)
    for (int k = 0; k < d; ++k)
      split_into(Pi[(size_t)n * d + k], &gpi[(size_t)n * dp + k], &gpi[((size_t)dp + n) * dp + k]);
  if (variant == TQ_PROD) {
    const size_t w2 = (size_t)2 * dp;
    gst.assign(2 * (size_t)dp * w2, 0);
    for (int n = 0; n < d; ++n)
      for (int k = 0; k < d; ++k) {
        split_into(S[(size_t)n * d + k], &gst[(size_t)n * w2 + k], &gst[((size_t)dp + n) * w2 + k]);
        split_into(Td[(size_t)n * d + k], &gst[(size_t)n * w2 + dp + k], &gst[((size_t)dp + n) * w2 + dp + k]);
      }
  }
  // fused quantizer pieces (d <= 256): hi and remainder of kFusedPieceScale * Pi / T
  std::vector<uint16_t> fzp, fzt;
  const int n16 = (d + 15) / 16 * 16, k64 = (d + 63) / 64 * 64;
  if (d <= 256) {
    auto fill = [&](const double* M, std::vector<uint16_t>& out) {
      out.assign((size_t)2 * n16 * k64, 0);
      for (int n = 0; n < d; ++n)
        for (int k = 0; k < d; ++k) {
          const double v = (double)kFusedPieceScale * M[(size_t)n * d + k];
          const uint16_t hb = half_bits(v);
          out[(size_t)n * k64 + k] = hb;
          out[((size_t)n16 + n) * k64 + k] = half_bits(v - half_value(hb));
        }
    };
    fill(Pi, fzp);
    if (variant == TQ_PROD) fill(Td.data(), fzt);
    h->fz_n16 = n16;
    h->fz_k64 = k64;
  }
  std::vector<float> cf(K), tf(K);
  for (int k = 0; k < K; ++k) cf[k] = (float)h->host_centroids[k];
  for (int k = 0; k + 1 < K; ++k) tf[k] = (float)h->host_thresholds[k];

  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t oPi = take(dd * 4), oPT = take(dd * 4);
  const size_t oS = (variant == TQ_PROD) ? take(dd * 4) : 0;
  const size_t oTT = (variant == TQ_PROD) ? take(dd * 4) : 0;
  const size_t oC = take(64 * 4), oT = take(64 * 4), oStatus = take(256);
  const bool tc = (d == 64 || d == 128);
  std::vector<uint16_t> pieces;
  if (tc) split_rotation_bf16(Pi, d, pieces);
  const size_t oPiTc = tc ? take(pieces.size() * 2) : 0;
  std::vector<uint16_t> tpieces;
  std::vector<uint32_t> lut(16, 0u);
  if (tc) {
    split_rotation_t_f16(Pi, d, tpieces);
    for (int k = 0; k < K; ++k) {
      const uint16_t hi = half_bits(h->host_centroids[k]);
      const uint16_t lo = half_bits((h->host_centroids[k] - half_value(hi)) * 2048.0);
      lut[k] = (uint32_t)hi | ((uint32_t)lo << 16);
    }
  }
  const size_t oPitF16 = tc ? take(tpieces.size() * 2) : 0;
  const size_t oLut = take(16 * 4);
  // fp16 byte tables for register decoding: 8 entries as lo-byte and hi-byte words
  auto byte_table = [&](const double* c8, uint32_t* t4) {
    for (int w = 0; w < 2; ++w) {
      uint32_t lo = 0, hi = 0;
      for (int k = 0; k < 4; ++k) {
        const uint16_t hb = half_bits(c8[4 * w + k]);
        lo |= (uint32_t)(hb & 0xFFu) << (8 * k);
        hi |= (uint32_t)(hb >> 8) << (8 * k);
      }
      t4[w] = lo;
      t4[2 + w] = hi;
    }
  };
  uint32_t ktab[4] = {0, 0, 0, 0}, vtab[4] = {0, 0, 0, 0};
  const bool has_ktab = (bm == 3);
  bool has_vtab = (bm == 4);
  for (int k = 0; has_vtab && k < 16; ++k)
    if (h->host_centroids[15 - k] != -h->host_centroids[k]) has_vtab = false;  // needs c[15-i] = -c[i]
  if (has_ktab) byte_table(h->host_centroids, ktab);
  for (int k = 0; k < 4; ++k) h->host_ktab[k] = ktab[k];
  if (has_vtab) byte_table(h->host_centroids + 8, vtab);
  const size_t oTabs = take(8 * 4);
  const size_t oGenPi = take(gpi.size() * 2);
  const size_t oGenSt = gst.empty() ? 0 : take(gst.size() * 2);
  const size_t oFzPi = fzp.empty() ? 0 : take(fzp.size() * 2);
  const size_t oFzT = fzt.empty() ? 0 : take(fzt.size() * 2);
  h->block_bytes = off;
  e = cudaMalloc(&h->block, h->block_bytes);
  if (e != cudaSuccess) {
    delete h;
    return set_error(TQ_ENOMEM, "tq_create: cudaMalloc of %zu bytes failed", off);
  }
  char* base = (char*)h->block;
  h->dev.Pi = (float*)(base + oPi);
  h->dev.PiT = (float*)(base + oPT);
  h->dev.centroids = (float*)(base + oC);
  h->dev.thresholds = (float*)(base + oT);
  h->dev.status = (int*)(base + oStatus);
  if (tc) h->dev.pi_tc = (uint8_t*)(base + oPiTc);
  if (tc) h->dev.pit_f16 = (uint8_t*)(base + oPitF16);
  h->dev.lut_dq = (uint32_t*)(base + oLut);
  h->dev.gen_pi = (uint16_t*)(base + oGenPi);
  if (!gst.empty()) h->dev.gen_st = (uint16_t*)(base + oGenSt);
  if (!fzp.empty()) h->dev.fz_pi = (uint16_t*)(base + oFzPi);
  if (!fzt.empty()) h->dev.fz_t = (uint16_t*)(base + oFzT);
  if (has_ktab) h->dev.ktab = (uint32_t*)(base + oTabs);
  if (has_vtab) h->dev.vtab = (uint32_t*)(base + oTabs + 16);
  if (variant == TQ_PROD) {
    h->dev.S = (float*)(base + oS);
    h->dev.TT = (float*)(base + oTT);
  }
  e = cudaMemcpy(h->dev.Pi, Pf.data(), dd * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->dev.PiT, PTf.data(), dd * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->dev.centroids, cf.data(), K * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && K > 1)
    e = cudaMemcpy(h->dev.thresholds, tf.data(), (K - 1) * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemset(h->dev.status, 0, 256);
  {
    // TQ_RUNTIME_TABLE_ADDRESSES=1 keeps the kernels that add table addresses at run time
    const char* ev = getenv("TQ_RUNTIME_TABLE_ADDRESSES");
    if (e == cudaSuccess && !(ev && ev[0] == '1'))
      e = (cudaError_t)probe_dyn_smem_base((uint32_t*)(h->dev.status + 16), &h->dyn_base);
    const char* fr = getenv("TQ_FUSED_REGISTER_LOADS");
    h->fused_register_loads = fr && fr[0] == '1';
    const char* dl = getenv("TQ_TCGEN05_ATTN");
    h->tc_attn = dl && dl[0] == '1';
    const char* st = getenv("TQ_DEBUG_STALL_MS");
    if (st && atof(st) > 0) h->debug_stall_ns = (uint64_t)(atof(st) * 1e6);
    const char* db = getenv("TQ_DEBUG_DYN_BASE");
    if (db && db[0]) {
      h->dyn_base = (uint32_t)strtoul(db, nullptr, 0);
      h->debug_fixed_tables = true;
    }
  }
  if (e == cudaSuccess && tc)
    e = cudaMemcpy(h->dev.pi_tc, pieces.data(), pieces.size() * 2, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && tc)
    e = cudaMemcpy(h->dev.pit_f16, tpieces.data(), tpieces.size() * 2, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->dev.lut_dq, lut.data(), 16 * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(base + oTabs, ktab, 16, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(base + oTabs + 16, vtab, 16, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->dev.gen_pi, gpi.data(), gpi.size() * 2, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && !gst.empty())
    e = cudaMemcpy(h->dev.gen_st, gst.data(), gst.size() * 2, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && !fzp.empty())
    e = cudaMemcpy(h->dev.fz_pi, fzp.data(), fzp.size() * 2, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && !fzt.empty())
    e = cudaMemcpy(h->dev.fz_t, fzt.data(), fzt.size() * 2, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && variant == TQ_PROD) {
    e = cudaMemcpy(h->dev.S, Sf.data(), dd * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(h->dev.TT, TTf.data(), dd * 4, cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    cudaFree(h->block);
    delete h;
    return cuda_error("tq_create upload", e);
  }
  *out = h;
  return clear_error();
}

extern "C" int tq_create_polar(tq_handle* out, int d, int b1, int bh, const double* Pi) {
  TQ_TRACE("tq_create_polar");
  if (!out || !Pi) return set_error(TQ_EINVAL, "tq_create_polar: NULL handle or rotation");
  *out = nullptr;
  if (d != 64 && d != 128) return set_error(TQ_EUNSUPPORTED, "tq_create_polar: d = %d (need 64 or 128)", d);
  if ((b1 != 2 && b1 != 4) || (bh != 1 && bh != 2))
    return set_error(TQ_EUNSUPPORTED, "tq_create_polar: b1 = %d, bh = %d (need b1 in {2, 4}, bh in {1, 2})", b1, bh);
  // the rotation operands of an mse instance, then the polar constants
  int rc = tq_create(out, d, b1, TQ_MSE, Pi, nullptr, nullptr);
  if (rc) return rc;
  tq_ctx* h = *out;
  h->variant = TQ_POLAR;
  h->polar_b1 = b1;
  h->polar_bh = bh;
  int L = 0;
  while ((1 << L) < d) ++L;
  std::vector<float> cs(2 * 8 * 16, 0.f);
  double c[16], t[15];
  rc = tq_polar_codebook(b1, 1, c, nullptr);
  for (int k = 0; rc == TQ_OK && k < (1 << b1); ++k) {
    cs[0 * 128 + 1 * 16 + k] = (float)std::cos(c[k]);
    cs[1 * 128 + 1 * 16 + k] = (float)std::sin(c[k]);
  }
  for (int l = 2; rc == TQ_OK && l <= L; ++l) {
    rc = tq_polar_codebook(bh, l, c, t);
    for (int k = 0; rc == TQ_OK && k < (1 << bh); ++k) {
      cs[0 * 128 + l * 16 + k] = (float)std::cos(c[k]);
      cs[1 * 128 + l * 16 + k] = (float)std::sin(c[k]);
      if (k + 1 < (1 << bh)) h->polar_tan2[l][k] = (float)(std::tan(t[k]) * std::tan(t[k]));
    }
  }
  int e = rc == TQ_OK ? (int)cudaMalloc(&h->polar_cs, cs.size() * 4) : 0;
  if (rc == TQ_OK && e == cudaSuccess) e = cudaMemcpy(h->polar_cs, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice);
  if (rc != TQ_OK || e != cudaSuccess) {
    tq_destroy(h);
    *out = nullptr;
    return rc != TQ_OK ? rc : cuda_error("tq_create_polar", e);
  }
  return clear_error();
}

extern "C" int tq_destroy(tq_handle h) {
  TQ_TRACE("tq_destroy");
  if (!h) return clear_error();
  int e = cudaDeviceSynchronize();
  if (h->polar_cs) cudaFree(h->polar_cs);
  int e2 = cudaFree(h->block);
  delete h;
  if (e != cudaSuccess) return cuda_error("tq_destroy", e);
  if (e2 != cudaSuccess) return cuda_error("tq_destroy", e2);
  return clear_error();
}

extern "C" int tq_device_status(tq_handle h, int* status) {
  if (!h || !status) return set_error(TQ_EINVAL, "tq_device_status: NULL argument");
  int e = cudaMemcpy(status, h->dev.status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(h->dev.status, 0, sizeof(int));
  return e ? cuda_error("tq_device_status", e) : clear_error();
}

extern "C" int tq_handle_info(tq_handle h, int* d, int* b, int* variant, int* mse_bits) {
  TQ_TRACE("tq_handle_info");
  if (!h) return set_error(TQ_EINVAL, "tq_handle_info: NULL handle");
  if (d) *d = h->d;
  if (b) *b = h->b;
  if (variant) *variant = h->variant;
  if (mse_bits) *mse_bits = h->bm;
  return clear_error();
}

static int check_quant_args(const char* fn, tq_handle h, int want_variant, const void* x, int dtype,
                            int64_t N, int64_t x_stride, const void* codes, const void* norms,
                            int64_t out_stride) {
  if (!h) return set_error(TQ_EINVAL, "%s: NULL handle", fn);
  if (h->variant != want_variant) return set_error(TQ_EINVAL, "%s: wrong handle variant", fn);
  if (N < 0) return set_error(TQ_EINVAL, "%s: N < 0", fn);
  if (dtype != TQ_F32 && dtype != TQ_BF16) return set_error(TQ_EUNSUPPORTED, "%s: dtype %d", fn, dtype);
  if (x_stride < h->d || x_stride % 8 != 0)
    return set_error(TQ_EINVAL, "%s: x_stride %lld (need >= d and a multiple of 8)", fn,
                     (long long)x_stride);
  if (out_stride < 1) return set_error(TQ_EINVAL, "%s: out_stride < 1", fn);
  if (N > 0 && (!x || !codes || !norms)) return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  TQ_CHECK_ALIGN(x, "x");
  TQ_CHECK_ALIGN(codes, "codes");
  TQ_CHECK_ALIGN(norms, "norms");
  return TQ_OK;
}

extern "C" int tq_quant_mse(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                            uint32_t* codes, float* norms, int64_t out_stride, void* stream) {
  TQ_TRACE("tq_quant_mse");
  int rc = check_quant_args("tq_quant_mse", h, TQ_MSE, x, dtype, N, x_stride, codes, norms, out_stride);
  if (rc) return rc;
  if (N == 0) return clear_error();
  int e = quant_tc_supported(h, dtype)
              ? launch_quant_mse_tc(h, x, N, x_stride, codes, norms, out_stride, stream)
          : quant_fused_supported(h)
              ? launch_quant_fused(h, x, dtype, N, x_stride, codes, nullptr, norms, nullptr, out_stride, stream)
          : quant_gen_supported(h)
              ? launch_quant_gen(h, x, dtype, N, x_stride, codes, nullptr, norms, nullptr, out_stride, nullptr, 0,
                                 stream)
              : launch_quant_simple(h, x, dtype, N, x_stride, codes, nullptr, norms, nullptr, out_stride, stream);
  return e ? cuda_error("tq_quant_mse", e) : clear_error();
}

static int quant_prod_impl(const char* fn, tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                           uint32_t* codes, uint32_t* signs, float* norms, float* rnorms, int64_t out_stride,
                           void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_quant_args(fn, h, TQ_PROD, x, dtype, N, x_stride, codes, norms, out_stride);
  if (rc) return rc;
  if (N > 0 && (!signs || !rnorms)) return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  TQ_CHECK_ALIGN(signs, "signs");
  TQ_CHECK_ALIGN(rnorms, "rnorms");
  TQ_CHECK_ALIGN(workspace, "workspace");
  if (N == 0) return clear_error();
  const bool need_ws = quant_gen_supported(h) && quant_gen_needs_workspace(h);
  if (need_ws && workspace && ws_bytes < (size_t)128 * quant_gen_workspace_rows_bytes(h))
    return set_error(TQ_EWORKSPACE, "%s: workspace of %zu bytes is below the %zu-byte minimum", fn, ws_bytes,
                     (size_t)128 * quant_gen_workspace_rows_bytes(h));
  // tensor cores unless this d needs the residual workspace and none was given
  const bool gen = quant_gen_supported(h) && (!need_ws || workspace);
  int e = quant_fused_supported(h)
              ? launch_quant_fused(h, x, dtype, N, x_stride, codes, signs, norms, rnorms, out_stride, stream)
          : gen ? launch_quant_gen(h, x, dtype, N, x_stride, codes, signs, norms, rnorms, out_stride, workspace,
                                 ws_bytes, stream)
              : launch_quant_simple(h, x, dtype, N, x_stride, codes, signs, norms, rnorms, out_stride, stream);
  return e ? cuda_error(fn, e) : clear_error();
}

extern "C" int tq_quant_prod(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                             uint32_t* codes, uint32_t* signs, float* norms, float* rnorms,
                             int64_t out_stride, void* stream) {
  TQ_TRACE("tq_quant_prod");
  return quant_prod_impl("tq_quant_prod", h, x, dtype, N, x_stride, codes, signs, norms, rnorms, out_stride,
                         nullptr, 0, stream);
}

extern "C" int tq_quant_prod_ws(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                                uint32_t* codes, uint32_t* signs, float* norms, float* rnorms, int64_t out_stride,
                                void* workspace, size_t ws_bytes, void* stream) {
  TQ_TRACE("tq_quant_prod_ws");
  return quant_prod_impl("tq_quant_prod_ws", h, x, dtype, N, x_stride, codes, signs, norms, rnorms, out_stride,
                         workspace, ws_bytes, stream);
}

extern "C" size_t tq_quant_prod_workspace(tq_handle h, int64_t N) {
  if (!h || N <= 0 || h->variant != TQ_PROD || !quant_gen_supported(h) || !quant_gen_needs_workspace(h)) return 0;
  // whole 128-row tiles, at most four per SM per launch
  const int64_t cap = (int64_t)4 * h->sm_count * 128;
  const int64_t rows = std::min((N + 127) / 128 * 128, cap);
  return (size_t)rows * quant_gen_workspace_rows_bytes(h);
}

extern "C" int tq_dequant_mse(tq_handle h, const uint32_t* codes, const float* norms, int64_t N,
                              void* out, int out_dtype, void* stream) {
  TQ_TRACE("tq_dequant_mse");
  if (!h) return set_error(TQ_EINVAL, "tq_dequant_mse: NULL handle");
  if (h->variant == TQ_POLAR) return set_error(TQ_EINVAL, "tq_dequant_mse: a TQ_POLAR handle (use tq_dequant_polar)");
  if (N < 0) return set_error(TQ_EINVAL, "tq_dequant_mse: N < 0");
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16)
    return set_error(TQ_EUNSUPPORTED, "tq_dequant_mse: out_dtype %d", out_dtype);
  if (N > 0 && (!codes || !norms || !out)) return set_error(TQ_EINVAL, "tq_dequant_mse: NULL pointer");
  TQ_CHECK_ALIGN(codes, "codes");
  TQ_CHECK_ALIGN(norms, "norms");
  TQ_CHECK_ALIGN(out, "out");
  if (N == 0) return clear_error();
  int e = dequant_tc_supported(h) ? launch_dequant_tc(h, codes, norms, N, out, out_dtype, stream)
                                  : launch_dequant_simple(h, codes, norms, N, out, out_dtype, stream);
  return e ? cuda_error("tq_dequant_mse", e) : clear_error();
}

// workspace of tq_ip_scores: rotated + projected queries, and the score matrix
// when only the top-k is requested
extern "C" size_t tq_ip_scores_workspace(tq_handle h, int64_t nq, int64_t N, int topk) {
  if (!h || nq < 0 || N < 0) return 0;
  size_t bytes = align_up((size_t)nq * h->d * 4, 256) * 2;
  if (topk > 0 && !scores_tc_supported(h, topk)) bytes += align_up((size_t)nq * N * 4, 256);
  if (scores_tc_supported(h, topk)) bytes = std::max(bytes, scores_tc_workspace(h, nq, N, topk));
  return bytes;
}

extern "C" int tq_ip_scores(tq_handle h, const float* q, int64_t nq, const uint32_t* codes,
                            const uint32_t* signs, const float* norms, const float* rnorms,
                            int64_t N, float* scores, int topk, int32_t* top_idx, float* top_val,
                            void* workspace, size_t ws_bytes, void* stream) {
  TQ_TRACE("tq_ip_scores");
  if (!h) return set_error(TQ_EINVAL, "tq_ip_scores: NULL handle");
  if (h->variant == TQ_POLAR) return set_error(TQ_EINVAL, "tq_ip_scores: a TQ_POLAR handle");
  if (nq < 0 || N < 0) return set_error(TQ_EINVAL, "tq_ip_scores: negative size");
  if (topk < 0 || topk > TQ_MAX_TOPK || (topk > 0 && topk > N && N > 0))
    return set_error(TQ_EINVAL, "tq_ip_scores: topk %d (need 0..min(N, %d))", topk, TQ_MAX_TOPK);
  const bool prod = h->variant == TQ_PROD;
  if (nq > 0 && N > 0) {
    if (!q || !codes || !norms || (prod && (!signs || !rnorms)))
      return set_error(TQ_EINVAL, "tq_ip_scores: NULL input");
    if (!scores && topk == 0) return set_error(TQ_EINVAL, "tq_ip_scores: no output requested");
    if (topk > 0 && (!top_idx || !top_val)) return set_error(TQ_EINVAL, "tq_ip_scores: NULL top-k output");
  }
  for (const void* p : {(const void*)q, (const void*)codes, (const void*)signs, (const void*)norms,
                        (const void*)rnorms, (const void*)scores, (const void*)top_idx,
                        (const void*)top_val, (const void*)workspace})
    TQ_CHECK_ALIGN(p, "a device pointer");
  if (nq == 0 || N == 0) return clear_error();
  const size_t need = tq_ip_scores_workspace(h, nq, N, topk);
  if (!workspace || ws_bytes < need)
    return set_error(TQ_EWORKSPACE, "tq_ip_scores: workspace %zu < %zu bytes", ws_bytes, need);
  if (scores_tc_supported(h, topk)) {
    int e = launch_scores_tc(h, q, nq, codes, signs, norms, rnorms, N, scores, topk, top_idx, top_val, workspace,
                             stream);
    return e ? cuda_error("tq_ip_scores", e) : clear_error();
  }
  char* ws = (char*)workspace;
  float* qrot = (float*)ws;
  float* qproj = (float*)(ws + align_up((size_t)nq * h->d * 4, 256));
  float* sc = scores;
  if (topk > 0 && !scores) sc = (float*)(ws + 2 * align_up((size_t)nq * h->d * 4, 256));
  int e = launch_query_prep(h, q, TQ_F32, nq, qrot, prod ? qproj : nullptr, stream);
  if (!e) e = launch_scores_simple(h, qrot, qproj, nq, codes, signs, norms, rnorms, N, sc, stream);
  if (!e && topk > 0) e = launch_topk_simple(sc, nq, N, topk, top_idx, top_val, stream);
  return e ? cuda_error("tq_ip_scores", e) : clear_error();
}

namespace tqi {

size_t decode_workspace_bytes(const tq_ctx* hk, int B, int Hq, int Hkv, int64_t T) {
  const size_t nq = (size_t)B * Hq;
  const size_t simple = nq * decode_splits(B, Hq, T, hk->sm_count) * (hk->d + 2) * 4;
  const size_t fast = (size_t)decode_mma_grid(B, Hkv, T, hk->sm_count) * decode_mma_max_seg(B, Hkv, T, hk->sm_count) *
                      4 * (hk->d + 2) * 4;
  const size_t tc = (size_t)decode_tc_grid(B, Hkv, T, hk->sm_count) * decode_tc_max_seg(B, Hkv, T, hk->sm_count) * 4 *
                    (hk->d + 2) * 4;
  const size_t qops = std::max(nq * 2 * hk->d * 2, decode_tc_qtile_bytes(B, Hkv));
  return 2 * align_up(nq * hk->d * 4, 256) + align_up(qops, 256) + align_up(nq * 2 * 4, 256) +
         align_up(std::max(simple, std::max(fast, tc)), 256);
}

// workspace: rotated queries | projected queries (fp32) | fp16 query operands (fragments, or the
// tcgen05 kernel's query tiles) | their scales | partials
int decode_dispatch(const tq_ctx* hk, const tq_ctx* hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
                    int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                    const float* knorms, const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                    float scale, float* out, void* workspace, void* stream, int partial_out, PagedCache pg) {
  const size_t nq = (size_t)B * Hq;
  char* ws = (char*)workspace;
  const size_t q32 = align_up(nq * hk->d * 4, 256);
  float* qrot = (float*)ws;
  float* qproj = (float*)(ws + q32);
  void* qfrag = ws + 2 * q32;
  const size_t qops = std::max(nq * 2 * hk->d * 2, decode_tc_qtile_bytes(B, Hkv));
  float* qscale = (float*)(ws + 2 * q32 + align_up(qops, 256));
  float* partials = (float*)((char*)qscale + align_up(nq * 2 * 4, 256));
  int e = launch_query_prep(hk, (const float*)q, q_dtype, (int64_t)nq, qrot, qproj, stream);
  if (e) return e;
  if (!pg.page && decode_tc_supported(hk, hv, Hq, Hkv, kv_stride, pg.rn16))
    return launch_decode_tc(hk, hv, qrot, qproj, (uint8_t*)qfrag, qscale, B, Hq, Hkv, T, kv_stride, kcodes, ksigns,
                            knorms, krnorms, vcodes, vnorms, scale, partials, out, stream, partial_out, pg.rn16);
  const bool mma = pg.page ? decode_mma_supported(hk, hv, Hq, Hkv, 4) && pg.page % 8 == 0
                            : decode_mma_supported(hk, hv, Hq, Hkv, kv_stride) && (!pg.rn16 || kv_stride % 8 == 0);
  if (mma) {
    e = launch_qfrag(qrot, qproj, (int64_t)nq, qfrag, qscale, stream);
    if (e) return e;
    return launch_decode_mma(hk, hv, (const uint32_t*)qfrag, qscale, B, Hq, Hkv, T, kv_stride, kcodes, ksigns,
                             knorms, krnorms, vcodes, vnorms, scale, partials, out, stream, partial_out, pg);
  }
  const int splits = decode_splits(B, Hq, T, hk->sm_count);
  return launch_decode_simple(hk, hv, qrot, qproj, B, Hq, Hkv, T, kv_stride, kcodes, ksigns, knorms, krnorms,
                              vcodes, vnorms, scale, splits, partials, out, stream, partial_out, pg);
}

}  // namespace tqi

extern "C" size_t tq_attn_decode_workspace(tq_handle hk, int B, int Hq, int Hkv, int64_t T) {
  if (!hk || B < 0 || Hq < 0 || Hkv <= 0 || T < 0) return 0;
  return decode_workspace_bytes(hk, B, Hq, Hkv, T);
}

extern "C" int tq_attn_decode(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int Hq,
                              int Hkv, int64_t T, int64_t kv_stride, const uint32_t* kcodes,
                              const uint32_t* ksigns, const float* knorms, const float* krnorms,
                              const uint32_t* vcodes, const float* vnorms, float scale, float* out,
                              void* workspace, size_t ws_bytes, void* stream) {
  TQ_TRACE("tq_attn_decode");
  if (!hk || !hv) return set_error(TQ_EINVAL, "tq_attn_decode: NULL handle");
  if (hk->variant != TQ_PROD || hv->variant != TQ_MSE)
    return set_error(TQ_EINVAL, "tq_attn_decode: need a TQ_PROD key handle and a TQ_MSE value handle");
  if (hk->d != hv->d) return set_error(TQ_EINVAL, "tq_attn_decode: key and value d differ");
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16)
    return set_error(TQ_EUNSUPPORTED, "tq_attn_decode: q_dtype %d", q_dtype);
  if (B < 0 || Hq < 0 || Hkv <= 0 || (Hq % Hkv) != 0 || T < 1 || kv_stride < T)
    return set_error(TQ_EINVAL, "tq_attn_decode: bad shape (B=%d Hq=%d Hkv=%d T=%lld stride=%lld)", B,
                     Hq, Hkv, (long long)T, (long long)kv_stride);
  if (!std::isfinite(scale)) return set_error(TQ_EINVAL, "tq_attn_decode: scale is not finite");
  if (B == 0 || Hq == 0) return clear_error();
  if (!q || !kcodes || !ksigns || !knorms || !krnorms || !vcodes || !vnorms || !out)
    return set_error(TQ_EINVAL, "tq_attn_decode: NULL pointer");
  for (const void* p : {(const void*)q, (const void*)kcodes, (const void*)ksigns, (const void*)knorms,
                        (const void*)krnorms, (const void*)vcodes, (const void*)vnorms,
                        (const void*)out, (const void*)workspace})
    TQ_CHECK_ALIGN(p, "a device pointer");
  const size_t need = tq_attn_decode_workspace(hk, B, Hq, Hkv, T);
  if (!workspace || ws_bytes < need)
    return set_error(TQ_EWORKSPACE, "tq_attn_decode: workspace %zu < %zu bytes", ws_bytes, need);
  int e = decode_dispatch(hk, hv, q, q_dtype, B, Hq, Hkv, T, kv_stride, kcodes, ksigns, knorms, krnorms, vcodes,
                          vnorms, scale, out, workspace, stream);
  return e ? cuda_error("tq_attn_decode", e) : clear_error();
}

extern "C" int tq_quant_polar(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride, uint32_t* codes,
                              float* norms, int64_t out_stride, void* stream) {
  TQ_TRACE("tq_quant_polar");
  int rc = check_quant_args("tq_quant_polar", h, TQ_POLAR, x, dtype, N, x_stride, codes, norms, out_stride);
  if (rc) return rc;
  if (N == 0) return clear_error();
  if (reinterpret_cast<uintptr_t>(x) & 15u) return set_error(TQ_EALIGN, "tq_quant_polar: x is not 16-byte aligned");
  const int e = launch_quant_fused2(h, x, dtype, N, x_stride, codes, nullptr, norms, nullptr, out_stride, stream,
                                    nullptr, 0);
  return e ? cuda_error("tq_quant_polar", e) : clear_error();
}

extern "C" int tq_dequant_polar(tq_handle h, const uint32_t* codes, const float* norms, int64_t N, void* out,
                                int out_dtype, void* stream) {
  TQ_TRACE("tq_dequant_polar");
  if (!h) return set_error(TQ_EINVAL, "tq_dequant_polar: NULL handle");
  if (h->variant != TQ_POLAR) return set_error(TQ_EINVAL, "tq_dequant_polar: need a TQ_POLAR handle");
  if (N < 0) return set_error(TQ_EINVAL, "tq_dequant_polar: N < 0");
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16)
    return set_error(TQ_EUNSUPPORTED, "tq_dequant_polar: out_dtype %d", out_dtype);
  if (N > 0 && (!codes || !norms || !out)) return set_error(TQ_EINVAL, "tq_dequant_polar: NULL pointer");
  TQ_CHECK_ALIGN(codes, "codes");
  TQ_CHECK_ALIGN(norms, "norms");
  TQ_CHECK_ALIGN(out, "out");
  if (N == 0) return clear_error();
  const int e = launch_dequant_tc(h, codes, norms, N, out, out_dtype, stream);
  return e ? cuda_error("tq_dequant_polar", e) : clear_error();
}

extern "C" int tq_quant_gather(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                               const int32_t* channels, uint32_t* codes, uint32_t* signs, float* norms,
                               float* rnorms, int64_t out_stride, void* stream) {
  TQ_TRACE("tq_quant_gather");
  if (!h) return set_error(TQ_EINVAL, "tq_quant_gather: NULL handle");
  if (h->variant == TQ_POLAR) return set_error(TQ_EINVAL, "tq_quant_gather: a TQ_POLAR handle");
  if (N < 0) return set_error(TQ_EINVAL, "tq_quant_gather: N < 0");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return set_error(TQ_EUNSUPPORTED, "tq_quant_gather: dtype %d", dtype);
  if (x_stride < 1 || out_stride < 1) return set_error(TQ_EINVAL, "tq_quant_gather: stride < 1");
  const bool prod = h->variant == TQ_PROD;
  if (N > 0 && (!x || !channels || !codes || !norms || (prod && (!signs || !rnorms))))
    return set_error(TQ_EINVAL, "tq_quant_gather: NULL pointer");
  // appends point at one token slot of a cache: element alignment is enough here
  for (const void* p : {(const void*)x, (const void*)channels, (const void*)codes, (const void*)signs,
                        (const void*)norms, (const void*)rnorms})
    if (reinterpret_cast<uintptr_t>(p) & 3u)
      return set_error(TQ_EALIGN, "tq_quant_gather: a device pointer is not 4-byte aligned");
  if (N == 0) return clear_error();
  // bulk gathers (a cache fill) on the tensor cores; a few arriving tokens in one short launch
  const bool bulk = N >= 256 && quant_fused_supported(h) && !(reinterpret_cast<uintptr_t>(x) & 15u);
  int e;
  if (bulk) {
    e = launch_quant_fused(h, x, dtype, N, x_stride, codes, prod ? signs : nullptr, norms, prod ? rnorms : nullptr,
                           out_stride, stream, channels);
  } else if (h->d <= 256 && N < 65536) {
    uint32_t* sg = prod ? signs : nullptr;
    float* rn = prod ? rnorms : nullptr;
    e = launch_quant_small(&h, 1, x, dtype, N, x_stride, channels, &codes, &sg, &norms, &rn, out_stride, stream);
  } else {
    e = launch_quant_simple(h, x, dtype, N, x_stride, codes, prod ? signs : nullptr, norms, prod ? rnorms : nullptr,
                            out_stride, stream, channels);
  }
  return e ? cuda_error("tq_quant_gather", e) : clear_error();
}

extern "C" int tq_quant_gather_groups(const tq_handle* h, int ngroups, const void* x, int dtype, int64_t N,
                                      int64_t x_stride, const int32_t* channels, uint32_t* const* codes,
                                      uint32_t* const* signs, float* const* norms, float* const* rnorms,
                                      int64_t out_stride, void* stream) {
  TQ_TRACE("tq_quant_gather_groups");
  const char* fn = "tq_quant_gather_groups";
  if (!h || ngroups < 1 || ngroups > 2) return set_error(TQ_EINVAL, "%s: need 1 or 2 groups", fn);
  if (N < 0 || N >= 65536) return set_error(TQ_EINVAL, "%s: N = %lld (need 0 <= N < 65536)", fn, (long long)N);
  if (dtype != TQ_F32 && dtype != TQ_BF16) return set_error(TQ_EUNSUPPORTED, "%s: dtype %d", fn, dtype);
  if (x_stride < 1 || out_stride < 1) return set_error(TQ_EINVAL, "%s: stride < 1", fn);
  if (!codes || !norms || (N > 0 && (!x || !channels))) return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  for (int g = 0; g < ngroups; ++g) {
    if (!h[g]) return set_error(TQ_EINVAL, "%s: NULL handle", fn);
    if (h[g]->variant == TQ_POLAR) return set_error(TQ_EINVAL, "%s: a TQ_POLAR handle", fn);
    if (h[g]->d > 256) return set_error(TQ_EUNSUPPORTED, "%s: d = %d (need <= 256)", fn, h[g]->d);
    const bool prod = h[g]->variant == TQ_PROD;
    if (!codes[g] || !norms[g] || (prod && (!signs || !rnorms || !signs[g] || !rnorms[g])))
      return set_error(TQ_EINVAL, "%s: NULL pointer of group %d", fn, g);
    for (const void* p : {(const void*)codes[g], (const void*)norms[g], prod ? (const void*)signs[g] : nullptr,
                          prod ? (const void*)rnorms[g] : nullptr})
      if (reinterpret_cast<uintptr_t>(p) & 3u) return set_error(TQ_EALIGN, "%s: a pointer is not 4-byte aligned", fn);
  }
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(channels)) & 3u)
    return set_error(TQ_EALIGN, "%s: a pointer is not 4-byte aligned", fn);
  if (N == 0) return clear_error();
  uint32_t* sg[2] = {nullptr, nullptr};
  float* rn[2] = {nullptr, nullptr};
  for (int g = 0; g < ngroups; ++g)
    if (h[g]->variant == TQ_PROD) sg[g] = signs[g], rn[g] = rnorms[g];
  const tq_ctx* hs[2] = {h[0], ngroups > 1 ? h[1] : nullptr};
  const int e = launch_quant_small(hs, ngroups, x, dtype, N, x_stride, channels, codes, sg, norms, rn, out_stride,
                                   stream);
  return e ? cuda_error(fn, e) : clear_error();
}

extern "C" size_t tq_attn_logits_workspace(const tq_handle* hk, int ngroups, int B, int Hq) {
  if (!hk || ngroups < 1 || ngroups > 2 || B < 0 || Hq < 0) return 0;
  size_t bytes = 0;
  for (int g = 0; g < ngroups; ++g) {
    if (!hk[g]) return 0;
    bytes += 2 * align_up((size_t)B * Hq * hk[g]->d * 4, 256);
  }
  // fp16 query operands of the tensor-core paths (fragments, or query tiles)
  if (ngroups == 2) bytes += std::max(logits_mma_workspace((int64_t)B * Hq), logits_tc_workspace(B, (Hq + 3) / 4));
  return bytes;
}

extern "C" int tq_attn_logits(const tq_handle* hk, int ngroups, const int32_t* channels, const void* q, int q_dtype,
                              int dq, int B, int Hq, int Hkv, int64_t T, int64_t kv_stride,
                              const uint32_t* const* kcodes, const uint32_t* const* ksigns,
                              const float* const* knorms, const float* const* krnorms, float scale, float* logits,
                              void* workspace, size_t ws_bytes, void* stream) {
  TQ_TRACE("tq_attn_logits");
  if (!hk || ngroups < 1 || ngroups > 2) return set_error(TQ_EINVAL, "tq_attn_logits: need 1 or 2 groups");
  int dsum = 0;
  for (int g = 0; g < ngroups; ++g) {
    if (!hk[g] || hk[g]->variant != TQ_PROD) return set_error(TQ_EINVAL, "tq_attn_logits: need TQ_PROD handles");
    dsum += hk[g]->d;
  }
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16)
    return set_error(TQ_EUNSUPPORTED, "tq_attn_logits: q_dtype %d", q_dtype);
  if (B < 0 || Hq < 0 || Hkv <= 0 || Hq != 4 * Hkv || T < 0 || kv_stride < T)
    return set_error(TQ_EUNSUPPORTED, "tq_attn_logits: need Hq = 4 Hkv and kv_stride >= T");
  if (!channels && (ngroups != 1 || dq != hk[0]->d))
    return set_error(TQ_EINVAL, "tq_attn_logits: channels may be NULL only for one group with dq = d");
  if (channels && dq < 1) return set_error(TQ_EINVAL, "tq_attn_logits: dq < 1");
  (void)dsum;
  if (!std::isfinite(scale)) return set_error(TQ_EINVAL, "tq_attn_logits: scale is not finite");
  if (!logits_supported(hk, ngroups))
    return set_error(TQ_EUNSUPPORTED, "tq_attn_logits: groups must be d = 64 (two groups) or 64/128 (one), mse bits 1..3");
  if (B == 0 || Hq == 0 || T == 0) return clear_error();
  if (!q || !logits || !kcodes || !ksigns || !knorms || !krnorms)
    return set_error(TQ_EINVAL, "tq_attn_logits: NULL pointer");
  for (int g = 0; g < ngroups; ++g) {
    if (!kcodes[g] || !ksigns[g] || !knorms[g] || !krnorms[g]) return set_error(TQ_EINVAL, "tq_attn_logits: NULL pointer");
    for (const void* p : {(const void*)kcodes[g], (const void*)ksigns[g], (const void*)knorms[g],
                          (const void*)krnorms[g]})
      TQ_CHECK_ALIGN(p, "a device pointer");
  }
  for (const void* p : {(const void*)q, (const void*)logits, (const void*)channels, (const void*)workspace})
    TQ_CHECK_ALIGN(p, "a device pointer");
  const size_t need = tq_attn_logits_workspace(hk, ngroups, B, Hq);
  if (!workspace || ws_bytes < need)
    return set_error(TQ_EWORKSPACE, "tq_attn_logits: workspace %zu < %zu bytes", ws_bytes, need);
  const float* qr[2] = {nullptr, nullptr};
  const float* qp[2] = {nullptr, nullptr};
  char* ws = (char*)workspace;
  int off = 0;
  int e = 0;
  for (int g = 0; g < ngroups && !e; ++g) {
    const size_t qb = align_up((size_t)B * Hq * hk[g]->d * 4, 256);
    float* r = (float*)ws;
    float* p = (float*)(ws + qb);
    ws += 2 * qb;
    e = launch_query_prep_gather(hk[g], q, q_dtype, (int64_t)B * Hq, dq, channels ? channels + off : nullptr, r, p,
                                 stream);
    qr[g] = r;
    qp[g] = p;
    off += hk[g]->d;
  }
  if (!e) {
    if (logits_tc_supported(hk, ngroups, kv_stride))
      e = launch_logits_tc(hk, qr, qp, B, Hq, Hkv, T, kv_stride, kcodes, ksigns, knorms, krnorms, scale, logits, ws,
                           stream);
    else if (logits_mma_supported(hk, ngroups, kv_stride))
      e = launch_logits_mma(hk, qr, qp, B, Hq, Hkv, T, kv_stride, kcodes, ksigns, knorms, krnorms, scale, logits, ws,
                            stream);
    else
      e = launch_logits(hk, ngroups, qr, qp, B, Hq, Hkv, T, kv_stride, kcodes, ksigns, knorms, krnorms, scale,
                        logits, stream);
  }
  return e ? cuda_error("tq_attn_logits", e) : clear_error();
}
