// TurboQuant quantization of one 128-vector tile per step, both contractions
// fused in one persistent kernel, for dimensions up to 256 (sm_100a).
//
// [ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: store the norm,
// rotate, quantize every coordinate against the Lloyd-Max codebook; for
// TurboQuant_prod keep the 1-bit signs of the projected residual and its norm.
// Both steps are plain matrix products
// (ttakun.com/news/45354, "为什么随机旋转是整个算法的底层杠杆").
//
// Per tile of 128 vectors (M = 128 rows of every MMA):
//   rotation   Y = (s X) (2^10 Pi)^T         N = d rounded up to 16, one MMA per
//                                            16-wide K step; accumulator in TMEM
//                                            columns [0, 256)
//   epilogue   codes of y against s n 2^10 t_k; u = y / (s n 2^10) - c[idx] (the
//              residual in the unit frame, exact in fp32); ||r|| = n ||u||; u is
//              written (x 2^12, fp16 hi + lo) straight into the operand ring the
//              tensor core reads next -- it never leaves the SM
//   projection V = (2^12 U) (2^10 T)^T, T = S Pi^T; sign bits of V are the QJL
//              bits of S r = n T u.  Accumulator in TMEM columns [256, 512)
// so x is read from HBM once (by the producers) and nothing but the outputs is
// written.  The norms come from gen_norms_kernel (float64 sums) before this
// kernel; s = 2^(14 - e) with n = f 2^e, f in [0.5, 1), keeps s x below 2^14.
//
// Split precision with one accumulator: every fp32 operand v is carried as
// v_hi = fp16(v) and v_lo = fp16(v - v_hi) (the remainder itself, not rescaled),
// and hi.hi + hi.lo + lo.hi accumulate into the same fp32 TMEM accumulator,
// a relative error of about 2^-22 per product.  The constant pieces are of
// 2^10 Pi and 2^10 T so that their remainders stay fp16-normal.  bf16 input is
// exact in fp16 after the power-of-two scaling: its lo piece is zero and that
// product is skipped.
//
// Warp roles (448 threads, one CTA per SM):
//   warp 0       TMA producer of the constant pieces: [N16 x 64] fp16 boxes
//                (hi and lo) of Pi, then of T, per 64-wide K chunk
//   warp 1       TMEM allocation and the single-thread MMA issuer
//   warps 2-5    x producers: coalesced loads of the tile, s x -> fp16 hi/lo in
//                128B-swizzled K-major [128 x 64] tiles of the operand ring
//   warps 6-13   epilogue: warp % 4 = TMEM lane quarter (32 vectors), warps
//                6-9 take the even 32-coordinate groups, 10-13 the odd ones
// The operand ring carries, per tile, the K chunks of s X and then (prod) the
// K chunks of 2^12 U; the constant ring the chunks of Pi and then T.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>

#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;

constexpr int kTM = 128;                 // vectors per tile
constexpr int kThreads = 448;
constexpr int kPieceA = kTM * 128;       // one [128 x 64] fp16 tile
constexpr int kAStageBytes = 2 * kPieceA;  // hi + lo
constexpr int kBStages = 2;
constexpr int kYCol = 0, kVCol = 256;    // TMEM columns of the two accumulators
constexpr float kUScale = 4096.f;        // residual coordinates scaled into fp16's range
constexpr int kMiscBytes = 4096;

struct FzArgs {
  const void* x;
  int64_t x_stride;
  int xbf16;
  int64_t N;
  int d, n16, kc, G, W;      // n16 = d rounded up to 16, kc = 64-wide K chunks, G = 32-groups, W = code words
  int64_t out_stride;
  int prod;
  const float* norms;        // written by gen_norms_kernel
  uint32_t* codes;
  uint32_t* signs;
  float* rnorms;
  const float* thresholds;   // [2^bm - 1]
  const float* centroids;    // [2^bm]
  float acc_scale;           // 2^10: scale of the constant pieces
  int a_stages;              // operand ring depth (2 or 3)
  int b_stage_bytes;         // 2 * n16 * 128
  int64_t row_tiles;
  const int32_t* channels;   // optional: vector i is (x_i[channels[0]], .., x_i[channels[d-1]])
  const int64_t* slots;      // optional: vector i's outputs go to row slots[i] (else i * out_stride)
  int rn_f16;                // residual norms stored as fp16 (rnorms points at __half)
  int* status;
};

// output row of vector v
__device__ __forceinline__ int64_t out_row(const FzArgs& a, int64_t v) {
  return a.slots ? a.slots[v] : v * a.out_stride;
}

__host__ __device__ __forceinline__ int64_t first_tile(int64_t i, int64_t total, int64_t G) { return i * total / G; }

__device__ __forceinline__ float vec_scale(float n) {
  if (!(n > 0.f)) return 1.f;
  int e;
  (void)frexpf(n, &e);
  return ldexpf(1.f, 14 - e);
}

__device__ __forceinline__ uint32_t half2_bits(__half a, __half b) {
  return (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
}

// byte offset of element (row r, column c) of a [rows x 64] fp16 tile, 128B swizzle
__device__ __forceinline__ int sw_off(int r, int c) { return r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + (c & 7) * 2; }

__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t cnt) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(cnt) : "memory");
}

// number of 16-wide K steps of chunk k that hold coordinates below d
__device__ __forceinline__ int k_steps(int d, int k) {
  const int rem = d - 64 * k;
  return rem >= 64 ? 4 : (rem + 15) / 16;
}

template <int BM>
__device__ __forceinline__ uint32_t cell_of(float y, const float (&P)[8]) {
  // P[m] = m-th positive threshold in the accumulator's frame (m = 1 .. 2^(BM-1) - 1)
  constexpr uint32_t H = 1u << (BM - 1);
  const float a = fabsf(y);
  uint32_t m = 0;
  if constexpr (BM == 2) {
    m = (a >= P[1]) ? 1u : 0u;
  } else if constexpr (BM == 3) {
    const uint32_t m1 = (a >= P[2]) ? 1u : 0u;
    m = 2u * m1 + ((a >= (m1 ? P[3] : P[1])) ? 1u : 0u);
  } else if constexpr (BM == 4) {
    const uint32_t m2 = (a >= P[4]) ? 1u : 0u;
    const uint32_t m1 = (a >= (m2 ? P[6] : P[2])) ? 1u : 0u;
    const float t2 = m2 ? (m1 ? P[7] : P[5]) : (m1 ? P[3] : P[1]);
    m = 4u * m2 + 2u * m1 + ((a >= t2) ? 1u : 0u);
  }
  return ((y >= 0.f) ? H : H - 1u) ^ m;
}

// the 32 cells of a group into its BM words (layout of include/tq.h)
template <int BM>
__device__ __forceinline__ void pack_group(const uint32_t (&c)[32], uint32_t (&w)[BM]) {
#pragma unroll
  for (int k = 0; k < BM; ++k) w[k] = 0u;
  if constexpr (BM == 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[0] |= c[i] << i;
  } else if constexpr (BM == 2) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i >> 4] |= c[i] << (2 * (i & 15));
  } else if constexpr (BM == 4) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i >> 3] |= c[i] << (4 * (i & 7));
  } else {
#pragma unroll
    for (int i = 0; i < 24; ++i) w[i >> 3] |= c[i] << (4 * (i & 7));
    uint32_t X = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) X |= c[24 + j] << (4 * j);
    w[0] |= (X << 3) & 0x88888888u;
    w[1] |= (X << 2) & 0x88888888u;
    w[2] |= (X << 1) & 0x88888888u;
  }
}

template <int BM>
__global__ void __launch_bounds__(kThreads, 1) quant_fused_kernel(const __grid_constant__ CUtensorMap pimap,
                                                                  const __grid_constant__ CUtensorMap tmap, FzArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem;                                    // [a_stages][hi, lo]
  uint8_t* b_s = a_s + a.a_stages * kAStageBytes;         // [kBStages][hi, lo]
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_s + kBStages * a.b_stage_bytes);
  uint64_t* a_full = bars;                 // [3]  count 256 (x producers arrive with 2 each, epilogue with 1)
  uint64_t* a_empty = a_full + 3;          // [3]  MMA commit
  uint64_t* b_full = a_empty + 3;          // [2]  TMA bytes
  uint64_t* b_empty = b_full + kBStages;   // [2]  MMA commit
  uint64_t* y_full = b_empty + kBStages;   // MMA commit
  uint64_t* y_empty = y_full + 1;          // 8 epilogue warps
  uint64_t* v_full = y_empty + 1;
  uint64_t* v_empty = v_full + 1;
  uint64_t* rn_bar = v_empty + 1;          // [2] count 256
  uint64_t* done_bar = rn_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  float* thr_s = reinterpret_cast<float*>(tmem_slot + 4);  // [16]
  float* cen_s = thr_s + 16;                               // [16]
  float* rn_s = cen_s + 16;                                // [2 parity][2 halves][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t Gc = gridDim.x;
  const int64_t t_lo = first_tile(blockIdx.x, a.row_tiles, Gc);
  const int64_t t_hi = first_tile(blockIdx.x + 1, a.row_tiles, Gc);
  const int kc = a.kc;
  const int per_tile = a.prod ? 2 * kc : kc;   // ring entries per tile (both rings)
  const int AS = a.a_stages;
  constexpr int K = 1 << BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 3; ++s) {
      mbar_init(&a_full[s], 256);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(y_full, 1);
    mbar_init(y_empty, 8);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 8);
    mbar_init(&rn_bar[0], 256);
    mbar_init(&rn_bar[1], 256);
    mbar_init(done_bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < K - 1) thr_s[threadIdx.x] = a.thresholds[threadIdx.x];
  if (threadIdx.x < K) cen_s[threadIdx.x] = a.centroids[threadIdx.x];
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer of the constant pieces
    if (lane == 0) {
      int64_t seq = 0, issued = 0;
      bool ok = true;
      const uint32_t bytes = (uint32_t)a.b_stage_bytes;
      for (int64_t t = t_lo; ok && t < t_hi; ++t) {
        for (int e = 0; e < per_tile; ++e, ++seq) {
          const int s = (int)(seq % kBStages);
          if (!mbar_wait(&b_empty[s], (uint32_t)(((seq / kBStages) & 1) ^ 1))) {
            ok = false;
            break;
          }
          const CUtensorMap* map = e < kc ? &pimap : &tmap;
          const int k = e < kc ? e : e - kc;
          uint8_t* dst = b_s + s * a.b_stage_bytes;
          mbar_arrive_expect_tx(&b_full[s], bytes);
          tma_load_2d(map, &b_full[s], dst, 64 * k, 0);
          tma_load_2d(map, &b_full[s], dst + bytes / 2, 64 * k, a.n16);
          issued = seq + 1;
        }
      }
      // every copy issued into this CTA's shared memory lands before it exits
      for (int64_t q = issued - kBStages > 0 ? issued - kBStages : 0; q < issued; ++q)
        if (!mbar_wait(&b_full[q % kBStages], (uint32_t)((q / kBStages) & 1))) ok = false;
      if (!ok) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kTM, a.n16, false);
      const uint32_t aaddr = smem_u32(a_s), baddr = smem_u32(b_s);
      const bool x_lo = !a.xbf16;
      int64_t seq = 0;
      bool ok = true;
      int i = 0;
      for (int64_t t = t_lo; ok && t < t_hi; ++t, ++i) {
        for (int ph = 0; ok && ph < (a.prod ? 2 : 1); ++ph) {
          uint64_t* acc_empty = ph ? v_empty : y_empty;
          if (!mbar_wait(acc_empty, (uint32_t)((i & 1) ^ 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t acc = tmem_base + (uint32_t)(ph ? kVCol : kYCol);
          const bool has_lo = ph ? true : x_lo;
          for (int k = 0; k < kc; ++k, ++seq) {
            const int sa = (int)(seq % AS), sb = (int)(seq % kBStages);
            if (!mbar_wait(&a_full[sa], (uint32_t)((seq / AS) & 1)) ||
                !mbar_wait(&b_full[sb], (uint32_t)((seq / kBStages) & 1))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t ah = aaddr + sa * kAStageBytes, al = ah + kPieceA;
            const uint32_t bh = baddr + sb * a.b_stage_bytes, bl = bh + a.b_stage_bytes / 2;
            const int nk = k_steps(a.d, k);
            for (int k4 = 0; k4 < nk; ++k4) {
              const uint64_t dah = sw128_kmajor_desc(ah + k4 * 32), dbh = sw128_kmajor_desc(bh + k4 * 32);
              mma_f16(acc, dah, dbh, idesc, (k | k4) != 0 ? 1u : 0u);
              mma_f16(acc, dah, sw128_kmajor_desc(bl + k4 * 32), idesc, 1u);
              if (has_lo) mma_f16(acc, sw128_kmajor_desc(al + k4 * 32), dbh, idesc, 1u);
            }
            mma_commit(&a_empty[sa]);
            mma_commit(&b_empty[sb]);
          }
          if (!ok) break;
          mma_commit(ph ? v_full : y_full);
        }
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done_bar);
    }
  } else if (warp < 6) {
    // ---------------- x producers: s x -> fp16 hi/lo tiles
    const int wl = warp - 2;  // 0..3
    int64_t seq = 0;
    bool ok = true;
    for (int64_t t = t_lo; ok && t < t_hi; ++t) {
      const int64_t row0 = t * kTM;
      float sc[16];
      if (a.xbf16) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t v = row0 + 4 * (wl * 8 + i) + (lane >> 3);
          sc[i] = v < a.N ? vec_scale(a.norms[out_row(a, v)]) : 0.f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int64_t v = row0 + 2 * (wl * 16 + i) + (lane >> 4);
          sc[i] = v < a.N ? vec_scale(a.norms[out_row(a, v)]) : 0.f;
        }
      }
      for (int k = 0; k < kc; ++k, ++seq) {
        const int s = (int)(seq % AS);
        if (!mbar_wait_warp(&a_empty[s], (uint32_t)(((seq / AS) & 1) ^ 1))) {
          ok = false;
          break;
        }
        uint8_t* th = a_s + s * kAStageBytes;
        uint8_t* tl = th + kPieceA;
        if (a.xbf16) {
          const int c8 = (lane & 7) * 8;
          const int col = 64 * k + c8;
          uint4 v[8];
          if (a.channels) {  // gathered: eight 2-byte loads per 16-byte unit
            int ch[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) ch[q] = col < a.d ? a.channels[col + q] : 0;
            const uint16_t* xs = static_cast<const uint16_t*>(a.x);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int64_t r = row0 + 4 * (wl * 8 + i) + (lane >> 3);
              uint32_t w[4] = {0u, 0u, 0u, 0u};
              if (r < a.N && col < a.d) {
#pragma unroll
                for (int q = 0; q < 8; ++q) w[q >> 1] |= (uint32_t)xs[r * a.x_stride + ch[q]] << (16 * (q & 1));
              }
              v[i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int64_t r = row0 + 4 * (wl * 8 + i) + (lane >> 3);
              v[i] = (r < a.N && col < a.d)
                         ? *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.x) + r * a.x_stride + col)
                         : make_uint4(0u, 0u, 0u, 0u);
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * (wl * 8 + i) + (lane >> 3);
            const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float f0 = __uint_as_float(w4[q] << 16) * sc[i];
              const float f1 = __uint_as_float(w4[q] & 0xFFFF0000u) * sc[i];
              o[q] = half2_bits(__float2half_rn(f0), __float2half_rn(f1));
            }
            *reinterpret_cast<uint4*>(th + sw_off(rr, c8)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else {
          const int c4 = (lane & 15) * 4;
          const int col = 64 * k + c4;
#pragma unroll
          for (int bt = 0; bt < 2; ++bt) {  // two batches of 8 rows in flight
            float4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int64_t r = row0 + 2 * (wl * 16 + 8 * bt + i) + (lane >> 4);
              if (!(r < a.N && col < a.d)) {
                v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
              } else if (a.channels) {  // gathered: four 4-byte loads
                const float* xr = static_cast<const float*>(a.x) + r * a.x_stride;
                v[i] = make_float4(xr[a.channels[col]], xr[a.channels[col + 1]], xr[a.channels[col + 2]],
                                   xr[a.channels[col + 3]]);
              } else {
                v[i] = *reinterpret_cast<const float4*>(static_cast<const float*>(a.x) + r * a.x_stride + col);
              }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int rr = 2 * (wl * 16 + 8 * bt + i) + (lane >> 4);
              const float sv = sc[8 * bt + i];
              const float f[4] = {v[i].x * sv, v[i].y * sv, v[i].z * sv, v[i].w * sv};
              __half hi[4], lo[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                hi[q] = __float2half_rn(f[q]);
                lo[q] = __float2half_rn(f[q] - __half2float(hi[q]));
              }
              *reinterpret_cast<uint2*>(th + sw_off(rr, c4)) =
                  make_uint2(half2_bits(hi[0], hi[1]), half2_bits(hi[2], hi[3]));
              *reinterpret_cast<uint2*>(tl + sw_off(rr, c4)) =
                  make_uint2(half2_bits(lo[0], lo[1]), half2_bits(lo[2], lo[3]));
            }
          }
        }
        fence_async_smem();
        mbar_arrive_cnt(&a_full[s], 2);
      }
      if (a.prod) seq += kc;  // the residual chunks of this tile are filled by the epilogue
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  } else {
    // ---------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 6) >> 2;   // 0: even groups, 1: odd groups
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float P[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) P[m] = 0.f;
    int64_t seq = 0;
    int i = 0;
    bool ok = true;
    for (int64_t t = t_lo; ok && t < t_hi; ++t, ++i) {
      const int64_t vec = t * kTM + row;
      const bool live = vec < a.N;
      const int64_t orow = live ? out_row(a, vec) : 0;
      const float n = live ? a.norms[orow] : 0.f;
      const float ns = n * vec_scale(n) * a.acc_scale;   // the accumulator holds ns * y_unit
      const float inv_ns = n > 0.f ? 1.f / ns : 0.f;
#pragma unroll
      for (int m = 1; m < 8; ++m)
        if (m < (1 << (BM - 1))) P[m] = n > 0.f ? ns * thr_s[(1 << (BM - 1)) - 1 + m] : INFINITY;
      float u2 = 0.f;
      if (!mbar_wait_warp(y_full, (uint32_t)(i & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      seq += kc;  // this tile's x chunks
      for (int k = 0; k < kc; ++k) {
        const int g = 2 * k + half;  // warp-uniform
        const int jg = 32 * g;
        float v[32];
        uint32_t uh[16], ul[16];
        if (g < a.G) {
          tmem_ld32(tmem_base + lane_base + (uint32_t)(kYCol + jg), v);
          tmem_wait_ld();
          uint32_t c[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const bool in = jg + e < a.d;
            c[e] = in ? cell_of<BM>(v[e], P) : 0u;
          }
          if (live) {
            uint32_t w[BM];
            pack_group<BM>(c, w);
            uint32_t* dst = a.codes + orow * a.W + g * BM;
#pragma unroll
            for (int q = 0; q < BM; ++q) dst[q] = w[q];
          }
          if (a.prod) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float us[2];
#pragma unroll
              for (int o = 0; o < 2; ++o) {
                const bool in = jg + e + o < a.d && n > 0.f;
                const float u = in ? fmaf(v[e + o], inv_ns, -cen_s[c[e + o]]) : 0.f;
                u2 = fmaf(u, u, u2);
                us[o] = u * kUScale;
              }
              const __half h0 = __float2half_rn(us[0]), h1 = __float2half_rn(us[1]);
              uh[e >> 1] = half2_bits(h0, h1);
              ul[e >> 1] = half2_bits(__float2half_rn(us[0] - __half2float(h0)),
                                      __float2half_rn(us[1] - __half2float(h1)));
            }
          }
        }
        if (a.prod) {
          // the residual chunk k of this tile into the operand ring
          const int s = (int)(seq % AS);
          if (!mbar_wait_warp(&a_empty[s], (uint32_t)(((seq / AS) & 1) ^ 1))) {
            ok = false;
            break;
          }
          if (g < a.G) {
            uint8_t* th = a_s + s * kAStageBytes;
            uint8_t* tl = th + kPieceA;
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // 8 coordinates per 16-byte unit
              const int off = sw_off(row, 32 * half + 8 * q);
              *reinterpret_cast<uint4*>(th + off) = make_uint4(uh[4 * q], uh[4 * q + 1], uh[4 * q + 2], uh[4 * q + 3]);
              *reinterpret_cast<uint4*>(tl + off) = make_uint4(ul[4 * q], ul[4 * q + 1], ul[4 * q + 2], ul[4 * q + 3]);
            }
          }
          fence_async_smem();
          mbar_arrive(&a_full[s]);
          ++seq;
        }
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(y_empty);
      if (!a.prod) continue;
      // ||r|| = n ||u||: the two halves of every row meet in shared memory
      float* rs = rn_s + (i & 1) * 256;
      rs[half * 128 + row] = u2;
      mbar_arrive(&rn_bar[i & 1]);
      if (!mbar_wait_warp(&rn_bar[i & 1], (uint32_t)((i >> 1) & 1))) {
        ok = false;
        break;
      }
      if (half == 0 && live) {
        const float rn = n > 0.f ? n * sqrtf(rs[row] + rs[128 + row]) : 0.f;
        if (a.rn_f16)
          reinterpret_cast<__half*>(a.rnorms)[orow] = __float2half_rn(rn);
        else
          a.rnorms[orow] = rn;
      }
      // QJL bits from the projection
      if (!mbar_wait_warp(v_full, (uint32_t)(i & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int k = 0; k < kc; ++k) {
        const int g = 2 * k + half;
        if (g >= a.G) break;
        const int jg = 32 * g;
        float v[32];
        tmem_ld32(tmem_base + lane_base + (uint32_t)(kVCol + jg), v);
        tmem_wait_ld();
        uint32_t w = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) w |= ((v[e] >= 0.f && jg + e < a.d) ? 1u : 0u) << e;
        if (live) a.signs[orow * a.G + g] = w;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(v_empty);
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  }

  __syncthreads();
  if (warp == 1) {
    if (!mbar_wait(done_bar, 0) && lane == 0) atomicOr(a.status, kStatusTimeout);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

bool make_piece_map(CUtensorMap* m, const void* base, int k64, int n16) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t gdim[2] = {(cuuint64_t)k64, (cuuint64_t)(2 * n16)};
  const cuuint64_t gstride[1] = {(cuuint64_t)k64 * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)n16};
  const cuuint32_t estride[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int fused_smem_bytes(int n16, int* a_stages) {
  const int b = kBStages * 2 * n16 * 128;
  int as = 3;
  while (as > 2 && as * kAStageBytes + b + kMiscBytes + 1024 > 227 * 1024) --as;
  *a_stages = as;
  return as * kAStageBytes + b + kMiscBytes + 1024;
}

}  // namespace

bool quant_fused_supported(const tq_ctx* h) { return h->dev.fz_pi != nullptr; }

int launch_quant_fused(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride, uint32_t* codes,
                       uint32_t* signs, float* norms, void* rnorms, int64_t out_stride, void* stream,
                       const int32_t* channels, const int64_t* slots, int rn_f16) {
  // contiguous rows: the TMA-staged kernel; a channel gather stays on this one
  const int esz = dtype == TQ_BF16 ? 2 : 4;
  if (!channels && !(reinterpret_cast<uintptr_t>(x) & 15u) && (x_stride * esz) % 16 == 0 && !h->fused_register_loads)
    return launch_quant_fused2(h, x, dtype, N, x_stride, codes, signs, norms, rnorms, out_stride, stream, slots,
                               rn_f16);
  cudaStream_t s = (cudaStream_t)stream;
  const bool prod = h->variant == TQ_PROD;
  if (int e = launch_gen_norms(h, x, dtype, N, x_stride, norms, out_stride, stream, channels, slots)) return e;
  FzArgs a;
  a.x = x;
  a.x_stride = x_stride;
  a.xbf16 = dtype == TQ_BF16 ? 1 : 0;
  a.N = N;
  a.d = h->d;
  a.n16 = h->fz_n16;
  a.kc = h->fz_k64 / 64;
  a.G = (h->d + 31) / 32;
  a.W = a.G * h->bm;
  a.out_stride = out_stride;
  a.prod = prod ? 1 : 0;
  a.norms = norms;
  a.codes = codes;
  a.signs = prod ? signs : nullptr;
  a.rnorms = prod ? static_cast<float*>(rnorms) : nullptr;
  a.channels = channels;
  a.slots = slots;
  a.rn_f16 = rn_f16;
  a.thresholds = h->dev.thresholds;
  a.centroids = h->dev.centroids;
  a.acc_scale = kFusedPieceScale;
  const int smem = fused_smem_bytes(a.n16, &a.a_stages);
  a.b_stage_bytes = 2 * a.n16 * 128;
  a.row_tiles = (N + kTM - 1) / kTM;
  a.status = h->dev.status;
  CUtensorMap pm, tm;
  if (!make_piece_map(&pm, h->dev.fz_pi, h->fz_k64, a.n16)) return (int)cudaErrorInvalidValue;
  if (!make_piece_map(&tm, prod ? h->dev.fz_t : h->dev.fz_pi, h->fz_k64, a.n16)) return (int)cudaErrorInvalidValue;
  const int grid = (int)(a.row_tiles < h->sm_count ? a.row_tiles : h->sm_count);
  auto go = [&](auto kern) -> int {
    if (int e = ensure_dyn_smem((const void*)kern, smem)) return e;
    kern<<<grid, kThreads, smem, s>>>(pm, tm, a);
    return (int)cudaGetLastError();
  };
  switch (h->bm) {
    case 1: return go(quant_fused_kernel<1>);
    case 2: return go(quant_fused_kernel<2>);
    case 3: return go(quant_fused_kernel<3>);
    default: return go(quant_fused_kernel<4>);
  }
}

}  // namespace tqi
