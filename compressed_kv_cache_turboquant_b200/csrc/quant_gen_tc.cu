// TurboQuant quantization of any dimension on the tensor cores (sm_100a):
// TurboQuant_mse and TurboQuant_prod, fp32 or bf16 input.
//
// [ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: store the norm,
// rotate, quantize each coordinate against the Lloyd-Max codebook; the prod
// variant quantizes the residual r = x - x_hat to the signs of S r and stores
// ||r||.  Both rotations are plain matrix products
// (ttakun.com/news/45354, "为什么随机旋转是整个算法的底层杠杆").
//
// Three launches:
//   gen_norms_kernel     n = ||x|| (float64 accumulation) -> the norms output.
//                        Every later stage derives the vector's scale from it:
//                        s = 2^(14 - e), n = f 2^e with f in [0.5, 1), so every
//                        entry of s x lies below 2^14 (fp16 range).
//   quant_gen_kernel<1>  Y = (s X) Pi^T; codes against s n t_k; ||r|| = n ||y - c[idx]||
//   quant_gen_kernel<2>  (prod, d_pad <= 256) V = (s X) S^T - (s n C) T^T = s S r
//                        (T = S Pi^T, C = c[idx] from the codes of stage 1); sign
//                        bits of V.  S x - n T c[idx] = S (x - x_hat) needs no
//                        residual buffer, but both terms are of size ||x|| and
//                        cancel to ||r||: the fp32 accumulation error grows with
//                        sqrt(d) ||x|| while the bit is the sign of a value of
//                        size ||r||.
//   quant_gen_kernel<3>  (prod, larger d, with a caller workspace) stage 1 also
//                        writes u = y - c[idx] (unit frame, x 2^12, fp16 hi/lo
//                        rows); V = U T^T = 2^12 T u, whose partial sums are of
//                        size ||u|| instead of ||x||.
// Split precision (fp16 pieces, the low piece scaled by 2^11 to stay normal):
//   A = A_hi + 2^-11 A_lo,  B = B_hi + 2^-11 B_lo
//   acc0 = A_hi B_hi,  acc1 = A_hi B_lo + A_lo B_hi,  A B = acc0 + 2^-11 acc1
// with relative error ~2^-21 per product.  bf16 input is exact in fp16 after
// the power-of-two scaling, so its A_lo is zero and that product is skipped.
//
// A work item is (tile of 128 vectors, chunk of 128 output coordinates); items
// go to persistent CTAs in contiguous row-tile-major runs, so a CTA walks the
// output chunks of one tile of x while that tile stays in L2.
//   warp 0       TMA producer of the constant pieces ([128 x 64] fp16, hi and lo)
//   warp 1       TMEM allocation and the single-thread MMA issuer
//   warps 2-5    A producers: x -> scaled fp16 hi/lo tiles (coalesced float4 /
//                bf16x8 loads); in stage 2 also -s n c[idx] from the codes
//   warps 6-13   epilogue: warp % 4 = TMEM lane quarter (32 vectors), the two
//                warpgroups take 64 of the 128 columns each
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;

constexpr int kTM = 128;                  // vectors per tile
constexpr int kTN = 128;                  // output coordinates per item
constexpr int kStages = 3;
constexpr int kPiece = kTM * 128;         // one [128 x 64] fp16 tile, 128B-swizzled
constexpr int kStage = 2 * kPiece;        // hi + lo
constexpr int kThreads = 448;
constexpr int kMisc = 4096;
constexpr int kSmem = 2 * kStages * kStage + kMisc + 1024;
constexpr float kLoScale = 2048.f, kLoInv = 4.8828125e-4f;
constexpr float kUScale = 4096.f;  // residual coordinates (~||u|| / sqrt(d)) scaled into fp16's range

struct GenArgs {
  const void* x;
  int64_t x_stride;
  int xbf16;
  int64_t N;
  int d, d_pad, bm, G, W;
  int64_t out_stride;
  const float* norms;        // written by gen_norms_kernel
  const uint32_t* codes_in;  // stage 2: the codes of stage 1
  uint32_t* codes;
  uint32_t* signs;
  float* rnorms;
  const float* thresholds;   // [2^bm - 1]
  const float* centroids;    // [2^bm]
  int prod;
  int64_t row_tiles, nc_count;
  uint16_t* u_out;           // stage 1 with a workspace: [2][N][d_pad] fp16 (hi, lo) of 2^12 u
  int* status;
};

__host__ __device__ __forceinline__ int64_t first_item(int64_t i, int64_t total, int64_t G) { return i * total / G; }

// power-of-two scale of a vector of norm n (1 for n = 0)
__device__ __forceinline__ float vec_scale(float n) {
  if (!(n > 0.f)) return 1.f;
  int e;
  (void)frexpf(n, &e);
  return ldexpf(1.f, 14 - e);
}

__device__ __forceinline__ uint32_t half2_bits(__half a, __half b) {
  return (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
}

// byte offset of element (row r, column c) of a [128 x 64] fp16 tile, 128B swizzle
__device__ __forceinline__ int sw_off(int r, int c) { return r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + (c & 7) * 2; }

template <int BM>
__device__ __forceinline__ uint32_t cell_of(float y, const float (&P)[8]) {
  // P[m] = m-th positive threshold in the scaled frame (m = 1 .. 2^(BM-1) - 1)
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

// cell i (0..31) of a group into its words (layout of include/tq.h)
template <int BM>
__device__ __forceinline__ void put_cell(uint32_t (&w)[BM], int i, uint32_t c) {
  if constexpr (BM == 1) {
    w[0] |= c << i;
  } else if constexpr (BM == 2) {
    w[i >> 4] |= c << (2 * (i & 15));
  } else if constexpr (BM == 4) {
    w[i >> 3] |= c << (4 * (i & 7));
  } else {
    if (i < 24) {
      w[i >> 3] |= c << (4 * (i & 7));
    } else {
      const int sh = 4 * (i - 24) + 3;
      w[0] |= (c & 1u) << sh;
      w[1] |= ((c >> 1) & 1u) << sh;
      w[2] |= ((c >> 2) & 1u) << sh;
    }
  }
}

template <int BM>
__device__ __forceinline__ uint32_t code_of(const uint32_t* w /*BM words of the group*/, int i) {
  if constexpr (BM == 1) return (w[0] >> i) & 1u;
  else if constexpr (BM == 2) return (w[i >> 4] >> (2 * (i & 15))) & 3u;
  else if constexpr (BM == 4) return (w[i >> 3] >> (4 * (i & 7))) & 15u;
  else {
    if (i < 24) return (w[i >> 3] >> (4 * (i & 7))) & 7u;
    const int sh = 4 * (i - 24) + 3;
    return ((w[0] >> sh) & 1u) | (((w[1] >> sh) & 1u) << 1) | (((w[2] >> sh) & 1u) << 2);
  }
}

__global__ void gen_norms_kernel(const void* x, int xbf16, int64_t x_stride, int64_t N, int d, float* norms,
                                 int64_t out_stride, const int32_t* channels, const int64_t* slots, int vec16) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t v = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; v < N; v += warps) {
    double acc = 0.0;
    if (vec16) {
      // 16-byte loads: rows start 16-byte aligned and d is a whole number of them
      const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(x) + v * x_stride * (xbf16 ? 2 : 4));
      const int nv = xbf16 ? d / 8 : d / 4;
      for (int j = lane; j < nv; j += 32) {
        const uint4 w = p[j];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        if (xbf16) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const double t0 = (double)__uint_as_float(ws[k] << 16), t1 = (double)__uint_as_float(ws[k] & 0xFFFF0000u);
            acc = fma(t0, t0, fma(t1, t1, acc));
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const double t = (double)__uint_as_float(ws[k]);
            acc = fma(t, t, acc);
          }
        }
      }
    } else if (xbf16) {
      const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(x) + v * x_stride;
      for (int j = lane; j < d; j += 32) {
        const double t = (double)__bfloat162float(p[channels ? channels[j] : j]);
        acc = fma(t, t, acc);
      }
    } else {
      const float* p = static_cast<const float*>(x) + v * x_stride;
      for (int j = lane; j < d; j += 32) {
        const double t = (double)p[channels ? channels[j] : j];
        acc = fma(t, t, acc);
      }
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) norms[slots ? slots[v] : v * out_stride] = (float)sqrt(acc);
  }
}

template <int STAGE, int BM>
__global__ void __launch_bounds__(kThreads, 1) quant_gen_kernel(const __grid_constant__ CUtensorMap bmap,
                                                                const __grid_constant__ CUtensorMap umap, GenArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem;                        // [kStages][hi, lo]
  uint8_t* b_s = smem + kStages * kStage;     // [kStages][hi, lo]
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_s + kStages * kStage);
  uint64_t* a_full = bars;                    // [kStages] count 128
  uint64_t* a_empty = a_full + kStages;       // [kStages]
  uint64_t* b_full = a_empty + kStages;       // [kStages] tx
  uint64_t* b_empty = b_full + kStages;       // [kStages]
  uint64_t* acc_full = b_empty + kStages;     // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2] count 8 (epilogue warps)
  uint64_t* rn_bar = acc_empty + 2;           // [2] count 256
  uint64_t* done_bar = rn_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  float* thr_s = reinterpret_cast<float*>(tmem_slot + 4);  // [16]
  float* cen_s = thr_s + 16;                               // [16]
  float* rn_s = cen_s + 16;                                // [2 parity][2 halves][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  // whole row tiles per CTA (the residual norm sums over all chunks of a tile)
  const int64_t it_lo = first_item(blockIdx.x, a.row_tiles, G) * a.nc_count;
  const int64_t it_hi = first_item(blockIdx.x + 1, a.row_tiles, G) * a.nc_count;
  const int KX = a.d_pad / 64;                        // k-chunks of the x part
  const int KC = (STAGE == 2) ? 2 * KX : KX;          // stage 2 adds the codebook part
  constexpr int K = 1 << BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&a_full[s], STAGE == 3 ? 1 : 128);
      mbar_init(&a_empty[s], 1);
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 8);
      mbar_init(&rn_bar[s], 256);
    }
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
    if (lane == 0) {
      int64_t ch = 0;
      for (int64_t it = it_lo; it < it_hi; ++it) {
        const int nc = (int)(it % a.nc_count);
        for (int kc = 0; kc < KC; ++kc, ++ch) {
          const int s = (int)(ch % kStages);
          if (!mbar_wait(&b_empty[s], (uint32_t)(((ch / kStages) & 1) ^ 1))) {
            atomicOr(a.status, kStatusTimeout);
            it = it_hi;
            break;
          }
          mbar_arrive_expect_tx(&b_full[s], kStage);
          uint8_t* dst = b_s + s * kStage;
          tma_load_2d(&bmap, &b_full[s], dst, kc * 64, nc * kTN);
          tma_load_2d(&bmap, &b_full[s], dst + kPiece, kc * 64, a.d_pad + nc * kTN);
          if (STAGE == 3) {
            // the residual rows of this tile (hi, lo), rows past N read as zero
            if (!mbar_wait(&a_empty[s], (uint32_t)(((ch / kStages) & 1) ^ 1))) {
              atomicOr(a.status, kStatusTimeout);
              it = it_hi;
              break;
            }
            const int rt = (int)(it / a.nc_count);
            mbar_arrive_expect_tx(&a_full[s], kStage);
            uint8_t* ad = a_s + s * kStage;
            tma_load_2d(&umap, &a_full[s], ad, kc * 64, rt * kTM);
            tma_load_2d(&umap, &a_full[s], ad + kPiece, kc * 64, (int)a.N + rt * kTM);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(kTM, kTN, false);
      const uint32_t aaddr = smem_u32(a_s), baddr = smem_u32(b_s);
      int64_t ch = 0;
      bool ok = true;
      int i = 0;
      for (int64_t it = it_lo; ok && it < it_hi; ++it, ++i) {
        const int ab = i & 1;
        if (!mbar_wait(&acc_empty[ab], (uint32_t)(((i >> 1) & 1) ^ 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc0 = tmem_base + (uint32_t)(ab * 256), acc1 = acc0 + kTN;
        for (int kc = 0; kc < KC; ++kc, ++ch) {
          const int s = (int)(ch % kStages);
          const uint32_t par = (uint32_t)((ch / kStages) & 1);
          if (!mbar_wait(&a_full[s], par) || !mbar_wait(&b_full[s], par)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool has_lo = STAGE == 3 || (kc >= KX) || !a.xbf16;
          const uint32_t ah = aaddr + s * kStage, al = ah + kPiece;
          const uint32_t bh = baddr + s * kStage, bl = bh + kPiece;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint32_t acc = (kc | k4) != 0 ? 1u : 0u;
            mma_f16(acc0, sw128_kmajor_desc(ah + k4 * 32), sw128_kmajor_desc(bh + k4 * 32), idesc, acc);
            mma_f16(acc1, sw128_kmajor_desc(ah + k4 * 32), sw128_kmajor_desc(bl + k4 * 32), idesc, acc);
            if (has_lo)
              mma_f16(acc1, sw128_kmajor_desc(al + k4 * 32), sw128_kmajor_desc(bh + k4 * 32), idesc, 1u);
          }
          mma_commit(&a_empty[s]);
          mma_commit(&b_empty[s]);
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done_bar);
    }
  } else if (warp < 6) {
    // A producers (stage 3 takes its A tiles by TMA)
    if (STAGE != 3) {
    const int p = threadIdx.x - 64;      // 0..127
    const int wl = p >> 5;               // producer warp 0..3
    int64_t ch = 0;
    bool ok = true;
    for (int64_t it = it_lo; ok && it < it_hi; ++it) {
      const int64_t rt = it / a.nc_count;
      const int64_t row0 = rt * kTM;
      // scales of this thread's rows in the x part (fixed across k-chunks)
      float sc[16];
      if (a.xbf16) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t v = row0 + 4 * (wl * 8 + i) + (lane >> 3);
          sc[i] = v < a.N ? vec_scale(a.norms[v * a.out_stride]) : 0.f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int64_t v = row0 + 2 * (wl * 16 + i) + (lane >> 4);
          sc[i] = v < a.N ? vec_scale(a.norms[v * a.out_stride]) : 0.f;
        }
      }
      for (int kc = 0; kc < KC; ++kc, ++ch) {
        const int s = (int)(ch % kStages);
        if (!mbar_wait_warp(&a_empty[s], (uint32_t)(((ch / kStages) & 1) ^ 1))) {
          ok = false;
          break;
        }
        uint8_t* th = a_s + s * kStage;
        uint8_t* tl = th + kPiece;
        if (kc < KX) {
          if (a.xbf16) {
            const int c8 = (lane & 7) * 8;
            const int col = kc * 64 + c8;
            uint4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int64_t r = row0 + 4 * (wl * 8 + i) + (lane >> 3);
              v[i] = (r < a.N && col < a.d)
                         ? *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.x) + r * a.x_stride + col)
                         : make_uint4(0u, 0u, 0u, 0u);
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
            const int col = kc * 64 + c4;
#pragma unroll
            for (int bt = 0; bt < 2; ++bt) {  // two batches of 8 rows in flight
              float4 v[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int64_t r = row0 + 2 * (wl * 16 + 8 * bt + i) + (lane >> 4);
                v[i] = (r < a.N && col < a.d)
                           ? *reinterpret_cast<const float4*>(static_cast<const float*>(a.x) + r * a.x_stride + col)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
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
                  lo[q] = __float2half_rn((f[q] - __half2float(hi[q])) * kLoScale);
                }
                *reinterpret_cast<uint2*>(th + sw_off(rr, c4)) =
                    make_uint2(half2_bits(hi[0], hi[1]), half2_bits(hi[2], hi[3]));
                *reinterpret_cast<uint2*>(tl + sw_off(rr, c4)) =
                    make_uint2(half2_bits(lo[0], lo[1]), half2_bits(lo[2], lo[3]));
              }
            }
          }
        } else {
          // stage 2, codebook part: row p, coordinates 64 (kc - KX) .. + 63 as -s n c[idx]
          const int64_t v = row0 + p;
          const int g0 = 2 * (kc - KX);
          float f = 0.f;
          uint32_t w[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
          bool gv[2] = {false, false};
          if (v < a.N) {
            const float n = a.norms[v * a.out_stride];
            f = -n * vec_scale(n);
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
              gv[gg] = g0 + gg < a.G;
              if (gv[gg]) {
                const uint32_t* src = a.codes_in + v * a.out_stride * a.W + (g0 + gg) * BM;
#pragma unroll
                for (int k = 0; k < BM; ++k) w[gg][k] = src[k];
              }
            }
          }
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {  // 16-byte units of 8 coordinates
              uint32_t oh[4], ol[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __half hv[2], lv[2];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                  const int i = 8 * u + 2 * e + t;
                  const float c = gv[gg] ? f * cen_s[code_of<BM>(w[gg], i)] : 0.f;
                  hv[t] = __float2half_rn(c);
                  lv[t] = __float2half_rn((c - __half2float(hv[t])) * kLoScale);
                }
                oh[e] = half2_bits(hv[0], hv[1]);
                ol[e] = half2_bits(lv[0], lv[1]);
              }
              const int off = sw_off(p, 32 * gg + 8 * u);
              *reinterpret_cast<uint4*>(th + off) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
              *reinterpret_cast<uint4*>(tl + off) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
            }
          }
        }
        fence_async_smem();
        mbar_arrive(&a_full[s]);
      }
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
    }
  } else {
    // epilogue
    const int quarter = warp & 3;
    const int half = (warp - 6) >> 2;
    const int row = quarter * 32 + lane;
    float P[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) P[m] = 0.f;
    float n = 0.f, inv_ns = 0.f, u2 = 0.f;
    int64_t cur_rt = -1;
    int nrt = 0;  // row tiles finished (parity of rn_bar)
    int i = 0;
    for (int64_t it = it_lo; it < it_hi; ++it, ++i) {
      const int64_t rt = it / a.nc_count;
      const int nc = (int)(it % a.nc_count);
      const int64_t vec = rt * kTM + row;
      if (rt != cur_rt) {
        cur_rt = rt;
        n = vec < a.N ? a.norms[vec * a.out_stride] : 0.f;
        const float ns = n * vec_scale(n);
        inv_ns = n > 0.f ? 1.f / ns : 0.f;
#pragma unroll
        for (int m = 1; m < 8; ++m)
          if (m < (1 << (BM - 1))) P[m] = n > 0.f ? ns * thr_s[(1 << (BM - 1)) - 1 + m] : INFINITY;
        u2 = 0.f;
      }
      const int ab = i & 1;
      if (!mbar_wait_warp(&acc_full[ab], (uint32_t)((i >> 1) & 1))) {
        atomicOr(a.status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * 256 + half * 64);
      const int j0 = nc * kTN + half * 64;  // first coordinate of this thread's 64
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = (j0 >> 5) + gg;  // warp-uniform
        if (g >= a.G) break;
        const int jg = 32 * g;
        float v[32];
        {
          float a1[32];
          tmem_ld32(t0 + gg * 32, v);
          tmem_ld32(t0 + kTN + gg * 32, a1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = fmaf(a1[e], kLoInv, v[e]);
        }
        if (STAGE == 1) {
          uint32_t w[BM];
#pragma unroll
          for (int k = 0; k < BM; ++k) w[k] = 0u;
          uint32_t uh[16], ul[16];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const uint32_t idx = cell_of<BM>(v[e], P);
            const bool in = jg + e < a.d;
            put_cell<BM>(w, e, in ? idx : 0u);
            float u = 0.f;
            if (a.prod && in) {
              u = fmaf(v[e], inv_ns, -cen_s[idx]);
              u2 = fmaf(u, u, u2);
            }
            if (a.u_out) {
              const float us = u * kUScale;
              const __half hi = __float2half_rn(us);
              const __half lo = __float2half_rn((us - __half2float(hi)) * kLoScale);
              const uint32_t sh = 16 * (e & 1);
              if ((e & 1) == 0) uh[e >> 1] = 0u, ul[e >> 1] = 0u;
              uh[e >> 1] |= (uint32_t)__half_as_ushort(hi) << sh;
              ul[e >> 1] |= (uint32_t)__half_as_ushort(lo) << sh;
            }
          }
          if (a.u_out && vec < a.N) {
            uint4* dh = reinterpret_cast<uint4*>(a.u_out + vec * a.d_pad + jg);
            uint4* dl = reinterpret_cast<uint4*>(a.u_out + (a.N + vec) * a.d_pad + jg);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              dh[q] = make_uint4(uh[4 * q], uh[4 * q + 1], uh[4 * q + 2], uh[4 * q + 3]);
              dl[q] = make_uint4(ul[4 * q], ul[4 * q + 1], ul[4 * q + 2], ul[4 * q + 3]);
            }
          }
          if (vec < a.N) {
            uint32_t* dst = a.codes + vec * a.out_stride * a.W + g * BM;
#pragma unroll
            for (int k = 0; k < BM; ++k) dst[k] = w[k];
          }
        } else {
          uint32_t w = 0u;
#pragma unroll
          for (int e = 0; e < 32; ++e) w |= ((v[e] >= 0.f && jg + e < a.d) ? 1u : 0u) << e;
          if (vec < a.N) a.signs[vec * a.out_stride * a.G + g] = w;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      if (STAGE == 1 && a.prod && nc == a.nc_count - 1) {
        // the tile's last chunk: combine the two column halves of ||y - c[idx]||^2
        float* rs = rn_s + (nrt & 1) * 256;
        rs[half * 128 + row] = u2;
        mbar_arrive(&rn_bar[nrt & 1]);
        if (!mbar_wait_warp(&rn_bar[nrt & 1], (uint32_t)((nrt >> 1) & 1))) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        if (half == 0 && vec < a.N) a.rnorms[vec * a.out_stride] = n > 0.f ? n * sqrtf(rs[row] + rs[128 + row]) : 0.f;
        ++nrt;
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    if (!mbar_wait(done_bar, 0) && lane == 0) atomicOr(a.status, kStatusTimeout);
    __syncwarp();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int STAGE>
int launch_stage(const tq_ctx* h, const GenArgs& a, const CUtensorMap& map, const CUtensorMap& umap, int grid,
                 cudaStream_t s) {
  auto pick = [&](auto kern) -> int {
    if (int e = ensure_dyn_smem((const void*)kern, kSmem)) return e;
    kern<<<grid, kThreads, kSmem, s>>>(map, umap, a);
    return (int)cudaGetLastError();
  };
  switch (h->bm) {
    case 1: return pick(quant_gen_kernel<STAGE, 1>);
    case 2: return pick(quant_gen_kernel<STAGE, 2>);
    case 3: return pick(quant_gen_kernel<STAGE, 3>);
    default: return pick(quant_gen_kernel<STAGE, 4>);
  }
}

bool make_f16_map(CUtensorMap* m, const void* base, int64_t kext, int64_t rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t gdim[2] = {(cuuint64_t)kext, (cuuint64_t)rows};
  const cuuint64_t gstride[1] = {(cuuint64_t)kext * 2};
  const cuuint32_t box[2] = {64, kTN};
  const cuuint32_t estride[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool quant_gen_supported(const tq_ctx* h) { return h->dev.gen_pi != nullptr; }

int launch_gen_norms(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride, float* norms,
                     int64_t out_stride, void* stream, const int32_t* channels, const int64_t* slots) {
  const int64_t blocks = (N + 7) / 8;  // 8 warps per block, one vector per warp
  const int grid = (int)(blocks < (int64_t)h->sm_count * 16 ? blocks : (int64_t)h->sm_count * 16);
  const int esz = dtype == TQ_BF16 ? 2 : 4;
  const int vec16 = !channels && (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (x_stride * esz) % 16 == 0 &&
                    (h->d * esz) % 16 == 0;
  gen_norms_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(x, dtype == TQ_BF16 ? 1 : 0, x_stride, N, h->d, norms,
                                                          out_stride, channels, slots, vec16);
  return (int)cudaGetLastError();
}

// the residual path (stage 3) is used for prod when d_pad > 256
bool quant_gen_needs_workspace(const tq_ctx* h) { return h->variant == TQ_PROD && h->gen_d_pad > 256; }

size_t quant_gen_workspace_rows_bytes(const tq_ctx* h) { return (size_t)4 * h->gen_d_pad; }

int launch_quant_gen(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride, uint32_t* codes,
                     uint32_t* signs, float* norms, float* rnorms, int64_t out_stride, void* workspace,
                     size_t ws_bytes, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  const bool prod = h->variant == TQ_PROD;
  const int xbf16 = dtype == TQ_BF16 ? 1 : 0;
  const int esz = xbf16 ? 2 : 4;
  if (int e = launch_gen_norms(h, x, dtype, N, x_stride, norms, out_stride, stream)) return e;
  const int dp = h->gen_d_pad;
  const bool resid = prod && quant_gen_needs_workspace(h);
  // rows per launch: all of them, or as many whole 128-row tiles as the workspace holds
  int64_t chunk = N;
  if (resid) {
    const int64_t fit = (int64_t)(ws_bytes / quant_gen_workspace_rows_bytes(h)) / kTM * kTM;
    if (fit < kTM) return (int)cudaErrorInvalidValue;
    chunk = fit < N ? fit : N;
  }
  CUtensorMap m1, m2, mu;
  if (!make_f16_map(&m1, h->dev.gen_pi, dp, 2 * dp)) return (int)cudaErrorInvalidValue;
  if (prod && !make_f16_map(&m2, h->dev.gen_st, resid ? dp : 2 * dp, 2 * dp)) return (int)cudaErrorInvalidValue;
  for (int64_t r0 = 0; r0 < N; r0 += chunk) {
    const int64_t n = (N - r0) < chunk ? (N - r0) : chunk;
    GenArgs a;
    a.x = static_cast<const char*>(x) + r0 * x_stride * esz;
    a.x_stride = x_stride;
    a.xbf16 = xbf16;
    a.N = n;
    a.d = h->d;
    a.d_pad = dp;
    a.bm = h->bm;
    a.G = (h->d + 31) / 32;
    a.W = a.G * h->bm;
    a.out_stride = out_stride;
    a.norms = norms + r0 * out_stride;
    a.codes_in = codes + r0 * out_stride * a.W;
    a.codes = codes + r0 * out_stride * a.W;
    a.signs = prod ? signs + r0 * out_stride * a.G : nullptr;
    a.rnorms = prod ? rnorms + r0 * out_stride : nullptr;
    a.thresholds = h->dev.thresholds;
    a.centroids = h->dev.centroids;
    a.prod = prod ? 1 : 0;
    a.nc_count = dp / kTN;
    a.row_tiles = (n + kTM - 1) / kTM;
    a.u_out = resid ? static_cast<uint16_t*>(workspace) : nullptr;
    a.status = h->dev.status;
    const int grid = (int)(a.row_tiles < h->sm_count ? a.row_tiles : h->sm_count);
    int e = launch_stage<1>(h, a, m1, m1, grid, s);
    if (e || !prod) {
      if (e) return e;
      continue;
    }
    if (resid) {
      // the T half of [S | T]: columns dp .. 2 dp of gen_st, as its own [2 dp][dp] view
      if (!make_f16_map(&mu, workspace, dp, 2 * n)) return (int)cudaErrorInvalidValue;
      CUtensorMap mt;
      {
        EncodeTiledFn enc = encode_tiled_fn();
        const cuuint64_t gdim[2] = {(cuuint64_t)dp, (cuuint64_t)(2 * dp)};
        const cuuint64_t gstride[1] = {(cuuint64_t)(2 * dp) * 2};
        const cuuint32_t box[2] = {64, kTN};
        const cuuint32_t estride[2] = {1, 1};
        if (enc(&mt, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h->dev.gen_st + dp, gdim, gstride, box, estride,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
          return (int)cudaErrorInvalidValue;
      }
      e = launch_stage<3>(h, a, mt, mu, grid, s);
    } else {
      e = launch_stage<2>(h, a, m2, m1, grid, s);
    }
    if (e) return e;
  }
  return 0;
}

}  // namespace tqi
