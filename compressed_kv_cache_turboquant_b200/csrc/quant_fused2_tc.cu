// TurboQuant quantization of 128-vector tiles for dimensions up to 256, both
// contractions in one persistent kernel, with the input staged by TMA and the
// residual kept in tensor memory (sm_100a).
//
// [ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: store the norm,
// rotate, quantize every coordinate against the Lloyd-Max codebook; for
// TurboQuant_prod keep the 1-bit signs of the projected residual and its norm.
// Both steps are plain matrix products
// (ttakun.com/news/45354, "为什么随机旋转是整个算法的底层杠杆").
//
// Per tile (M = 128 vectors), with s = 2^(14 - e) for n = ||x|| = f 2^e (from
// gen_norms_kernel) and the constant pieces scaled by 2^10:
//   Y = (s X) (2^10 Pi)^T                   TMEM columns [0, 256)
//   epilogue: codes of y against s n 2^10 t_k; u = y / (s n 2^10) - c[idx];
//     ||r|| = n ||u||; 2^12 u as fp16 hi / remainder, written back with
//     tcgen05.st into the Y columns it was read from (group g's 32 coordinates
//     -> 16 columns of hi pairs, 16 of lo pairs)
//   V = (2^12 U) (2^10 T)^T, T = S Pi^T, A read from tensor memory
//                                           TMEM columns [256, 512)
//   epilogue: QJL bits = sign bits of V
// Every operand moves in 32-wide K chunks (64-byte rows, 64-byte swizzle):
//   x staging ring   raw x (fp32 or bf16) by TMA, out-of-range rows and columns
//                    read as zero
//   operand ring     s x as fp16 hi / remainder (one converter thread per row)
//   constant ring    fp16 hi / remainder of 2^10 Pi, then of 2^10 T, by TMA
// so the next tile's input streams in while this tile's two products and its
// epilogue run; the projection of tile i overlaps the epilogue of tile i group
// by group, and the rotation of tile i + 1 waits only for that projection.
// Split precision with one accumulator: v = v_hi + v_lo (v_lo the fp16 of the
// remainder, not rescaled), hi.hi + hi.lo + lo.hi into one fp32 accumulator;
// bf16 input has no lo piece.
//
// Warp roles (480 threads, one CTA per SM):
//   warp 0       TMA producer of the constant ring
//   warp 1       TMEM allocation and the single-thread MMA issuer
//   warp 2       TMA producer of the x staging ring
//   warps 3-6    converters: thread = row of the tile
//   warps 7-14   epilogue: warp % 4 = TMEM lane quarter, warps 7-10 even
//                32-coordinate groups, 11-14 odd ones
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "tq.h"

#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;

constexpr int kTM = 128;
constexpr int kThreads = 480;
constexpr int kAPiece = kTM * 64;          // [128 x 32] fp16
constexpr int kAStage = 2 * kAPiece;       // hi + lo
constexpr int kYCol = 0, kVCol = 256;
constexpr float kUScale = 4096.f;
constexpr int kMisc = 4096;

// PolarQuant decisions (variant TQ_POLAR): level-1 sectors by quadrant and
// tangent comparisons, levels >= 2 by squared radii against tan^2 of the
// thresholds (theta >= t <=> r_b^2 >= tan^2(t) r_a^2 for radii r >= 0)
struct PolarDec {
  float t1[3];      // b1 = 4: tan(pi/8), 1, tan(3 pi/8)
  float T[8][3];    // [level][k]: tan^2 of level-l threshold k (l = 2..L)
  int b1, bh, L;
  int base[9];      // first entry of level l among the packed codes of levels >= 2
  int w1;           // words of the level-1 codes
};

struct F2Args {
  int64_t N;
  int d, n16, kc, G, W;     // kc = 32-wide K chunks = G
  int64_t out_stride;
  int prod, xbf16;
  const float* norms;
  uint32_t* codes;
  uint32_t* signs;
  float* rnorms;
  const int64_t* slots;
  int rn_f16;
  const float* thresholds;
  const float* centroids;
  float acc_scale;
  int xs, as, bs;           // stage counts of the three rings
  int x_stage_bytes, b_stage_bytes;
  int64_t row_tiles;
  PolarDec pol;
  int* status;
};

__host__ __device__ __forceinline__ int64_t tile_lo(int64_t i, int64_t total, int64_t G) { return i * total / G; }

__device__ __forceinline__ int64_t out_row2(const F2Args& a, int64_t v) {
  return a.slots ? a.slots[v] : v * a.out_stride;
}

__device__ __forceinline__ float vscale(float n) {
  if (!(n > 0.f)) return 1.f;
  int e;
  (void)frexpf(n, &e);
  return ldexpf(1.f, 14 - e);
}

__device__ __forceinline__ uint32_t h2bits(__half a, __half b) {
  return (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
}

__device__ __forceinline__ void arrive_cnt(uint64_t* bar, uint32_t cnt) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(cnt) : "memory");
}

// byte offset of 16-byte unit j of row r in a tile of 64-byte rows, 64B swizzle
__device__ __forceinline__ int sw64(int r, int j) { return r * 64 + ((j ^ ((r >> 1) & 3)) << 4); }

// shared-memory descriptor of a K-major operand in 64-byte rows, 64B swizzle
// (8-row atoms 512 bytes apart)
__device__ __forceinline__ uint64_t sw64_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(512u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)4u << 61;
  return d;
}

// 16-wide K steps of 32-wide chunk k below d
__device__ __forceinline__ int steps16(int d, int k) {
  const int rem = d - 32 * k;
  return rem >= 32 ? 2 : (rem > 16 ? 2 : 1);
}

template <int BM>
__device__ __forceinline__ uint32_t cell2(float y, const float (&P)[8]) {
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

template <int BM>
__device__ __forceinline__ void pack32(const uint32_t (&c)[32], uint32_t (&w)[BM]) {
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

// level-1 cell of the angle of (a, b) on the uniform grid of 2^b1 cells over [0, 2 pi)
__device__ __forceinline__ uint32_t polar_sector(float a, float b, const PolarDec& P) {
  if (a == 0.f && b == 0.f) return 0u;
  uint32_t q;
  float ap, bp;  // (a, b) rotated by -q quarter turns into [0, pi/2)
  if (a > 0.f && b >= 0.f) q = 0u, ap = a, bp = b;
  else if (a <= 0.f && b > 0.f) q = 1u, ap = b, bp = -a;
  else if (a < 0.f && b <= 0.f) q = 2u, ap = -a, bp = -b;
  else q = 3u, ap = -b, bp = a;
  if (P.b1 == 2) return q;
  const uint32_t sub = (bp >= P.t1[0] * ap ? 1u : 0u) + (bp >= P.t1[1] * ap ? 1u : 0u) + (bp >= P.t1[2] * ap ? 1u : 0u);
  return 4u * q + sub;
}

// level-l (l >= 2) cell of atan2(r_b, r_a) from the squared radii
__device__ __forceinline__ uint32_t polar_cell(float sa, float sb, const float (&T)[3], int bh) {
  if (sa == 0.f && sb == 0.f) return 0u;
  uint32_t c = sb >= T[0] * sa ? 1u : 0u;
  if (bh == 2) c += (sb >= T[1] * sa ? 1u : 0u) + (sb >= T[2] * sa ? 1u : 0u);
  return c;
}

__device__ __forceinline__ void put_bits(uint32_t* w, int e, uint32_t code, int bits) {
  w[(e * bits) >> 5] |= code << ((e * bits) & 31);
}

// PolarQuant codes of one row whose rotated coordinates are the TMEM columns
// [0, D) of this thread's lane
template <int D>
__device__ __forceinline__ void polar_row(uint32_t taddr, const PolarDec& P, uint32_t* dst, bool live) {
  constexpr int G = D / 32;
  uint32_t w1[8], wh[4];
#pragma unroll
  for (int q = 0; q < 8; ++q) w1[q] = 0u;
#pragma unroll
  for (int q = 0; q < 4; ++q) wh[q] = 0u;
  float sg[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float v[32];
    tmem_ld32(taddr + (uint32_t)(32 * g), v);
    tmem_wait_ld();
    float s[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      put_bits(w1, 16 * g + p, polar_sector(v[2 * p], v[2 * p + 1], P), P.b1);
      s[p] = fmaf(v[2 * p], v[2 * p], v[2 * p + 1] * v[2 * p + 1]);
    }
    // levels 2..5 inside the group: 8, 4, 2, 1 entries
#pragma unroll
    for (int lev = 2, cnt = 8; cnt >= 1; ++lev, cnt >>= 1) {
#pragma unroll
      for (int p = 0; p < cnt; ++p) {
        put_bits(wh, P.base[lev] + cnt * g + p, polar_cell(s[2 * p], s[2 * p + 1], P.T[lev], P.bh), P.bh);
        s[p] = s[2 * p] + s[2 * p + 1];
      }
    }
    sg[g] = s[0];
  }
  // levels above the groups: pairs of group radii
#pragma unroll
  for (int lev = 6, cnt = G / 2; cnt >= 1; ++lev, cnt >>= 1) {
#pragma unroll
    for (int p = 0; p < cnt; ++p) {
      put_bits(wh, P.base[lev] + p, polar_cell(sg[2 * p], sg[2 * p + 1], P.T[lev], P.bh), P.bh);
      sg[p] = sg[2 * p] + sg[2 * p + 1];
    }
  }
  if (live) {
    for (int q = 0; q < P.w1; ++q) dst[q] = w1[q];
    const int wn = ((D / 2 - 1 + 31) / 32) * P.bh;
    for (int q = 0; q < wn; ++q) dst[P.w1 + q] = wh[q];
  }
}

template <int BM, int POLAR_D>
__global__ void __launch_bounds__(kThreads, 1) quant_fused2_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                   const __grid_constant__ CUtensorMap pimap,
                                                                   const __grid_constant__ CUtensorMap tmap,
                                                                   F2Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* x_s = smem;                                   // [xs][x_stage_bytes]
  uint8_t* a_s = x_s + a.xs * a.x_stage_bytes;           // [as][hi, lo]
  uint8_t* b_s = a_s + a.as * kAStage;                   // [bs][hi, lo]
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_s + a.bs * a.b_stage_bytes);
  uint64_t* x_full = bars;             // [4] TMA bytes
  uint64_t* x_empty = x_full + 4;      // [4] 4 converter warps
  uint64_t* a_full = x_empty + 4;      // [4] 4 converter warps
  uint64_t* a_empty = a_full + 4;      // [4] MMA commit
  uint64_t* b_full = a_empty + 4;      // [3] TMA bytes
  uint64_t* b_empty = b_full + 3;      // [3] MMA commit
  uint64_t* y_full = b_empty + 3;      // MMA commit
  uint64_t* y_empty = y_full + 1;      // 8 epilogue warps (mse)
  uint64_t* v_full = y_empty + 1;      // MMA commit
  uint64_t* v_empty = v_full + 1;      // 8 epilogue warps
  uint64_t* u_ready = v_empty + 1;     // [8] 4 epilogue warps per group
  uint64_t* rn_bar = u_ready + 8;      // [2] 256
  uint64_t* done_bar = rn_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  float* thr_s = reinterpret_cast<float*>(tmem_slot + 4);  // [16]
  float* cen_s = thr_s + 16;                               // [16]
  float* rn_s = cen_s + 16;                                // [2][2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t Gc = gridDim.x;
  const int64_t t_lo = tile_lo(blockIdx.x, a.row_tiles, Gc);
  const int64_t t_hi = tile_lo(blockIdx.x + 1, a.row_tiles, Gc);
  const int kc = a.kc;
  constexpr int K = 1 << BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 4);
      mbar_init(&a_full[s], 4);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(y_full, 1);
    mbar_init(y_empty, 8);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 8);
    for (int g = 0; g < 8; ++g) mbar_init(&u_ready[g], 4);
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
    // ---------------- constant ring: Pi chunks, then (prod) T chunks, per tile
    if (lane == 0) {
      const int per = a.prod ? 2 * kc : kc;
      int64_t seq = 0, issued = 0;
      bool ok = true;
      const uint32_t bytes = (uint32_t)a.b_stage_bytes;
      for (int64_t t = t_lo; ok && t < t_hi; ++t) {
        for (int e = 0; e < per; ++e, ++seq) {
          const int s = (int)(seq % a.bs);
          if (!mbar_wait(&b_empty[s], (uint32_t)(((seq / a.bs) & 1) ^ 1))) {
            ok = false;
            break;
          }
          const CUtensorMap* map = e < kc ? &pimap : &tmap;
          const int k = e < kc ? e : e - kc;
          uint8_t* dst = b_s + s * a.b_stage_bytes;
          mbar_arrive_expect_tx(&b_full[s], bytes);
          tma_load_2d(map, &b_full[s], dst, 32 * k, 0);
          tma_load_2d(map, &b_full[s], dst + bytes / 2, 32 * k, a.n16);
          issued = seq + 1;
        }
      }
      for (int64_t q = issued - a.bs > 0 ? issued - a.bs : 0; q < issued; ++q)
        if (!mbar_wait(&b_full[q % a.bs], (uint32_t)((q / a.bs) & 1))) ok = false;
      if (!ok) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 2) {
    // ---------------- x staging ring: [128 rows x 32] boxes of the input
    if (lane == 0) {
      int64_t seq = 0, issued = 0;
      bool ok = true;
      const uint32_t bytes = (uint32_t)a.x_stage_bytes;
      for (int64_t t = t_lo; ok && t < t_hi; ++t) {
        for (int k = 0; k < kc; ++k, ++seq) {
          const int s = (int)(seq % a.xs);
          if (!mbar_wait(&x_empty[s], (uint32_t)(((seq / a.xs) & 1) ^ 1))) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&x_full[s], bytes);
          tma_load_2d(&xmap, &x_full[s], x_s + s * a.x_stage_bytes, 32 * k, (int)(t * kTM));
          issued = seq + 1;
        }
      }
      for (int64_t q = issued - a.xs > 0 ? issued - a.xs : 0; q < issued; ++q)
        if (!mbar_wait(&x_full[q % a.xs], (uint32_t)((q / a.xs) & 1))) ok = false;
      if (!ok) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kTM, a.n16, false);
      const uint32_t aaddr = smem_u32(a_s), baddr = smem_u32(b_s);
      const uint32_t ycol = tmem_base + kYCol, vcol = tmem_base + kVCol;
      const bool x_lo = !a.xbf16;
      int64_t seq_a = 0, seq_b = 0;
      bool ok = true;
      int i = 0;
      for (int64_t t = t_lo; ok && t < t_hi; ++t, ++i) {
        // the Y columns are free again once the previous tile's projection has
        // read its residual from them (prod) or its epilogue has read Y (mse)
        if (i > 0 && !mbar_wait(a.prod ? v_full : y_empty, (uint32_t)((i - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int k = 0; k < kc; ++k, ++seq_a, ++seq_b) {
          const int sa = (int)(seq_a % a.as), sb = (int)(seq_b % a.bs);
          if (!mbar_wait(&a_full[sa], (uint32_t)((seq_a / a.as) & 1)) ||
              !mbar_wait(&b_full[sb], (uint32_t)((seq_b / a.bs) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ah = aaddr + sa * kAStage, al = ah + kAPiece;
          const uint32_t bh = baddr + sb * a.b_stage_bytes, bl = bh + a.b_stage_bytes / 2;
          const int ns = steps16(a.d, k);
          for (int kk = 0; kk < ns; ++kk) {
            const uint64_t dah = sw64_desc(ah + kk * 32), dbh = sw64_desc(bh + kk * 32);
            mma_f16(ycol, dah, dbh, idesc, (k | kk) != 0 ? 1u : 0u);
            mma_f16(ycol, dah, sw64_desc(bl + kk * 32), idesc, 1u);
            if (x_lo) mma_f16(ycol, sw64_desc(al + kk * 32), dbh, idesc, 1u);
          }
          mma_commit(&a_empty[sa]);
          mma_commit(&b_empty[sb]);
        }
        if (!ok) break;
        mma_commit(y_full);
        if (!a.prod) continue;
        if (!mbar_wait(v_empty, (uint32_t)((i & 1) ^ 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int g = 0; g < kc; ++g, ++seq_b) {
          const int sb = (int)(seq_b % a.bs);
          if (!mbar_wait(&u_ready[g], (uint32_t)(i & 1)) || !mbar_wait(&b_full[sb], (uint32_t)((seq_b / a.bs) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bh = baddr + sb * a.b_stage_bytes, bl = bh + a.b_stage_bytes / 2;
          const int ns = steps16(a.d, g);
          for (int kk = 0; kk < ns; ++kk) {
            const uint32_t uh = ycol + 32 * g + 8 * kk, ul = uh + 16;
            const uint64_t dbh = sw64_desc(bh + kk * 32);
            mma_f16_ta(vcol, uh, dbh, idesc, (g | kk) != 0 ? 1u : 0u);
            mma_f16_ta(vcol, uh, sw64_desc(bl + kk * 32), idesc, 1u);
            mma_f16_ta(vcol, ul, dbh, idesc, 1u);
          }
          mma_commit(&b_empty[sb]);
        }
        if (!ok) break;
        mma_commit(v_full);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done_bar);
    }
  } else if (warp < 7) {
    // ---------------- converters: thread r = row r of the tile
    const int r = threadIdx.x - 96;
    int64_t seq = 0;
    bool ok = true;
    for (int64_t t = t_lo; ok && t < t_hi; ++t) {
      const int64_t v = t * kTM + r;
      const float sc = v < a.N ? vscale(a.norms[out_row2(a, v)]) : 0.f;
      for (int k = 0; k < kc; ++k, ++seq) {
        const int sx = (int)(seq % a.xs), sa = (int)(seq % a.as);
        if (!mbar_wait_warp(&x_full[sx], (uint32_t)((seq / a.xs) & 1)) ||
            !mbar_wait_warp(&a_empty[sa], (uint32_t)(((seq / a.as) & 1) ^ 1))) {
          ok = false;
          break;
        }
        const uint8_t* xs = x_s + sx * a.x_stage_bytes;
        uint8_t* th = a_s + sa * kAStage;
        uint8_t* tl = th + kAPiece;
        if (a.xbf16) {
          // row of 64 bytes, 64B swizzle: 4 units of 8 values, exact in fp16 after the scaling
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 w = *reinterpret_cast<const uint4*>(xs + sw64(r, j));
            const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              o[q] = h2bits(__float2half_rn(__uint_as_float(w4[q] << 16) * sc),
                            __float2half_rn(__uint_as_float(w4[q] & 0xFFFF0000u) * sc));
            *reinterpret_cast<uint4*>(th + sw64(r, j)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else {
          // row of 128 bytes, 128B swizzle: unit j at (j ^ (r & 7)); two input units per output unit
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float4 f0 = *reinterpret_cast<const float4*>(xs + r * 128 + (((2 * j) ^ (r & 7)) << 4));
            const float4 f1 = *reinterpret_cast<const float4*>(xs + r * 128 + (((2 * j + 1) ^ (r & 7)) << 4));
            const float f[8] = {f0.x * sc, f0.y * sc, f0.z * sc, f0.w * sc, f1.x * sc, f1.y * sc, f1.z * sc, f1.w * sc};
            uint32_t oh[4], ol[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const __half h0 = __float2half_rn(f[2 * q]), h1 = __float2half_rn(f[2 * q + 1]);
              oh[q] = h2bits(h0, h1);
              ol[q] = h2bits(__float2half_rn(f[2 * q] - __half2float(h0)), __float2half_rn(f[2 * q + 1] - __half2float(h1)));
            }
            *reinterpret_cast<uint4*>(th + sw64(r, j)) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
            *reinterpret_cast<uint4*>(tl + sw64(r, j)) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&x_empty[sx]);
          mbar_arrive(&a_full[sa]);
        }
      }
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  } else {
    // ---------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 7) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float P[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) P[m] = 0.f;
    int i = 0;
    bool ok = true;
    for (int64_t t = t_lo; ok && t < t_hi; ++t, ++i) {
      const int64_t vec = t * kTM + row;
      const bool live = vec < a.N;
      const int64_t orow = live ? out_row2(a, vec) : 0;
      const float n = live ? a.norms[orow] : 0.f;
      const float ns = n * vscale(n) * a.acc_scale;
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
      if constexpr (POLAR_D > 0) {
        // one thread per row walks the whole angle tree; the other half idles
        if (half == 0) polar_row<POLAR_D>(tmem_base + lane_base + kYCol, a.pol, a.codes + orow * a.W, live);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(y_empty);
        continue;
      }
      for (int g = half; g < a.G; g += 2) {
        const int jg = 32 * g;
        float v[32];
        tmem_ld32(tmem_base + lane_base + (uint32_t)(kYCol + jg), v);
        tmem_wait_ld();
        uint32_t c[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) c[e] = (jg + e < a.d) ? cell2<BM>(v[e], P) : 0u;
        if (live) {
          uint32_t w[BM];
          pack32<BM>(c, w);
          uint32_t* dst = a.codes + orow * a.W + g * BM;
#pragma unroll
          for (int q = 0; q < BM; ++q) dst[q] = w[q];
        }
        if (a.prod) {
          uint32_t uh[16], ul[16];
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
            uh[e >> 1] = h2bits(h0, h1);
            ul[e >> 1] = h2bits(__float2half_rn(us[0] - __half2float(h0)), __float2half_rn(us[1] - __half2float(h1)));
          }
          tmem_st16(tmem_base + lane_base + (uint32_t)(kYCol + jg), uh);
          tmem_st16(tmem_base + lane_base + (uint32_t)(kYCol + jg + 16), ul);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&u_ready[g]);
        }
      }
      if (!a.prod) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(y_empty);
        continue;
      }
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
      if (!mbar_wait_warp(v_full, (uint32_t)(i & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int g = half; g < a.G; g += 2) {
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

bool make_map(CUtensorMap* m, CUtensorMapDataType ty, const void* base, int64_t cols, int64_t rows,
              int64_t row_bytes, int box_cols, int box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t gstride[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return enc(m, ty, 2, const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ring depths that fit one CTA's shared memory
int plan(int n16, int esz, F2Args* a) {
  a->x_stage_bytes = kTM * 32 * esz;
  a->b_stage_bytes = 2 * n16 * 64;
  const int limit = 227 * 1024;
  for (int bs = 3; bs >= 2; --bs)
    for (int xs = 4; xs >= 2; --xs) {
      const int bytes = xs * a->x_stage_bytes + 4 * kAStage + bs * a->b_stage_bytes + kMisc + 1024;
      if (bytes <= limit) {
        a->xs = xs, a->as = 4, a->bs = bs;
        return bytes;
      }
    }
  a->xs = 2, a->as = 2, a->bs = 2;
  return 2 * a->x_stage_bytes + 2 * kAStage + 2 * a->b_stage_bytes + kMisc + 1024;
}

}  // namespace

int launch_quant_fused2(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride, uint32_t* codes,
                        uint32_t* signs, float* norms, void* rnorms, int64_t out_stride, void* stream,
                        const int64_t* slots, int rn_f16) {
  cudaStream_t s = (cudaStream_t)stream;
  const bool prod = h->variant == TQ_PROD;
  if (int e = launch_gen_norms(h, x, dtype, N, x_stride, norms, out_stride, stream, nullptr, slots)) return e;
  F2Args a;
  a.N = N;
  a.d = h->d;
  a.n16 = h->fz_n16;
  a.G = (h->d + 31) / 32;
  a.kc = a.G;
  a.W = a.G * h->bm;
  a.out_stride = out_stride;
  a.prod = prod ? 1 : 0;
  a.xbf16 = dtype == TQ_BF16 ? 1 : 0;
  a.norms = norms;
  a.codes = codes;
  a.signs = prod ? signs : nullptr;
  a.rnorms = prod ? static_cast<float*>(rnorms) : nullptr;
  a.slots = slots;
  a.rn_f16 = rn_f16;
  a.thresholds = h->dev.thresholds;
  a.centroids = h->dev.centroids;
  a.acc_scale = kFusedPieceScale;
  const int esz = a.xbf16 ? 2 : 4;
  const int smem = plan(a.n16, esz, &a);
  a.row_tiles = (N + kTM - 1) / kTM;
  a.status = h->dev.status;
  CUtensorMap xm, pm, tm;
  if (!make_map(&xm, a.xbf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, x, h->d, N,
                x_stride * esz, 32, kTM, a.xbf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B))
    return (int)cudaErrorInvalidValue;
  if (!make_map(&pm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, h->dev.fz_pi, h->fz_k64, 2 * a.n16, (int64_t)h->fz_k64 * 2, 32,
                a.n16, CU_TENSOR_MAP_SWIZZLE_64B))
    return (int)cudaErrorInvalidValue;
  if (!make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, prod ? h->dev.fz_t : h->dev.fz_pi, h->fz_k64, 2 * a.n16,
                (int64_t)h->fz_k64 * 2, 32, a.n16, CU_TENSOR_MAP_SWIZZLE_64B))
    return (int)cudaErrorInvalidValue;
  const int grid = (int)(a.row_tiles < h->sm_count ? a.row_tiles : h->sm_count);
  auto go = [&](auto kern) -> int {
    if (int e = ensure_dyn_smem((const void*)kern, smem)) return e;
    kern<<<grid, kThreads, smem, s>>>(xm, pm, tm, a);
    return (int)cudaGetLastError();
  };
  if (h->variant == TQ_POLAR) {
    a.prod = 0;
    a.W = TQ_POLAR_WORDS(h->polar_b1, h->polar_bh, h->d);
    PolarDec& P = a.pol;
    P.b1 = h->polar_b1;
    P.bh = h->polar_bh;
    P.L = 0;
    while ((1 << P.L) < h->d) ++P.L;
    P.t1[0] = (float)std::tan(M_PI / 8);
    P.t1[1] = 1.f;
    P.t1[2] = (float)std::tan(3 * M_PI / 8);
    P.base[2] = 0;
    for (int l = 2; l < 8; ++l) P.base[l + 1] = P.base[l] + (h->d >> l);
    for (int l = 0; l < 8; ++l)
      for (int k = 0; k < 3; ++k) P.T[l][k] = (l >= 2 && l <= P.L) ? h->polar_tan2[l][k] : 0.f;
    P.w1 = TQ_CODE_WORDS(P.b1, h->d / 2);
    return h->d == 64 ? go(quant_fused2_kernel<1, 64>) : go(quant_fused2_kernel<1, 128>);
  }
  switch (h->bm) {
    case 1: return go(quant_fused2_kernel<1, 0>);
    case 2: return go(quant_fused2_kernel<2, 0>);
    case 3: return go(quant_fused2_kernel<3, 0>);
    default: return go(quant_fused2_kernel<4, 0>);
  }
}

}  // namespace tqi
