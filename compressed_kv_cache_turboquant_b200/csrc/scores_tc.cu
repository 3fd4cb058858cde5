// Inner-product scores of many queries against many TurboQuant vectors on the
// tensor cores (sm_100a), with a fused top-k.
//
// tmdm.cn ("谷歌悄悄扔下一颗“性能核弹”…", 双剑合璧 / ✦ QJL): the unbiased estimator
// corrects the quantization error while the score is computed; m.admirer.cn
// ("TurboQuant: Online Vector Quantization with Near-optimal Distortion Rate",
// 內存價格能下來嗎？): nearest-neighbour search over the codes.
//
// The estimate of a (query, key) pair is
//   s = n <q', c[idx]> + rn sqrt(pi/2)/d <q'', sigma>,   q' = Pi q, q'' = S q,
// two dot products whose key-side factors are exact small tables: the
// codebook (held in fp16 as alpha c[idx], with one fp32 scale alpha chosen so
// those values are nearly exact fp16 numbers) and the signs +-1.  A tile of
// 128 queries x TN keys is therefore a GEMM with fp32 accumulators in TMEM, one
// for the codebook part and (TurboQuant_prod) one for the sign part, and the
// per-key factors n / alpha and rn sqrt(pi/2)/d are applied in fp32 in the
// epilogue.  The query side of the codebook part is split as q' s = hi + lo
// (two fp16 pieces, s a power of two per query) and both pieces multiply the
// same decoded key chunk, so those products carry the query to about 2^-22;
// the sign part (a term of size ~||r|| ||q|| / sqrt(d)) takes q'' s in one fp16
// piece, whose rounding stays below 2e-5 of the score bound.
//
// Persistent CTAs walk (query tile, key tile) work items in query-tile-major
// order; the epilogue keeps a running top-k per query (k <= 16) and writes
// candidates when the query tile changes; a merge kernel combines candidates
// of the CTAs that covered a query tile.
//   warp 0      TMA producer of query chunks [128 x 64] fp16 (hi and lo)
//   warp 1      TMEM allocation and the MMA issuer
//   warps 2-9   decoders: 256 threads, one (key, 32-coordinate group) pair
//               each (prod: 128 keys x 2 groups; mse: 256 keys x both groups);
//               each thread stages its own packed words for the chunks ahead in
//               a shared-memory ring with 4-byte asynchronous copies
//   warps 10-13 epilogue: one thread per query row
// Tiles: TurboQuant_mse 128 x 256 with one accumulator, TurboQuant_prod
// 128 x 128 with two; either way two accumulator sets (512 TMEM columns) let the
// epilogue of one tile overlap the MMAs of the next.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>

#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;

constexpr int kTM = 128;          // queries per tile
constexpr int kAStages = 3;
constexpr int kABytes = kTM * 128;  // one 64-wide fp16 chunk of the query tile
constexpr int kTabBytes = 32768;
constexpr int kThreads = 448;
constexpr int kKMax = 16;          // largest fused top-k
// per-key factor buffers: the decoders start item j only after the MMA issuer
// has released all but kBStages chunks of item j-1, and the issuer is at most
// two items ahead of the epilogue, so items closer than 2 + kBStages + 1 apart
// never share a buffer
constexpr int kMkBufs = 8;

template <bool PROD>
struct Tile {
  static constexpr int TN = PROD ? 128 : 256;       // keys per tile
  static constexpr int BStages = PROD ? 3 : 2;
  static constexpr int BBytes = TN * 128;           // one 64-wide fp16 chunk of the key tile
  static constexpr int Tabs = PROD ? 2 : 1;         // codebook table (+ sign table)
  static constexpr int Ring = PROD ? 8 : 4;         // staged chunks ahead per decoder thread
  static constexpr int RingWords = 8;               // words staged per key per chunk (4 per group)
  static constexpr int RingBytes = Ring * TN * RingWords * 4;
  static constexpr int TopkBytes = 2 * kKMax * kTM * 4;  // running top-k values and indices per query row
  static constexpr int Smem = kAStages * kABytes + BStages * BBytes + Tabs * kTabBytes + kMkBufs * TN * 8 +
                              RingBytes + TopkBytes + 512 + 1024;
};

struct ScArgs {
  const uint32_t* codes;
  const uint32_t* signs;
  const float* norms;
  const float* rnorms;
  const float* inv_s;   // [nq_pad] 1 / query scale
  int64_t nq, N;
  int d, d_pad, bm, W, G;
  int64_t qt_count, kt_count, total;  // work items = qt_count * kt_count
  float qjl_coef;       // sqrt(pi/2) / d
  float inv_alpha;      // 1 / codebook scale
  float* scores;        // [nq][N] or null
  int topk;
  float* cand_val;      // [G][max_seg][128][topk]
  int32_t* cand_idx;
  int max_seg;
  uint32_t ctab[8];     // fp16 alpha c[k] pairs (k = 2i in the low half)
  int* status;
};

__host__ __device__ __forceinline__ int64_t first_item(int64_t i, int64_t total, int64_t G) { return i * total / G; }

__device__ __forceinline__ uint32_t ctab_at(const ScArgs& a, uint32_t k) {
  return (a.ctab[k >> 1] >> (16 * (k & 1u))) & 0xFFFFu;
}

// one group of 32 coordinates (BM words) -> 16 fp16 pairs (coordinate order)
// of the scaled codebook, by byte-indexed lookups in per-lane table copies
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 ld_s64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 ld_s128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// (the table addresses below are 32-bit shared-window addresses: this kernel aligns its
// shared base through an integer, after which plain pointers would compile to generic loads)
template <int BM>
__device__ __forceinline__ void decode_mse32(const uint32_t* p, uint32_t tab, int lane, uint32_t (&o)[16]) {
  if constexpr (BM == 3) {
    const uint32_t s3 = ((p[0] >> 3) & 0x11111111u) | ((p[1] >> 2) & 0x22222222u) | ((p[2] >> 1) & 0x44444444u);
    const uint32_t ws[4] = {p[0], p[1], p[2], s3};
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[4 * q + i] = ld_s32(tab + ((ws[q] >> (8 * i)) & 0xFFu) * 128 + lane * 4);
  } else if constexpr (BM == 2) {
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint2 v = ld_s64(tab + ((p[k] >> (8 * i)) & 0xFFu) * 128 + (lane & 15) * 8);
        o[8 * k + 2 * i] = v.x;
        o[8 * k + 2 * i + 1] = v.y;
      }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = ld_s128(tab + ((p[0] >> (8 * i)) & 0xFFu) * 128 + (lane & 7) * 16);
      o[4 * i + 0] = v.x;
      o[4 * i + 1] = v.y;
      o[4 * i + 2] = v.z;
      o[4 * i + 3] = v.w;
    }
  }
}

// 32 sign bits -> 16 fp16 pairs of +-1
__device__ __forceinline__ void decode_sign32(uint32_t sw, uint32_t tab, int lane, uint32_t (&o)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = ld_s128(tab + ((sw >> (8 * i)) & 0xFFu) * 128 + (lane & 7) * 16);
    o[4 * i + 0] = v.x;
    o[4 * i + 1] = v.y;
    o[4 * i + 2] = v.z;
    o[4 * i + 3] = v.w;
  }
}

// Insert (s, key) into the descending top-K list (bv, bi) of one query row
// (s > bv[K-1] on entry); an equal score stays behind the earlier, lower key.
// Rare after the first keys, so kept out of line: the unrolled epilogue only
// compares against the returned new k-th value.
// The lists live in shared memory, entry j of row r at [j * 128 + r]: this
// kernel leaves L1 almost no room beside its shared memory, so a list in local
// memory would be an L2 round trip per access.
__device__ __noinline__ float topk_insert(float* bv, int32_t* bi, int K, float s, int32_t key) {
  int j = K - 1;
  while (j > 0 && bv[(j - 1) * kTM] < s) {
    bv[j * kTM] = bv[(j - 1) * kTM];
    bi[j * kTM] = bi[(j - 1) * kTM];
    --j;
  }
  bv[j * kTM] = s;
  bi[j * kTM] = key;
  return bv[(K - 1) * kTM];
}

template <bool PROD, int BM>
__global__ void __launch_bounds__(kThreads, 1) scores_tc_kernel(const __grid_constant__ CUtensorMap qmap, ScArgs a) {
  using T = Tile<PROD>;
  constexpr int TN = T::TN, kBStages = T::BStages, kBBytes = T::BBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem;                                  // [kAStages][kABytes]
  uint8_t* b_s = a_s + kAStages * kABytes;              // [kBStages][kBBytes]
  uint8_t* mtab = b_s + kBStages * kBBytes;             // codebook table (layout by bm)
  uint8_t* stab = mtab + kTabBytes;                     // sign table (prod)
  // per-key factors of each work item: n / alpha (negative = no key) and rn sqrt(pi/2)/d
  float* mk_s = reinterpret_cast<float*>(mtab + T::Tabs * kTabBytes);  // [kMkBufs][TN]
  float* qk_s = mk_s + kMkBufs * TN;                                   // [kMkBufs][TN]
  uint32_t* ring_s = reinterpret_cast<uint32_t*>(qk_s + kMkBufs * TN); // [Ring][TN][RingWords]
  float* tkv_s = reinterpret_cast<float*>(ring_s + T::Ring * TN * T::RingWords);  // [kKMax][128]
  int32_t* tki_s = reinterpret_cast<int32_t*>(tkv_s + kKMax * kTM);               // [kKMax][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(tki_s + kKMax * kTM);
  uint64_t* a_full = bars;                 // [kAStages]
  uint64_t* a_empty = a_full + kAStages;   // [kAStages]
  uint64_t* b_full = a_empty + kAStages;   // [kBStages] count 128
  uint64_t* b_empty = b_full + kBStages;   // [kBStages]
  uint64_t* acc_full = b_empty + kBStages; // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2] count 128
  uint64_t* done_bar = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t it_lo = first_item(blockIdx.x, a.total, G), it_hi = first_item(blockIdx.x + 1, a.total, G);
  const int nkc_m = a.d_pad / 64;              // key chunks of the codebook part
  const int nkc = nkc_m * (PROD ? 2 : 1);      // key chunks in all (each meets a hi and a lo query chunk)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAStages; ++s) mbar_init(&a_full[s], 1), mbar_init(&a_empty[s], 1);
    for (int s = 0; s < kBStages; ++s) mbar_init(&b_full[s], 256), mbar_init(&b_empty[s], 1);
    for (int s = 0; s < 2; ++s) mbar_init(&acc_full[s], 1), mbar_init(&acc_empty[s], 128);
    mbar_init(done_bar, 1);
    fence_mbar_init();
  }
  // tables: codebook entries by bm, and +-1 sign pairs (8 copies of 16 bytes per row)
  for (int w = threadIdx.x; w < kTabBytes / 4; w += blockDim.x) {
    const uint32_t row = (uint32_t)w >> 5, col = (uint32_t)w & 31u;
    uint32_t v;
    if (BM == 3) {
      v = ctab_at(a, row & 7u) | (ctab_at(a, (row >> 4) & 7u) << 16);
    } else if (BM == 2) {  // 16 copies of 2 pairs (4 two-bit codes)
      const uint32_t pr = col & 1u, i0 = (row >> (4 * pr)) & 3u, i1 = (row >> (4 * pr + 2)) & 3u;
      v = ctab_at(a, i0) | (ctab_at(a, i1) << 16);
    } else {  // 8 copies of 4 pairs (8 one-bit codes)
      const uint32_t pr = col & 3u, i0 = (row >> (2 * pr)) & 1u, i1 = (row >> (2 * pr + 1)) & 1u;
      v = ctab_at(a, i0) | (ctab_at(a, i1) << 16);
    }
    reinterpret_cast<uint32_t*>(mtab)[w] = v;
    if (PROD) {
      const uint32_t pr = col & 3u;
      const uint32_t lo = ((row >> (2 * pr)) & 1u) ? 0x3C00u : 0xBC00u;
      const uint32_t hi = ((row >> (2 * pr + 1)) & 1u) ? 0x3C00u : 0xBC00u;
      reinterpret_cast<uint32_t*>(stab)[w] = lo | (hi << 16);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // per key chunk kc: the hi query chunk kc, then (codebook part) the lo chunk nkc + kc
      int64_t ch = 0;
      bool ok = true;
      for (int64_t it = it_lo; ok && it < it_hi; ++it) {
        const int64_t qt = it / a.kt_count;
        for (int kc = 0; ok && kc < nkc; ++kc) {
          for (int piece = 0; piece < (kc < nkc_m ? 2 : 1); ++piece, ++ch) {
            const int s = (int)(ch % kAStages);
            const uint32_t u = (uint32_t)(ch / kAStages);
            if (!mbar_wait(&a_empty[s], (u & 1u) ^ 1u)) {
              atomicOr(a.status, kStatusTimeout);
              ok = false;
              break;
            }
            const int col = piece ? nkc + kc : kc;
            mbar_arrive_expect_tx(&a_full[s], kABytes);
            tma_load_2d(&qmap, &a_full[s], a_s + s * kABytes, col * 64, (int)(qt * kTM));
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(kTM, TN, false);
      const uint32_t aaddr = smem_u32(a_s), baddr = smem_u32(b_s);
      int64_t cha = 0, chb = 0;
      bool ok = true;
      int i = 0;
      for (int64_t it = it_lo; ok && it < it_hi; ++it, ++i) {
        const int ab = i & 1;
        const uint32_t ua = (uint32_t)(i >> 1);
        if (!mbar_wait(&acc_empty[ab], (ua & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kc = 0; ok && kc < nkc; ++kc, ++chb) {
          const int sb = (int)(chb % kBStages);
          if (!mbar_wait(&b_full[sb], (uint32_t)((chb / kBStages) & 1))) {
            ok = false;
            break;
          }
          const bool qpart = PROD && kc >= nkc_m;
          const uint32_t d_tmem = tmem_base + (uint32_t)(ab * 256) + (qpart ? 128u : 0u);
          const int kfirst = qpart ? nkc_m : 0;
          for (int piece = 0; piece < (kc < nkc_m ? 2 : 1); ++piece, ++cha) {
            const int sa = (int)(cha % kAStages);
            if (!mbar_wait(&a_full[sa], (uint32_t)((cha / kAStages) & 1))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              mma_f16(d_tmem, sw128_kmajor_desc(aaddr + sa * kABytes + k4 * 32),
                      sw128_kmajor_desc(baddr + sb * kBBytes + k4 * 32), idesc,
                      (kc != kfirst || piece != 0 || k4 != 0) ? 1u : 0u);
            mma_commit(&a_empty[sa]);
          }
          if (!ok) break;
          mma_commit(&b_empty[sb]);
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done_bar);
    }
  } else if (warp < 10) {
    // decoders.  Thread t takes key row kr of the tile and, for prod, group hf
    // of each 64-coordinate chunk (mse: both groups).  The words of flattened
    // chunk c (item it_lo + c / nkc, key chunk c % nkc) land in ring slot
    // c % Ring, row kr, words 4 j .. 4 j + 3 for group j; word 3 (7) of a tile's
    // first chunk carries n (rn).  Each thread copies what it decodes, Ring - 1
    // chunks ahead, so a wait for its own copy groups is the only sync needed.
    const int t = threadIdx.x - 64;
    constexpr int R = T::Ring, RW = T::RingWords;
    constexpr int NG = PROD ? 1 : 2;          // groups per thread per chunk
    const int kr = PROD ? (t & 127) : t;      // key row in the tile
    const int hf = PROD ? (t >> 7) : 0;       // first group (within the chunk)
    const int64_t nch = (it_hi - it_lo) * nkc;
    // the next chunk to stage, as (flattened index, key tile, key chunk), advanced by one
    // per call (no 64-bit division per chunk)
    int64_t iss_c = 0, iss_kt = it_lo % a.kt_count;
    int iss_kc = 0;
    auto issue = [&]() {
      const int64_t c = iss_c;
      if (c < nch) {
        const int64_t kt = iss_kt;
        const int kc = iss_kc;
        const bool qpart = PROD && kc >= nkc_m;
        const int g0 = 2 * (qpart ? kc - nkc_m : kc);
        const int64_t key = kt * TN + kr;
        if (key < a.N) {
          uint32_t* dst = ring_s + ((size_t)(c % R) * TN + kr) * RW;
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            const int gj = hf + j;  // group within the chunk
            const int g = g0 + gj;
            if (g >= a.G) break;
            if (!qpart) {
              const uint32_t* src = a.codes + key * a.W + g * BM;
#pragma unroll
              for (int q = 0; q < BM; ++q) cp_async4(dst + 4 * gj + q, src + q);
            } else {
              cp_async4(dst + 4 * gj, a.signs + key * a.G + g);
            }
          }
          if (kc == 0) {
            if (hf == 0) cp_async4(dst + 3, a.norms + key);
            else cp_async4(dst + 7, a.rnorms + key);
          }
        }
      }
      cp_async_commit();  // one group per chunk, empty or not
      ++iss_c;
      if (++iss_kc == nkc) {
        iss_kc = 0;
        if (++iss_kt == a.kt_count) iss_kt = 0;
      }
    };
    for (int64_t c = 0; c < R - 1; ++c) issue();
    int64_t ch = 0;
    int i = 0;
    bool ok = true;
    for (int64_t it = it_lo; ok && it < it_hi; ++it, ++i) {
      const int64_t kt = it % a.kt_count;
      const bool valid = kt * TN + kr < a.N;
      float* mk = mk_s + (i % kMkBufs) * TN;
      float* qk = qk_s + (i % kMkBufs) * TN;
      for (int kc = 0; kc < nkc; ++kc, ++ch) {
        issue();  // chunk ch + R - 1
        cp_async_wait<R - 1>();  // this thread's copies of chunk ch have landed
        const uint32_t* slot = ring_s + ((size_t)(ch % R) * TN + kr) * RW;
        if (kc == 0) {
          if (hf == 0) mk[kr] = valid ? __uint_as_float(slot[3]) * a.inv_alpha : -1.f;
          else qk[kr] = valid ? __uint_as_float(slot[7]) * a.qjl_coef : 0.f;
        }
        const int sb = (int)(ch % kBStages);
        if (!mbar_wait_warp(&b_empty[sb], (uint32_t)(((ch / kBStages) & 1) ^ 1))) {
          ok = false;
          break;
        }
        uint8_t* brow = b_s + sb * kBBytes + kr * 128;
        const bool qpart = PROD && kc >= nkc_m;
        const int g0 = 2 * (qpart ? kc - nkc_m : kc);
#pragma unroll
        for (int j = 0; j < NG; ++j) {
          const int gj = hf + j;
          uint32_t o[16];
          if (!valid || g0 + gj >= a.G) {
#pragma unroll
            for (int q = 0; q < 16; ++q) o[q] = 0u;
          } else if (!qpart) {
            const uint4 w = *reinterpret_cast<const uint4*>(slot + 4 * gj);
            const uint32_t p[3] = {w.x, w.y, w.z};
            decode_mse32<BM>(p, smem_u32(mtab), lane, o);
          } else {
            decode_sign32(slot[4 * gj], smem_u32(stab), lane, o);
          }
          // 16-byte units 4 gj .. 4 gj + 3 of the key's row, 128B-swizzled
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(brow + (((4 * gj + u) ^ (kr & 7)) * 16)) =
                make_uint4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
        }
        fence_async_smem();
        mbar_arrive(&b_full[sb]);
      }
    }
    cp_async_wait<0>();  // no copy may still be writing when the block exits
    if (!ok) atomicOr(a.status, kStatusTimeout);
  } else {
    // epilogue: thread = query row of the tile
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    float* bv = tkv_s + row;    // entry j at bv[j * 128]
    int32_t* bi = tki_s + row;
    const int K = a.topk;
    float kth = -FLT_MAX;  // bv[K - 1], kept in a register
    int64_t cur_qt = -1;
    int seg = -1;
    int i = 0;
    auto flush = [&]() {
      if (seg < 0 || K == 0) return;
      const int64_t base = (((int64_t)blockIdx.x * a.max_seg + seg) * kTM + row) * K;
      for (int j = 0; j < K; ++j) a.cand_val[base + j] = bv[j * kTM], a.cand_idx[base + j] = bi[j * kTM];
    };
    for (int64_t it = it_lo; it < it_hi; ++it, ++i) {
      const int64_t qt = it / a.kt_count, kt = it % a.kt_count;
      if (qt != cur_qt) {
        flush();
        ++seg;
        cur_qt = qt;
        for (int j = 0; j < kKMax; ++j) bv[j * kTM] = -FLT_MAX, bi[j * kTM] = INT32_MAX;
        kth = -FLT_MAX;
      }
      const int ab = i & 1;
      if (!mbar_wait_warp(&acc_full[ab], (uint32_t)((i >> 1) & 1))) {
        atomicOr(a.status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const int64_t q = qt * kTM + row;
      const float invs = a.inv_s[q];
      const float* mk = mk_s + (i % kMkBufs) * TN;
      const float* qk = qk_s + (i % kMkBufs) * TN;
      const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * 256);
      for (int c = 0; c < TN / 32; ++c) {
        float v[32], vq[32];
        tmem_ld32(t0 + c * 32, v);
        if (PROD) tmem_ld32(t0 + 128 + c * 32, vq);
        // per-key factors of the 32 columns (same for every row: broadcast reads)
        float mv[32], qv[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 m4 = *reinterpret_cast<const float4*>(mk + c * 32 + 4 * u);
          mv[4 * u] = m4.x, mv[4 * u + 1] = m4.y, mv[4 * u + 2] = m4.z, mv[4 * u + 3] = m4.w;
          if (PROD) {
            const float4 q4 = *reinterpret_cast<const float4*>(qk + c * 32 + 4 * u);
            qv[4 * u] = q4.x, qv[4 * u + 1] = q4.y, qv[4 * u + 2] = q4.z, qv[4 * u + 3] = q4.w;
          }
        }
        tmem_wait_ld();
        uint32_t hits = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float sc = PROD ? fmaf(mv[e], v[e], qv[e] * vq[e]) * invs : mv[e] * v[e] * invs;
          v[e] = mv[e] < 0.f ? -FLT_MAX : sc;  // no key in this column
          hits |= (v[e] > kth ? 1u : 0u) << e;
        }
        const int64_t key0 = kt * TN + c * 32;
        if (a.scores && q < a.nq) {
          const int nvalid = (int)((a.N - key0) < 32 ? (a.N - key0) : 32);
          float* dst = a.scores + q * a.N + key0;
          if (nvalid == 32 && ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0)) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<float4*>(dst + 4 * u) = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < nvalid) dst[e] = v[e];
          }
        }
        if (K > 0 && hits) {
          // rare after the first keys: insert the candidates straight from registers
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (((hits >> e) & 1u) && v[e] > kth) kth = topk_insert(bv, bi, K, v[e], (int32_t)(key0 + e));
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
    flush();
  }

  __syncthreads();
  if (warp == 1) {
    if (!mbar_wait(done_bar, 0) && lane == 0) atomicOr(a.status, kStatusTimeout);
    __syncwarp();
    tmem_dealloc(tmem_base, 512);
  }
}

// [q'; q''] s per query (s a power of two putting the largest entry in
// [2^13, 2^14)) in fp16, each part padded to d_pad: row = [hi(q' s), hi(q'' s) |
// lo(q' s)], lo = q' s - hi (exact in fp32, then rounded); 1/s kept
__global__ void qcat_kernel(const float* qrot, const float* qproj, int64_t nq, int64_t nq_pad, int d, int d_pad,
                            int prod, __half* qcat, float* inv_s) {
  const int64_t qi = blockIdx.x;
  const int half = d_pad * (prod ? 2 : 1);
  const int kdim = half + d_pad;
  __shared__ float red[32];
  float m = 0.f;
  if (qi < nq)
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
      m = fmaxf(m, fabsf(qrot[qi * d + j]));
      if (prod) m = fmaxf(m, fabsf(qproj[qi * d + j]));
    }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float mx = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
  int e = 0;
  if (mx > 0.f) (void)frexpf(mx, &e);
  const float s = (mx > 0.f) ? ldexpf(1.f, 14 - e) : 1.f;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    float v = 0.f;
    if (qi < nq) {
      if (j < d) v = qrot[qi * d + j];
      else if (prod && j >= d_pad && j - d_pad < d) v = qproj[qi * d + (j - d_pad)];
    }
    const float vs = v * s;  // exact: s is a power of two
    const __half hi = __float2half_rn(vs);
    qcat[qi * kdim + j] = hi;
    if (j < d_pad) qcat[qi * kdim + half + j] = __float2half_rn(vs - __half2float(hi));
  }
  if (threadIdx.x == 0) inv_s[qi] = (qi < nq) ? 1.f / s : 0.f;
}

// per query: top-k of the candidates written by the CTAs that covered its tile
__global__ void topk_merge_kernel(const float* cand_val, const int32_t* cand_idx, int64_t nq, int64_t G,
                                  int max_seg, int64_t total, int64_t kt_count, int K, int32_t* top_idx,
                                  float* top_val) {
  const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= nq) return;
  const int64_t qt = q / kTM, row = q % kTM;
  const int64_t lo = qt * kt_count, hi = lo + kt_count;
  int64_t i = lo * G / total;
  while (i > 0 && first_item(i, total, G) > lo) --i;
  while (i < G && first_item(i + 1, total, G) <= lo) ++i;
  float bv[kKMax];
  int32_t bi[kKMax];
  for (int j = 0; j < kKMax; ++j) bv[j] = -FLT_MAX, bi[j] = INT32_MAX;
  for (; i < G && first_item(i, total, G) < hi; ++i) {
    const int64_t sg = qt - first_item(i, total, G) / kt_count;
    const int64_t base = ((i * max_seg + sg) * kTM + row) * K;
    for (int j = 0; j < K; ++j) {
      float cv = cand_val[base + j];
      int32_t ci = cand_idx[base + j];
      if (ci == INT32_MAX) continue;
      for (int t = 0; t < K; ++t) {
        if (cv > bv[t] || (cv == bv[t] && ci < bi[t])) {
          const float tv = bv[t];
          const int32_t ti = bi[t];
          bv[t] = cv, bi[t] = ci;
          cv = tv, ci = ti;
        }
      }
    }
  }
  for (int j = 0; j < K; ++j) top_val[q * K + j] = bv[j], top_idx[q * K + j] = bi[j];
}


}  // namespace

struct ScoresPlan {
  int64_t nq_pad, qt, kt, total, G;
  int tn, d_pad, kdim, max_seg;
};

static ScoresPlan scores_plan(const tq_ctx* h, int64_t nq, int64_t N) {
  ScoresPlan p;
  const bool prod = h->variant == TQ_PROD;
  p.tn = prod ? Tile<true>::TN : Tile<false>::TN;
  p.nq_pad = (nq + kTM - 1) / kTM * kTM;
  p.d_pad = (h->d + 63) / 64 * 64;
  p.kdim = p.d_pad * (prod ? 3 : 2);  // hi of q' (and q''), lo of q'
  p.qt = p.nq_pad / kTM;
  p.kt = (N + p.tn - 1) / p.tn;
  p.total = p.qt * p.kt;
  p.G = p.total < h->sm_count ? p.total : h->sm_count;
  const int64_t per = (p.total + p.G - 1) / p.G;
  p.max_seg = (int)((per + p.kt - 1) / p.kt + 1);
  return p;
}

bool scores_tc_supported(const tq_ctx* h, int topk) {
  return h->bm >= 1 && h->bm <= 3 && topk <= kKMax && h->d >= 32;
}

size_t scores_tc_workspace(const tq_ctx* h, int64_t nq, int64_t N, int topk) {
  const ScoresPlan p = scores_plan(h, nq, N);
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t b = 2 * al((size_t)nq * h->d * 4);                 // q', q'' fp32
  b += al((size_t)p.nq_pad * p.kdim * 2) + al((size_t)p.nq_pad * 4);  // fp16 queries, scales
  if (topk > 0) b += 2 * al((size_t)p.G * p.max_seg * kTM * topk * 4);
  return b;
}

int launch_scores_tc(const tq_ctx* h, const float* q, int64_t nq, const uint32_t* codes, const uint32_t* signs,
                     const float* norms, const float* rnorms, int64_t N, float* scores, int topk, int32_t* top_idx,
                     float* top_val, void* workspace, void* stream) {
  const ScoresPlan p = scores_plan(h, nq, N);
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  char* ws = (char*)workspace;
  float* qrot = (float*)ws;
  ws += al((size_t)nq * h->d * 4);
  float* qproj = (float*)ws;
  ws += al((size_t)nq * h->d * 4);
  __half* qcat = (__half*)ws;
  ws += al((size_t)p.nq_pad * p.kdim * 2);
  float* inv_s = (float*)ws;
  ws += al((size_t)p.nq_pad * 4);
  float* cv = nullptr;
  int32_t* ci = nullptr;
  if (topk > 0) {
    cv = (float*)ws;
    ws += al((size_t)p.G * p.max_seg * kTM * topk * 4);
    ci = (int32_t*)ws;
  }
  const bool prod = h->variant == TQ_PROD;
  cudaStream_t s = (cudaStream_t)stream;
  int e = launch_query_prep(h, q, TQ_F32, nq, qrot, prod ? qproj : nullptr, stream);
  if (e) return e;
  qcat_kernel<<<(unsigned)p.nq_pad, 128, 0, s>>>(qrot, qproj, nq, p.nq_pad, h->d, p.d_pad, prod ? 1 : 0, qcat, inv_s);
  if ((e = (int)cudaGetLastError())) return e;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return (int)cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t gdim[2] = {(cuuint64_t)p.kdim, (cuuint64_t)p.nq_pad};
  const cuuint64_t gstride[1] = {(cuuint64_t)p.kdim * 2};
  const cuuint32_t box[2] = {64, kTM};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, qcat, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
      CUDA_SUCCESS)
    return (int)cudaErrorInvalidValue;
  ScArgs a;
  a.codes = codes;
  a.signs = signs;
  a.norms = norms;
  a.rnorms = rnorms;
  a.inv_s = inv_s;
  a.nq = nq;
  a.N = N;
  a.d = h->d;
  a.d_pad = p.d_pad;
  a.bm = h->bm;
  a.G = (h->d + 31) / 32;
  a.W = a.G * h->bm;
  a.qt_count = p.qt;
  a.kt_count = p.kt;
  a.total = p.total;
  a.qjl_coef = 1.2533141373155003f / (float)h->d;
  a.inv_alpha = h->sc_inv_alpha;
  a.scores = scores;
  a.topk = topk;
  a.cand_val = cv;
  a.cand_idx = ci;
  a.max_seg = p.max_seg;
  for (int k = 0; k < 8; ++k) a.ctab[k] = (uint32_t)h->sc_tab[2 * k] | ((uint32_t)h->sc_tab[2 * k + 1] << 16);
  a.status = h->dev.status;
  auto launch = [&](auto kern, int smem) -> int {
    if (int ee = ensure_dyn_smem((const void*)kern, smem)) return ee;
    kern<<<(unsigned)p.G, kThreads, smem, s>>>(map, a);
    return 0;
  };
  if (prod) {
    switch (h->bm) {
      case 1: e = launch(scores_tc_kernel<true, 1>, Tile<true>::Smem); break;
      case 2: e = launch(scores_tc_kernel<true, 2>, Tile<true>::Smem); break;
      default: e = launch(scores_tc_kernel<true, 3>, Tile<true>::Smem); break;
    }
  } else {
    switch (h->bm) {
      case 1: e = launch(scores_tc_kernel<false, 1>, Tile<false>::Smem); break;
      case 2: e = launch(scores_tc_kernel<false, 2>, Tile<false>::Smem); break;
      default: e = launch(scores_tc_kernel<false, 3>, Tile<false>::Smem); break;
    }
  }
  if (e) return e;
  if ((e = (int)cudaGetLastError())) return e;
  if (topk > 0) {
    topk_merge_kernel<<<(unsigned)((nq + 127) / 128), 128, 0, s>>>(cv, ci, nq, p.G, p.max_seg, p.total, p.kt, topk,
                                                                   top_idx, top_val);
    e = (int)cudaGetLastError();
  }
  return e;
}

}  // namespace tqi
