// TurboQuant_mse quantization on the 5th-generation tensor cores (sm_100a).
//
// [ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: store the norm, rotate,
// quantize every coordinate on its own against the precomputed Lloyd-Max
// codebook, [ttakun, "为什么随机旋转是整个算法的底层杠杆"]: the rotation is a plain
// matrix product followed by branch-free scalar work
// (ttakun.com/news/45354, "KV缓存52GB瞬间爆内存？TurboQuant随机旋转+标量量化…").
//
// One persistent CTA per SM, warp-specialised:
//   warp 0      TMA producer: 128-vector tiles of x (bf16, 128B-swizzled,
//               K-major) into a ring of shared-memory stages; the rotation
//               pieces are bulk-copied into shared memory once
//   warp 1      TMEM allocation and the single-thread MMA issuer:
//               Y[128 x d] = X[128 x d] . (Pi_hi + Pi_mid + Pi_lo)^T, three
//               bf16 passes accumulated in fp32 in TMEM (double-buffered)
//   warps 2-13  epilogue: three sets of four warps (one per TMEM lane
//               quarter) take the tiles in turn, each set with its own
//               accumulator buffer, so three tiles are in flight; one thread
//               per vector (TMEM lane) reads the vector's columns twice: once
//               for n = ||y|| (= ||x||, Pi orthogonal), once for the cell of
//               every coordinate against n * t_k, packing and stores.  Even
//               32-coordinate groups search the thresholds on the ALU pipe,
//               odd ones count them on the FMA pipe.
//
// Precision: x is exact in bf16; Pi = hi + mid + lo carries ~24 significant
// bits, so every product is exact in fp32 and y has fp32-level error (far
// inside the 1e-5/sqrt(d) band the decisions are allowed to differ in).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;

constexpr int kPieces = 3;
constexpr int kTileM = 128;
constexpr int kSets = 3;                  // epilogue warp sets = accumulator buffers
// warps: TMA producer, MMA issuer, kSets sets of 4 epilogue warps
template <int D>
constexpr int threads_for() { return 32 * (2 + 4 * kSets); }

template <int D>
struct TcShape {
  static constexpr int kSlabs = D / 64;                      // 128-byte K slabs
  static constexpr int kSlabBytesX = kTileM * 128;           // one slab of a 128-row x tile
  static constexpr int kStageBytes = kSlabs * kSlabBytesX;   // one x tile
  static constexpr int kSlabBytesPi = D * 128;               // one slab of a D-row piece
  static constexpr int kPieceBytes = kSlabs * kSlabBytesPi;  // = D * D * 2
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kTmemCols = (kSets * D <= 256) ? 256 : 512;  // kSets accumulators
  static constexpr int kMiscBytes = 8192;  // barriers, TMEM slot, thresholds, norm partials
  static constexpr int kSmemBytes = kPieces * kPieceBytes + kStages * kStageBytes + kMiscBytes +
                                    1024 /*alignment*/;
};

struct TcArgs {
  const uint8_t* pi_pieces;  // kPieces x [slab][row][128 B swizzled]
  const float* thresholds;   // [2^bm - 1]
  int64_t N;
  int64_t out_stride;
  uint32_t* codes;
  float* norms;
  int* status;
};

template <int BM>
__device__ __forceinline__ uint32_t cell_index(float y, const float (&P)[8]) {
  // P[m] = n * (m-th positive threshold), m = 1 .. 2^(BM-1) - 1 (symmetric codebook)
  constexpr uint32_t H = 1u << (BM - 1);
  const float a = fabsf(y);
  uint32_t m = 0;
  if constexpr (BM == 2) {
    m = (a >= P[1]) ? 1u : 0u;
  } else if constexpr (BM == 3) {
    const uint32_t m1 = (a >= P[2]) ? 1u : 0u;
    const float t = m1 ? P[3] : P[1];
    m = 2u * m1 + ((a >= t) ? 1u : 0u);
  } else if constexpr (BM == 4) {
    const uint32_t m2 = (a >= P[4]) ? 1u : 0u;
    const float t1 = m2 ? P[6] : P[2];
    const uint32_t m1 = (a >= t1) ? 1u : 0u;
    const float t2 = m2 ? (m1 ? P[7] : P[5]) : (m1 ? P[3] : P[1]);
    m = 4u * m2 + 2u * m1 + ((a >= t2) ? 1u : 0u);
  }
  // y >= 0 -> upper half H + m; y < 0 -> H - 1 - m (ties on a threshold: upper cell,
  // up to the exact-equality case that the parity band excuses)
  const uint32_t base = (y >= 0.f) ? H : H - 1u;
  return base ^ m;
}

// pack the 32 coordinates of one group (layout of include/tq.h)
template <int BM>
__device__ __forceinline__ void pack_group(const float* v, const float (&P)[8], uint32_t (&w)[BM]) {
#pragma unroll
  for (int k = 0; k < BM; ++k) w[k] = 0u;
  if constexpr (BM == 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[0] |= cell_index<1>(v[i], P) << i;
  } else if constexpr (BM == 2) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i >> 4] |= cell_index<2>(v[i], P) << (2 * (i & 15));
  } else if constexpr (BM == 4) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i >> 3] |= cell_index<4>(v[i], P) << (4 * (i & 7));
  } else {
    uint32_t X = 0u;
#pragma unroll
    for (int i = 0; i < 24; ++i) w[i >> 3] |= cell_index<3>(v[i], P) << (4 * (i & 7));
#pragma unroll
    for (int j = 0; j < 8; ++j) X |= cell_index<3>(v[24 + j], P) << (4 * j);
    w[0] |= (X << 3) & 0x88888888u;
    w[1] |= (X << 2) & 0x88888888u;
    w[2] |= (X << 1) & 0x88888888u;
  }
}

// The same cells computed on the FMA pipe (the binary search above runs on
// the ALU pipe, which the epilogue saturates at 3 and 4 bits; half of the
// groups go each way).  With B = 2^32 / n and C_k = 1 - 2^32 t_k, both rounded
// to float32:
//   sat(|y| B + C_k) = 1 when |y| >= n t_k and 0 when |y| < n t_k, up to a band
//   around the threshold: B carries the 2^-24 relative rounding of 2^32 / n and
//   C_k that of 2^32 t_k (its ulp is 32 to 256 for the thresholds here), so the
//   decision can move by about 2^-23 |t_k| in the unit frame y / n -- under
//   3e-8 at d = 128, some 30 times inside the parity band 1e-5 / sqrt(d) -- so
//   m = sum_k sat(|y| B + C_k) counts the positive thresholds at or below |y|,
//   s = sat(y B + 1) is 1 for y >= 0 (to the same band), and
//   cell = (H - 1 - m) + s (2m + 1).
// Adding 2^23 leaves the cell in the low mantissa bits, and integer
// multiply-adds shift it into place; the constant part of those bit patterns is
// cancelled by the starting value of each word.  A zero vector (n = 0) takes
// B = 0, C_k = -1: every count is 0 and s = 1, the cell above the middle.
template <int BM>
struct FmaCells {
  static constexpr int kFields = 32 / (BM == 3 ? 4 : BM);  // cells per word (3 bits: nibbles)
  static constexpr int kWidth = BM == 3 ? 4 : BM;
  __host__ __device__ static constexpr uint32_t init() {
    uint32_t c = 0u;
    for (int i = 0; i < kFields; ++i) c += (kWidth * i < 32) ? (0x4B000000u << (kWidth * i)) : 0u;
    return 0u - c;
  }
};

template <int BM>
__device__ __forceinline__ uint32_t cell_fma_bits(float y, float B, const float (&C)[8]) {
  constexpr int H = 1 << (BM - 1);
  const float s = __saturatef(fmaf(y, B, 1.f));
  float m = 0.f;
#pragma unroll
  for (int k = 1; k < H; ++k) m += __saturatef(fmaf(fabsf(y), B, C[k]));
  const float u = fmaf(m, 2.f, 1.f);
  const float v = ((float)(H - 1) + 8388608.f) - m;
  return __float_as_uint(fmaf(s, u, v));  // 0x4B000000 | cell
}

// pack one group of 32 coordinates with the FMA-pipe cells; for 3 bits the
// cells of coordinates 24..31 (spread over the spare bits) use the ALU search
template <int BM>
__device__ __forceinline__ void pack_group_fma(const float* v, const float (&P)[8], float B, const float (&C)[8],
                                               uint32_t (&w)[BM]) {
  using F = FmaCells<BM>;
#pragma unroll
  for (int k = 0; k < BM; ++k) w[k] = F::init();
  if constexpr (BM == 3) {
#pragma unroll
    for (int i = 0; i < 24; ++i) w[i >> 3] += cell_fma_bits<3>(v[i], B, C) * (1u << (4 * (i & 7)));
    uint32_t X = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) X |= cell_index<3>(v[24 + j], P) << (4 * j);
    w[0] |= (X << 3) & 0x88888888u;
    w[1] |= (X << 2) & 0x88888888u;
    w[2] |= (X << 1) & 0x88888888u;
  } else {
    constexpr int per = 32 / BM;
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i / per] += cell_fma_bits<BM>(v[i], B, C) * (1u << (BM * (i % per)));
  }
}

template <int BM>
__device__ __forceinline__ void store_words(uint32_t* dst, const uint32_t (&w)[BM]) {
  if constexpr (BM == 4) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (BM == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else {
#pragma unroll
    for (int k = 0; k < BM; ++k) dst[k] = w[k];
  }
}

template <int D, int BM>
__global__ void __launch_bounds__(threads_for<D>(), 1)
    quant_mse_tc_kernel(const __grid_constant__ CUtensorMap xmap, TcArgs a) {
  using S = TcShape<D>;
  constexpr int W = (D / 32) * BM;  // words per vector
  constexpr int K = 1 << BM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* pi_s = smem;
  uint8_t* x_s = smem + kPieces * S::kPieceBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(x_s + S::kStages * S::kStageBytes);
  uint64_t* full = bars;                       // [kStages]
  uint64_t* empty = bars + S::kStages;         // [kStages]
  uint64_t* acc_full = bars + 2 * S::kStages;  // [kSets]
  uint64_t* acc_empty = acc_full + kSets;      // [kSets]
  uint64_t* pi_bar = acc_empty + kSets;
  uint64_t* done_bar = pi_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  float* thr_s = reinterpret_cast<float*>(tmem_slot + 4);  // [16]
  constexpr int kGroups = D / 32;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (a.N + kTileM - 1) / kTileM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kSets; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(pi_bar, 1);
    mbar_init(done_bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < K - 1) thr_s[threadIdx.x] = a.thresholds[threadIdx.x];
  if (warp == 1) tmem_alloc(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // rotation pieces, once per CTA
      mbar_arrive_expect_tx(pi_bar, kPieces * S::kPieceBytes);
      for (int p = 0; p < kPieces; ++p)
        bulk_load(pi_s + p * S::kPieceBytes, a.pi_pieces + (size_t)p * S::kPieceBytes, S::kPieceBytes, pi_bar);
      int i = 0;
      for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
        const int s = i % S::kStages;
        const uint32_t u = (uint32_t)(i / S::kStages);
        if (!mbar_wait(&empty[s], (u & 1u) ^ 1u)) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        mbar_arrive_expect_tx(&full[s], S::kStageBytes);
        for (int sl = 0; sl < S::kSlabs; ++sl)
          tma_load_2d(&xmap, &full[s], x_s + s * S::kStageBytes + sl * S::kSlabBytesX, sl * 64,
                      (int)(tile * kTileM));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(kTileM, D, true);
      const uint32_t pi_addr = smem_u32(pi_s), x_addr = smem_u32(x_s);
      bool ok = mbar_wait(pi_bar, 0);
      int i = 0;
      for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++i) {
        const int s = i % S::kStages;
        const uint32_t u = (uint32_t)(i / S::kStages);
        const int ab = i % kSets;
        const uint32_t ua = (uint32_t)(i / kSets);
        if (!mbar_wait(&full[s], u & 1u) || !mbar_wait(&acc_empty[ab], (ua & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(ab * D);
#pragma unroll
        for (int p = 0; p < kPieces; ++p)
#pragma unroll
          for (int sl = 0; sl < S::kSlabs; ++sl)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint64_t ad = sw128_kmajor_desc(x_addr + s * S::kStageBytes + sl * S::kSlabBytesX + k4 * 32);
              const uint64_t bd = sw128_kmajor_desc(pi_addr + p * S::kPieceBytes + sl * S::kSlabBytesPi + k4 * 32);
              mma_f16(d_tmem, ad, bd, idesc, (p | sl | k4) != 0 ? 1u : 0u);
            }
        mma_commit(&empty[s]);
        mma_commit(&acc_full[ab]);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done_bar);  // arrives once everything issued above has completed
    }
  } else {
    // epilogue: set (warp - 2) / 4 takes tiles i = set (mod kSets) from its
    // accumulator buffer; warp % 4 selects the TMEM lane quarter
    const int set = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    constexpr int H = 1 << (BM - 1);
    const uint32_t lb = (uint32_t)(quarter * 32) << 16;
    int i = set;
    for (int64_t tile = blockIdx.x + (int64_t)set * gridDim.x; tile < ntiles; tile += (int64_t)kSets * gridDim.x,
                 i += kSets) {
      const int ab = set;
      const uint32_t ua = (uint32_t)(i / kSets);
      if (!mbar_wait_warp(&acc_full[ab], ua & 1u)) {
        atomicOr(a.status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t0 = tmem_base + lb + (uint32_t)(ab * D);
      // n = ||y|| from all of the vector's columns, two 32-column loads per wait
      float ss = 0.f;
#pragma unroll
      for (int g = 0; g < kGroups; g += 2) {
        float v[32], w[32];
        tmem_ld32(t0 + 32 * g, v);
        tmem_ld32(t0 + 32 * (g + 1), w);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) ss = fmaf(v[c], v[c], ss);
#pragma unroll
        for (int c = 0; c < 32; ++c) ss = fmaf(w[c], w[c], ss);
      }
      const float n = sqrtf(ss);
      // positive thresholds t_m (m = 1 .. H - 1) scaled by n, and the
      // constants of the FMA-pipe count; a zero vector has y = 0, which lies
      // below every positive threshold
      float P[8], Cz[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float tm = (m >= 1 && m < H) ? thr_s[H - 1 + m] : 0.f;
        P[m] = n > 0.f ? n * tm : INFINITY;
        Cz[m] = (n > 0.f && m >= 1 && m < H) ? 1.f - 4294967296.f * tm : -1.f;
      }
      const float Bf = n > 0.f ? 4294967296.f / n : 0.f;
      const int64_t vec = tile * kTileM + row;
      // two groups per iteration, loaded together (one wait): the even group
      // takes the ALU-pipe search, the odd one the FMA-pipe count, and the
      // loop is not unrolled further, so each cell path exists once in the code
      // (a fully unrolled loop outgrows the instruction cache at 4 bits)
#pragma unroll 1
      for (int g = 0; g < kGroups; g += 2) {
        float v[32], u[32];
        tmem_ld32(t0 + 32 * g, v);
        tmem_ld32(t0 + 32 * (g + 1), u);
        tmem_wait_ld();
        if (g + 2 == kGroups) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
        if (vec < a.N) {
          uint32_t w[BM];
          pack_group<BM>(v, P, w);
          store_words<BM>(a.codes + vec * a.out_stride * W + g * BM, w);
          if (BM >= 2) pack_group_fma<BM>(u, P, Bf, Cz, w);
          else pack_group<BM>(u, P, w);
          store_words<BM>(a.codes + vec * a.out_stride * W + (g + 1) * BM, w);
        }
      }
      if (vec < a.N) a.norms[vec * a.out_stride] = n;
    }
  }

  // teardown: the MMA thread's final commit tells when TMEM is no longer in use
  __syncthreads();
  if (warp == 1) {
    if (!mbar_wait(done_bar, 0) && lane == 0) atomicOr(a.status, kStatusTimeout);
    __syncwarp();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}


template <int D, int BM>
int launch_tc(const tq_ctx* h, const void* x, int64_t N, int64_t x_stride, uint32_t* codes, float* norms,
              int64_t out_stride, cudaStream_t stream) {
  using S = TcShape<D>;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return (int)cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)N};
  const cuuint64_t gstride[1] = {(cuuint64_t)x_stride * 2};
  const cuuint32_t box[2] = {64, kTileM};
  const cuuint32_t estride[2] = {1, 1};
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return (int)cudaErrorInvalidValue;
  auto kern = quant_mse_tc_kernel<D, BM>;
  if (int e = ensure_dyn_smem((const void*)kern, S::kSmemBytes)) return e;
  TcArgs a{h->dev.pi_tc, h->dev.thresholds, N, out_stride, codes, norms, h->dev.status};
  const int64_t ntiles = (N + kTileM - 1) / kTileM;
  const int grid = (int)(ntiles < h->sm_count ? ntiles : h->sm_count);
  kern<<<grid, threads_for<D>(), S::kSmemBytes, stream>>>(map, a);
  return (int)cudaGetLastError();
}

}  // namespace

bool quant_tc_supported(const tq_ctx* h, int dtype) {
  return h->dev.pi_tc != nullptr && dtype == TQ_BF16 && (h->d == 64 || h->d == 128) && h->variant == TQ_MSE;
}

int launch_quant_mse_tc(const tq_ctx* h, const void* x, int64_t N, int64_t x_stride, uint32_t* codes,
                        float* norms, int64_t out_stride, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  if (h->d == 128) {
    switch (h->bm) {
      case 1: return launch_tc<128, 1>(h, x, N, x_stride, codes, norms, out_stride, s);
      case 2: return launch_tc<128, 2>(h, x, N, x_stride, codes, norms, out_stride, s);
      case 3: return launch_tc<128, 3>(h, x, N, x_stride, codes, norms, out_stride, s);
      default: return launch_tc<128, 4>(h, x, N, x_stride, codes, norms, out_stride, s);
    }
  }
  switch (h->bm) {
    case 1: return launch_tc<64, 1>(h, x, N, x_stride, codes, norms, out_stride, s);
    case 2: return launch_tc<64, 2>(h, x, N, x_stride, codes, norms, out_stride, s);
    case 3: return launch_tc<64, 3>(h, x, N, x_stride, codes, norms, out_stride, s);
    default: return launch_tc<64, 4>(h, x, N, x_stride, codes, norms, out_stride, s);
  }
}

}  // namespace tqi
