// TurboQuant_mse dequantization on the tensor cores (sm_100a):
// x_hat = n * Pi^T c[idx]  ([ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]:
// rebuild by rotating back and rescaling; turboquant.net/zh, "实现步骤草图", dequant 原语).
// (ttakun.com/news/45354, "KV缓存52GB瞬间爆内存？TurboQuant随机旋转+标量量化…")
//
// As a GEMM: X_hat[128 x d] = C[128 x d] . Pi (C = centroid values of a tile of
// 128 vectors).  fp16 operands in two pieces each, with the low pieces scaled
// by 2^11 so they stay normal:
//   C  = C_hi + 2^-11 C_lo',   Pi = P_hi + 2^-11 P_lo'
//   acc0 = C_hi . P_hi,  acc1 = C_hi . P_lo' + C_lo' . P_hi
//   x_hat = n * (acc0 + 2^-11 acc1)        (relative error ~2^-21)
// Persistent CTA per SM; warps:
//   0      TMEM allocation and the single-thread MMA issuer
//   1..4   decoders: one thread per vector unpacks its codes, looks the two
//          fp16 pieces up in a 16-entry table and writes them into the
//          128B-swizzled K-major A tiles (double-buffered)
//   5..12  epilogue, two warps per TMEM lane quarter taking half of the column
//          chunks each: one thread per vector reads both accumulators from TMEM,
//          combines and scales by n; each warp stages its 32 rows x 128 B
//          column chunk in 128B-swizzled shared memory (two buffers) and
//          writes it with one TMA tensor store, so global writes are whole
//          128-byte lines instead of 32 scattered 16-byte pieces per store
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;

constexpr int kTileM = 128;
constexpr int kThreads = 416;  // 13 warps

template <int D>
struct DqShape {
  static constexpr int kSlabs = D / 64;
  static constexpr int kSlabBytesA = kTileM * 128;
  static constexpr int kABytes = kSlabs * kSlabBytesA;  // one piece of one A tile
  static constexpr int kSlabBytesB = D * 128;
  static constexpr int kBBytes = kSlabs * kSlabBytesB;  // one piece of Pi (as B, K-major)
  static constexpr int kStages = 2;
  static constexpr int kTmemCols = (4 * D <= 256) ? 256 : 512;  // 2 buffers x 2 accumulators
  static constexpr int kMiscBytes = 2048;
  static constexpr int kStageOut = 32 * 128;  // one warp's output chunk: 32 rows x 128 B
  static constexpr int kOutBytes = 8 * kStageOut;  // one staging box per epilogue warp
  static constexpr int kSmemBytes = 2 * kBBytes + kStages * 2 * kABytes + kOutBytes + kMiscBytes + 1024;
};

struct DqArgs {
  const uint32_t* codes;
  const float* norms;
  int64_t N;
  const uint8_t* pit_f16;  // 2 pieces x [slab][row i][128 B swizzled] of Pi^T (B[i][j] = Pi[j][i])
  const uint32_t* lut;     // [16]: fp16 hi | fp16 lo' << 16 of c_k
  int out_bf16;
  int* status;
  // PolarQuant codes (BM = 0): words per row, bits of level 1 / levels >= 2,
  // first entry of each level among the codes of levels >= 2, and the cos /
  // sin of every level's centroids ([2][8 levels][16])
  int polar_w, b1, bh, w1;
  int base[9];
  const float* polar_cs;
};

// the polar code of entry e (level 1) or of entry e of the levels >= 2
__device__ __forceinline__ uint32_t polar_code(const uint32_t* w, int word0, int e, int bits) {
  const int pos = e * bits;
  return (w[word0 + (pos >> 5)] >> (pos & 31)) & ((1u << bits) - 1u);
}

template <int D, int BM>
__global__ void __launch_bounds__(kThreads, 1) dequant_tc_kernel(const __grid_constant__ CUtensorMap omap, DqArgs a) {
  using S = DqShape<D>;
  constexpr int W = BM ? (D / 32) * BM : 12;  // BM = 0: PolarQuant codes, at most 12 words
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* b_s = smem;                      // [2 pieces][kBBytes]
  uint8_t* a_s = smem + 2 * S::kBBytes;     // [stage][2 pieces][kABytes]
  uint8_t* o_s = a_s + S::kStages * 2 * S::kABytes;  // [8 warps][kStageOut], 1024-aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(o_s + S::kOutBytes);
  uint64_t* a_full = bars;              // [2]  decoders -> MMA (count 128)
  uint64_t* a_empty = bars + 2;         // [2]  MMA commit -> decoders
  uint64_t* acc_full = bars + 4;        // [2]  MMA commit -> epilogue
  uint64_t* acc_empty = bars + 6;       // [2]  epilogue (4 warps) -> MMA
  uint64_t* b_bar = bars + 8;
  uint64_t* done_bar = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  uint32_t* lut_s = tmem_slot + 4;      // [16]
  float* pcs = reinterpret_cast<float*>(lut_s + 16);  // [2][8][16] (PolarQuant)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (a.N + kTileM - 1) / kTileM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&a_full[s], 128);
      mbar_init(&a_empty[s], 1);
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 8);
    }
    mbar_init(b_bar, 1);
    mbar_init(done_bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 16) lut_s[threadIdx.x] = a.lut[threadIdx.x];
  if (BM == 0)
    for (int e = threadIdx.x; e < 256; e += blockDim.x) pcs[e] = a.polar_cs[e];
  if (warp == 0) tmem_alloc(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(b_bar, 2 * S::kBBytes);
      bulk_load(b_s, a.pit_f16, S::kBBytes, b_bar);
      bulk_load(b_s + S::kBBytes, a.pit_f16 + S::kBBytes, S::kBBytes, b_bar);
      constexpr uint32_t idesc = idesc_f16(kTileM, D, false);
      const uint32_t b_addr = smem_u32(b_s), a_addr = smem_u32(a_s);
      bool ok = mbar_wait(b_bar, 0);
      int i = 0;
      for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++i) {
        const int s = i & 1;
        const uint32_t u = (uint32_t)(i >> 1);
        if (!mbar_wait(&a_full[s], u & 1u) || !mbar_wait(&acc_empty[s], (u & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc0 = tmem_base + (uint32_t)(s * 2 * D), acc1 = acc0 + D;
        const uint32_t a_hi = a_addr + s * 2 * S::kABytes, a_lo = a_hi + S::kABytes;
        const uint32_t p_hi = b_addr, p_lo = b_addr + S::kBBytes;
#pragma unroll
        for (int sl = 0; sl < S::kSlabs; ++sl)
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint32_t ka = sl * S::kSlabBytesA + k4 * 32, kb = sl * S::kSlabBytesB + k4 * 32;
            const uint32_t first = (sl | k4) != 0 ? 1u : 0u;
            mma_f16(acc0, sw128_kmajor_desc(a_hi + ka), sw128_kmajor_desc(p_hi + kb), idesc, first);
            mma_f16(acc1, sw128_kmajor_desc(a_hi + ka), sw128_kmajor_desc(p_lo + kb), idesc, first);
            mma_f16(acc1, sw128_kmajor_desc(a_lo + ka), sw128_kmajor_desc(p_hi + kb), idesc, 1u);
          }
        mma_commit(&a_empty[s]);
        mma_commit(&acc_full[s]);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done_bar);
    }
  } else if (warp <= 4) {
    // decoders: thread r of the 128 decodes vector r of the tile; the codes of
    // the next tile are loaded while this one is decoded
    const int r = threadIdx.x - 32;
    auto load_codes = [&](int64_t tile, uint32_t (&w)[W]) {
      const int64_t vec = tile * kTileM + r;
      if (BM == 0) {
#pragma unroll
        for (int q = 0; q < W; ++q) w[q] = (tile < ntiles && vec < a.N && q < a.polar_w) ? a.codes[vec * a.polar_w + q] : 0u;
      } else if (tile < ntiles && vec < a.N) {
        if constexpr (W % 4 == 0) {
          const uint4* src = reinterpret_cast<const uint4*>(a.codes + vec * W);
#pragma unroll
          for (int q = 0; q < W / 4; ++q) {
            const uint4 t = src[q];
            w[4 * q] = t.x, w[4 * q + 1] = t.y, w[4 * q + 2] = t.z, w[4 * q + 3] = t.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < W; ++q) w[q] = a.codes[vec * W + q];
        }
      } else {
#pragma unroll
        for (int q = 0; q < W; ++q) w[q] = 0u;
      }
    };
    uint32_t w_next[W];
    load_codes(blockIdx.x, w_next);
    int i = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      const int s = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      uint32_t w[W];
#pragma unroll
      for (int q = 0; q < W; ++q) w[q] = w_next[q];
      load_codes(tile + gridDim.x, w_next);
      if (!mbar_wait_warp(&a_empty[s], (u & 1u) ^ 1u)) {
        atomicOr(a.status, kStatusTimeout);
        break;
      }
      uint8_t* hi_tile = a_s + s * 2 * S::kABytes;
      uint8_t* lo_tile = hi_tile + S::kABytes;
      if constexpr (BM == 0) {
        // the unit angle tree run back down: radii of the top levels, then one
        // 32-coordinate group at a time
        constexpr int G = D / 32;
        const float* cosl = pcs;
        const float* sinl = pcs + 128;
        float rg[G];
        if (D == 128) {
          const uint32_t c7 = polar_code(w, a.w1, a.base[7], a.bh);
          const float r6[2] = {cosl[7 * 16 + c7], sinl[7 * 16 + c7]};
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const uint32_t c6 = polar_code(w, a.w1, a.base[6] + i, a.bh);
            rg[2 * i] = r6[i] * cosl[6 * 16 + c6];
            rg[2 * i + 1] = r6[i] * sinl[6 * 16 + c6];
          }
        } else {
          const uint32_t c6 = polar_code(w, a.w1, a.base[6], a.bh);
          rg[0] = cosl[6 * 16 + c6];
          rg[1] = sinl[6 * 16 + c6];
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float rr[16];
          rr[0] = rg[g];
          // levels 5 .. 2 inside the group: 1, 2, 4, 8 angles
#pragma unroll
          for (int lev = 5, cnt = 1; lev >= 2; --lev, cnt <<= 1) {
#pragma unroll
            for (int i = cnt - 1; i >= 0; --i) {
              const uint32_t c = polar_code(w, a.w1, a.base[lev] + cnt * g + i, a.bh);
              const float r = rr[i];
              rr[2 * i] = r * cosl[lev * 16 + c];
              rr[2 * i + 1] = r * sinl[lev * 16 + c];
            }
          }
          float y[32];
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const uint32_t c = polar_code(w, 0, 16 * g + p, a.b1);
            y[2 * p] = rr[p] * cosl[16 + c];
            y[2 * p + 1] = rr[p] * sinl[16 + c];
          }
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int kglob = 32 * g + 8 * c4;
            const int slab = kglob / 64, chunk = (kglob % 64) / 8;
            uint32_t hv[4], lv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float v0 = y[8 * c4 + 2 * e], v1 = y[8 * c4 + 2 * e + 1];
              const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
              const __half l0 = __float2half_rn((v0 - __half2float(h0)) * 2048.f);
              const __half l1 = __float2half_rn((v1 - __half2float(h1)) * 2048.f);
              hv[e] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
              lv[e] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
            }
            const int off = slab * S::kSlabBytesA + r * 128 + ((chunk ^ (r & 7)) * 16);
            *reinterpret_cast<uint4*>(hi_tile + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
            *reinterpret_cast<uint4*>(lo_tile + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
          }
        }
      } else {
#pragma unroll
      for (int g = 0; g < D / 32; ++g) {
        uint32_t idx[32];
        const uint32_t* p = w + g * BM;
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) {
          if constexpr (BM == 1) idx[ii] = (p[0] >> ii) & 1u;
          else if constexpr (BM == 2) idx[ii] = (p[ii >> 4] >> (2 * (ii & 15))) & 3u;
          else if constexpr (BM == 4) idx[ii] = (p[ii >> 3] >> (4 * (ii & 7))) & 15u;
          else {
            if (ii < 24) idx[ii] = (p[ii >> 3] >> (4 * (ii & 7))) & 7u;
            else {
              const int sh = 4 * (ii - 24) + 3;
              idx[ii] = ((p[0] >> sh) & 1u) | (((p[1] >> sh) & 1u) << 1) | (((p[2] >> sh) & 1u) << 2);
            }
          }
        }
        // 4 chunks of 8 coordinates: k = 32 g + 8 c4 + e
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int kglob = 32 * g + 8 * c4;
          const int slab = kglob / 64, chunk = (kglob % 64) / 8;
          uint32_t hv[4], lv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t x0 = lut_s[idx[8 * c4 + 2 * e]], x1 = lut_s[idx[8 * c4 + 2 * e + 1]];
            hv[e] = __byte_perm(x0, x1, 0x5410);
            lv[e] = __byte_perm(x0, x1, 0x7632);
          }
          const int off = slab * S::kSlabBytesA + r * 128 + ((chunk ^ (r & 7)) * 16);
          *reinterpret_cast<uint4*>(hi_tile + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          *reinterpret_cast<uint4*>(lo_tile + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
        }
      }
      }
      // generic-proxy writes must be visible to the tensor core's async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&a_full[s]);
    }
  } else {
    // epilogue: warp % 4 selects the TMEM lane quarter, (warp - 5) / 4 the half of the chunks
    const int quarter = warp & 3;
    const int part = (warp - 5) >> 2;
    const int r = quarter * 32 + lane;
    uint8_t* buf = o_s + (warp - 5) * S::kStageOut;
    constexpr int kCols = 32;  // fp32 columns per 128-byte chunk (bf16: 64)
    int nst = 0;
    int i = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      const int s = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      const int64_t vec = tile * kTileM + r;
      const int64_t row0 = tile * kTileM + quarter * 32;
      const float n = (vec < a.N) ? a.norms[vec] : 0.f;  // issued before the wait
      if (!mbar_wait_warp(&acc_full[s], u & 1u)) {
        atomicOr(a.status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(s * 2 * D);
      const int nchunks = a.out_bf16 ? D / 64 : D / 32;
      const int c_lo = part * (nchunks / 2), c_hi = (nchunks == 1) ? (part == 0 ? 1 : 0) : c_lo + nchunks / 2;
      for (int c = c_lo; c < c_hi; ++c, ++nst) {
        // the previous store from this warp's buffer must have read it
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        // 16 columns of both accumulators at a time (a 32-column pair of
        // loads plus the packed row does not fit the register budget of 13
        // warps without spilling); each half fills four 16-byte units of the row
        if (a.out_bf16) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v0[16], v1[16];
            tmem_ld16(t0 + c * 64 + q * 16, v0);
            tmem_ld16(t0 + D + c * 64 + q * 16, v1);
            tmem_wait_ld();
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float y0 = n * fmaf(v1[2 * e], 4.8828125e-4f, v0[2 * e]);
              const float y1 = n * fmaf(v1[2 * e + 1], 4.8828125e-4f, v0[2 * e + 1]);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
              pk[e] = *reinterpret_cast<uint32_t*>(&b2);
            }
#pragma unroll
            for (int j = 2 * q; j < 2 * q + 2; ++j)
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                  make_uint4(pk[4 * (j - 2 * q)], pk[4 * (j - 2 * q) + 1], pk[4 * (j - 2 * q) + 2],
                             pk[4 * (j - 2 * q) + 3]);
          }
        } else {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float v0[16], v1[16];
            tmem_ld16(t0 + c * kCols + 16 * hh, v0);
            tmem_ld16(t0 + D + c * kCols + 16 * hh, v1);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = __float_as_uint(n * fmaf(v1[e], 4.8828125e-4f, v0[e]));
            // row `lane` of the 128B-swizzled box: 16-byte unit j lands at j ^ (lane & 7)
#pragma unroll
            for (int j = 4 * hh; j < 4 * hh + 4; ++j)
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                  make_uint4(pk[4 * (j - 4 * hh)], pk[4 * (j - 4 * hh) + 1], pk[4 * (j - 4 * hh) + 2],
                             pk[4 * (j - 4 * hh) + 3]);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < a.N) {
          tma_store_2d(&omap, buf, c * (a.out_bf16 ? 64 : kCols), (int)row0);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[s]);
    }
    if (lane == 0) bulk_wait_all();
  }

  __syncthreads();
  if (warp == 0) {
    if (!mbar_wait(done_bar, 0) && lane == 0) atomicOr(a.status, kStatusTimeout);
    __syncwarp();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

template <int D, int BM>
int launch_dq(const tq_ctx* h, const uint32_t* codes, const float* norms, int64_t N, void* out, int out_bf16,
              cudaStream_t stream) {
  using S = DqShape<D>;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return (int)cudaErrorNotSupported;
  // output as a [N][D] tensor, boxes of 32 rows x 128 bytes
  CUtensorMap omap;
  const int esz = out_bf16 ? 2 : 4;
  const cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)N};
  const cuuint64_t gstride[1] = {(cuuint64_t)D * esz};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / esz), 32};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&omap, out_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, gdim, gstride,
          box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return (int)cudaErrorInvalidValue;
  auto kern = dequant_tc_kernel<D, BM>;
  if (int e = ensure_dyn_smem((const void*)kern, S::kSmemBytes)) return e;
  DqArgs a{codes, norms, N, h->dev.pit_f16, h->dev.lut_dq, out_bf16, h->dev.status};
  if (BM == 0) {
    a.b1 = h->polar_b1;
    a.bh = h->polar_bh;
    a.polar_w = TQ_POLAR_WORDS(a.b1, a.bh, D);
    a.w1 = TQ_CODE_WORDS(a.b1, D / 2);
    a.base[2] = 0;
    for (int l = 2; l < 8; ++l) a.base[l + 1] = a.base[l] + (D >> l);
    a.polar_cs = h->polar_cs;
  }
  const int64_t ntiles = (N + kTileM - 1) / kTileM;
  const int grid = (int)(ntiles < h->sm_count ? ntiles : h->sm_count);
  kern<<<grid, kThreads, S::kSmemBytes, stream>>>(omap, a);
  return (int)cudaGetLastError();
}

}  // namespace

bool dequant_tc_supported(const tq_ctx* h) {
  return h->dev.pit_f16 != nullptr && (h->d == 64 || h->d == 128);
}

int launch_dequant_tc(const tq_ctx* h, const uint32_t* codes, const float* norms, int64_t N, void* out,
                      int out_dtype, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  const int bf = out_dtype == TQ_BF16;
  if (h->variant == TQ_POLAR)
    return h->d == 128 ? launch_dq<128, 0>(h, codes, norms, N, out, bf, s) : launch_dq<64, 0>(h, codes, norms, N, out, bf, s);
  if (h->d == 128) {
    switch (h->bm) {
      case 1: return launch_dq<128, 1>(h, codes, norms, N, out, bf, s);
      case 2: return launch_dq<128, 2>(h, codes, norms, N, out, bf, s);
      case 3: return launch_dq<128, 3>(h, codes, norms, N, out, bf, s);
      default: return launch_dq<128, 4>(h, codes, norms, N, out, bf, s);
    }
  }
  switch (h->bm) {
    case 1: return launch_dq<64, 1>(h, codes, norms, N, out, bf, s);
    case 2: return launch_dq<64, 2>(h, codes, norms, N, out, bf, s);
    case 3: return launch_dq<64, 3>(h, codes, norms, N, out, bf, s);
    default: return launch_dq<64, 4>(h, codes, norms, N, out, bf, s);
  }
}

}  // namespace tqi
