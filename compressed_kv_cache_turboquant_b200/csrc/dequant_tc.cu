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
//          combines and scales by n, and writes its row's 128-byte chunk into
//          the warp's own shared-memory box (16-byte units XOR-swizzled by row,
//          so neither the writes nor the reads below meet in a bank); the warp
//          then reads the box back four rows per instruction and stores it
//          with 16-byte global stores, each instruction covering four whole
//          128-byte lines.  No store waits on an earlier one, so the warp moves
//          straight on to its next chunk.
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
  static constexpr int kMiscBytes = 1024;
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
  void* out;               // [N][D] of fp32 (or bf16 with out_bf16)
  int* status;
};

// 16 consecutive 32-bit TMEM columns of this warp's 32 lanes (lane = thread)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(taddr));
}

template <int D, int BM>
__global__ void __launch_bounds__(kThreads, 1) dequant_tc_kernel(DqArgs a) {
  using S = DqShape<D>;
  constexpr int W = (D / 32) * BM;
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
      if (tile < ntiles && vec < a.N) {
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
      if (!mbar_wait(&a_empty[s], (u & 1u) ^ 1u)) {
        atomicOr(a.status, kStatusTimeout);
        break;
      }
      uint8_t* hi_tile = a_s + s * 2 * S::kABytes;
      uint8_t* lo_tile = hi_tile + S::kABytes;
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
    const int row_bytes = a.out_bf16 ? 2 * D : 4 * D;   // one output row in global memory
    int i = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      const int s = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      const int64_t vec = tile * kTileM + r;
      const int64_t row0 = tile * kTileM + quarter * 32;
      const float n = (vec < a.N) ? a.norms[vec] : 0.f;  // issued before the wait
      if (!mbar_wait(&acc_full[s], u & 1u)) {
        atomicOr(a.status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(s * 2 * D);
      const int nchunks = a.out_bf16 ? D / 64 : D / 32;
      const int c_lo = part * (nchunks / 2), c_hi = (nchunks == 1) ? (part == 0 ? 1 : 0) : c_lo + nchunks / 2;
      for (int c = c_lo; c < c_hi; ++c) {
        // the row's 128 bytes in pieces of 16 TMEM columns; row `lane` of the
        // box: 16-byte unit j at lane * 128 + (j ^ (lane & 7)) * 16
        if (a.out_bf16) {
#pragma unroll
          for (int qt = 0; qt < 4; ++qt) {  // 16 columns -> 32 bytes = units 2 qt, 2 qt + 1
            float v0[16], v1[16];
            tmem_ld16(t0 + c * 64 + qt * 16, v0);
            tmem_ld16(t0 + D + c * 64 + qt * 16, v1);
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
            for (int jj = 0; jj < 2; ++jj) {
              const int j = 2 * qt + jj;
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                  make_uint4(pk[4 * jj], pk[4 * jj + 1], pk[4 * jj + 2], pk[4 * jj + 3]);
            }
          }
        } else {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {  // 16 columns -> 64 bytes = units 4 hf .. 4 hf + 3
            float v0[16], v1[16];
            tmem_ld16(t0 + c * 32 + hf * 16, v0);
            tmem_ld16(t0 + D + c * 32 + hf * 16, v1);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = __float_as_uint(n * fmaf(v1[e], 4.8828125e-4f, v0[e]));
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int j = 4 * hf + jj;
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                  make_uint4(pk[4 * jj], pk[4 * jj + 1], pk[4 * jj + 2], pk[4 * jj + 3]);
            }
          }
        }
        __syncwarp();
        // back out four rows per instruction: lane -> row 4 it + lane / 8, unit lane % 8
        uint8_t* gout = static_cast<uint8_t*>(a.out) + row0 * row_bytes + c * 128;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int rr = 4 * it + (lane >> 3), j = lane & 7;
          const uint4 v = *reinterpret_cast<const uint4*>(buf + rr * 128 + ((j ^ (rr & 7)) * 16));
          if (row0 + rr < a.N) *reinterpret_cast<uint4*>(gout + (int64_t)rr * row_bytes + j * 16) = v;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[s]);
    }
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
  auto kern = dequant_tc_kernel<D, BM>;
  if (int e = ensure_dyn_smem((const void*)kern, S::kSmemBytes)) return e;
  DqArgs a{codes, norms, N, h->dev.pit_f16, h->dev.lut_dq, out_bf16, out, h->dev.status};
  const int64_t ntiles = (N + kTileM - 1) / kTileM;
  const int grid = (int)(ntiles < h->sm_count ? ntiles : h->sm_count);
  kern<<<grid, kThreads, S::kSmemBytes, stream>>>(a);
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
