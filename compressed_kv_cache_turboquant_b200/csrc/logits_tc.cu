// Full-context attention logits over a key cache split into two d = 64
// TurboQuant_prod channel groups, on the tcgen05 tensor cores (sm_100a).
//
// Pages: ttakun.com/news/45354 ("KV缓存52GB瞬间爆内存？…", 为什么TurboQuant…): 3.5 bits
// per channel with the high-variance channels at more bits; tmdm.cn ("谷歌悄悄扔下
// 一颗“性能核弹”…", 双剑合璧 / ✦ QJL): the QJL estimator inside attention.
//
// The logit of query head h and token t is scale * (est_A + est_B) with, per group,
//   est = n <q', c[idx]> + rn sqrt(pi/2)/64 <q'', sigma>.
// Per 128-token block one product on the tensor cores:
//   S[128 tok x 32] = [C_A | Sg_A | C_B | Sg_B] . Bq^T     (K = 256)
// with the decoded keys as the A operand in tensor memory (lane = token): C =
// the group's centroids scaled by its alpha (nearly exact fp16 numbers), Sg =
// its QJL signs as +-1.  Bq rows 0-15 are q'_A, q''_A, q'_B, q''_B of the four
// heads (fp16, per-copy power-of-two scale), rows 16-31 their fp16 remainders;
// each row is zero outside its own quarter of K.
//
// Persistent CTAs own equal contiguous ranges of 128-token blocks over all
// (batch, kv-head) pairs.  Warps (320 threads, one CTA per SM):
//   0      producer: bulk copies of each block (codes, signs and the four norm
//          arrays of both groups) into a ring, and of the query tile when a
//          new (batch, kv-head) starts
//   1      TMEM allocation and the single-thread MMA issuer
//   2-5    decoders: thread = token = TMEM lane; code bytes through tables in
//          shared memory (3-bit: a pair of codes per byte, one 4-byte copy per
//          lane; 2-bit: four codes per byte, one 8-byte copy per half-warp
//          lane), QJL bits to +-1.0 with one shift and one logic op per pair
//   6-9    epilogue: thread = token; est of the 4 heads from the 32 columns,
//          stores of 4 x 128 consecutive logits per block
// Tensor memory: A stage s at 128 s, S[s] at 256 + 32 s.  Sign columns pair
// coordinates (32 w + c, 32 w + 16 + c); the q'' rows use the same pairing.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>

#include "mma_frag.cuh"
#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;
using frag::BlockCursor;

constexpr int kTok = 128;
constexpr int kStages = 6;
constexpr int kThreads = 320;
constexpr float kQjl64 = 1.2533141373155003f / 64.f;
constexpr int kQBytes = 4 * 32 * 128;       // query tile: 4 slabs x 32 rows x 128 B
constexpr int kTabBytes = 256 * 128;        // each code table
constexpr uint32_t kColA = 0, kColS = 256;

template <int BM0, int BM1>
struct LtLayout {
  static constexpr int W0 = 2 * BM0, W1 = 2 * BM1;  // code words per token of each group
  static constexpr int C0 = 0;
  static constexpr int S0 = C0 + kTok * W0 * 4;
  static constexpr int C1 = S0 + kTok * 2 * 4;
  static constexpr int S1 = C1 + kTok * W1 * 4;
  static constexpr int N0 = S1 + kTok * 2 * 4;
  static constexpr int R0 = N0 + kTok * 4;
  static constexpr int N1 = R0 + kTok * 4;
  static constexpr int R1 = N1 + kTok * 4;
  static constexpr int Stage = R1 + kTok * 4;
  static constexpr int CodeBytes = (W0 + 2 + W1 + 2) * 4;  // per token, codes and signs
  // shared layout (1024-aligned base)
  static constexpr int OffRing = 0;
  static constexpr int OffQ = (kStages * Stage + 1023) / 1024 * 1024;
  static constexpr int OffT3 = OffQ + 2 * kQBytes;
  static constexpr int OffT2 = OffT3 + kTabBytes;
  static constexpr int OffBar = OffT2 + kTabBytes;
  static constexpr int Smem = OffBar + 256 + 1024;
  static_assert(Stage % 16 == 0 && S0 % 16 == 0 && C1 % 16 == 0 && S1 % 16 == 0 && N0 % 16 == 0, "bulk copies");
  static_assert(Smem <= 227 * 1024, "shared memory of one CTA");
};

struct LtArgs {
  const uint32_t* codes[2];
  const uint32_t* signs[2];
  const float* norms[2];
  const float* rnorms[2];
  const uint8_t* qtiles;   // [B*Hkv][kQBytes]
  const float* qscale;     // [B*Hq][2 groups][2]: 1/s of q' and of q''
  uint32_t ctab[2][8];     // per group: fp16 alpha c[k] pairs (k = 2i in the low half)
  float inv_alpha[2];
  int B, Hq, Hkv;
  int64_t T, kv_stride;
  int64_t nblk, total;
  float scale;
  float* logits;           // [B][Hq][T]
  int* status;
};

constexpr uint32_t kIdesc = idesc_f16(128, 32, false);

__device__ __forceinline__ uint32_t ctab_half(const uint32_t (&t)[8], uint32_t k) {
  return (t[k >> 1] >> (16 * (k & 1u))) & 0xFFFFu;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// the 64 coordinates of one group of token t -> 32 fp16 pair columns
template <int BM>
__device__ __forceinline__ void decode_group(const uint32_t* w, uint32_t t3, uint32_t t2, uint32_t (&h)[32]) {
  if constexpr (BM == 3) {
    // per 32-coordinate half k: nibbles of w0, w1, w2 hold coordinates 0-23, the fourth bits 24-31
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t w0 = w[3 * k], w1 = w[3 * k + 1], w2 = w[3 * k + 2];
      const uint32_t s3 = ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
      const uint32_t src[4] = {w0, w1, w2, s3};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t x = src[q];
        h[16 * k + 4 * q + 0] = lds32(t3 + ((x << 7) & 0x7F80u));
        h[16 * k + 4 * q + 1] = lds32(t3 + ((x >> 1) & 0x7F80u));
        h[16 * k + 4 * q + 2] = lds32(t3 + ((x >> 9) & 0x7F80u));
        h[16 * k + 4 * q + 3] = lds32(t3 + ((x >> 17) & 0x7F80u));
      }
    }
  } else {
    // word q: coordinates 16 q .. 16 q + 15, byte b holding 16 q + 4 b .. + 3
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t x = w[q];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t by = b == 0 ? ((x << 7) & 0x7F80u) : ((x >> (8 * b - 7)) & 0x7F80u);
        const uint2 v = lds64(t2 + by);
        h[8 * q + 2 * b] = v.x;
        h[8 * q + 2 * b + 1] = v.y;
      }
    }
  }
}

template <int BM0, int BM1>
__global__ void __launch_bounds__(kThreads, 1) logits_tc_kernel(LtArgs a) {
  using L = LtLayout<BM0, BM1>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem + L::OffRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OffBar);
  uint64_t* full = bars;                 // [6] producer (tx)
  uint64_t* empty = bars + kStages;      // [6] 4 decoder + 4 epilogue warps
  uint64_t* aqk_full = empty + kStages;  // [2] 4 decoder warps
  uint64_t* qk_done = aqk_full + 2;      // [2] MMA commit
  uint64_t* s_full = qk_done + 2;        // [2] MMA commit
  uint64_t* s_free = s_full + 2;         // [2] 4 epilogue warps
  uint64_t* q_free = s_free + 2;         // [2] MMA commit after a (batch, kv-head)'s last product
  uint64_t* done = q_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t gb_lo = blockIdx.x * a.total / G;
  const int64_t gb_hi = (blockIdx.x + 1) * a.total / G;
  const int nb = (int)(gb_hi - gb_lo);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&aqk_full[s], 4);
      mbar_init(&qk_done[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
      mbar_init(&q_free[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  {
    // the 3-bit table comes from a group with 3 mse bits, the 2-bit one from a group with 2
    const int g3 = (BM0 == 3) ? 0 : 1, g2 = (BM0 == 2) ? 0 : 1;
    uint32_t* t3 = reinterpret_cast<uint32_t*>(smem + L::OffT3);
    uint32_t* t2 = reinterpret_cast<uint32_t*>(smem + L::OffT2);
    for (int w = threadIdx.x; w < kTabBytes / 4; w += blockDim.x) {
      const uint32_t row = (uint32_t)w >> 5;
      // 3-bit row: (c[B & 7], c[(B >> 4) & 7]) per lane
      t3[w] = ctab_half(a.ctab[g3], row & 7u) | (ctab_half(a.ctab[g3], (row >> 4) & 7u) << 16);
      // 2-bit row: 8-byte copies, (c[b0], c[b1]) in the low word, (c[b2], c[b3]) in the high word
      const uint32_t sh = (w & 1) ? 4u : 0u;
      t2[w] = ctab_half(a.ctab[g2], (row >> sh) & 3u) | (ctab_half(a.ctab[g2], (row >> (sh + 2)) & 3u) << 16);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      BlockCursor cur;
      cur.init(gb_lo, a.nblk);
      int issued = 0, seg = -1;
      for (int i = 0; i < nb; ++i, cur.next(a.nblk)) {
        const int r = i % kStages;
        if (!mbar_wait(&empty[r], (uint32_t)(((i / kStages) & 1) ^ 1))) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        const bool first = (i == 0 || cur.blk == 0);
        if (first) {
          ++seg;
          if (!mbar_wait(&q_free[seg & 1], (uint32_t)(((seg >> 1) & 1) ^ 1))) {
            atomicOr(a.status, kStatusTimeout);
            break;
          }
        }
        const int64_t t0 = cur.blk * kTok;
        const int n = (int)min((int64_t)kTok, a.T - t0);
        // whole groups of 4 tokens (every copy a multiple of 16 bytes); the
        // decoders and the epilogue read a tail of up to 3 tokens from global memory
        const int n4 = n & ~3;
        const int64_t row = cur.bh * a.kv_stride + t0;
        uint8_t* st = ring + r * L::Stage;
        mbar_arrive_expect_tx(&full[r], (uint32_t)(n4 * (L::CodeBytes + 16)) + (first ? (uint32_t)kQBytes : 0u));
        if (first) bulk_load(smem + L::OffQ + (seg & 1) * kQBytes, a.qtiles + cur.bh * kQBytes, kQBytes, &full[r]);
        if (n4) {
          bulk_load(st + L::C0, a.codes[0] + row * L::W0, n4 * L::W0 * 4, &full[r]);
          bulk_load(st + L::S0, a.signs[0] + row * 2, n4 * 8, &full[r]);
          bulk_load(st + L::C1, a.codes[1] + row * L::W1, n4 * L::W1 * 4, &full[r]);
          bulk_load(st + L::S1, a.signs[1] + row * 2, n4 * 8, &full[r]);
          bulk_load(st + L::N0, a.norms[0] + row, n4 * 4, &full[r]);
          bulk_load(st + L::R0, a.rnorms[0] + row, n4 * 4, &full[r]);
          bulk_load(st + L::N1, a.norms[1] + row, n4 * 4, &full[r]);
          bulk_load(st + L::R1, a.rnorms[1] + row, n4 * 4, &full[r]);
        }
        issued = i + 1;
      }
      for (int i = issued - kStages > 0 ? issued - kStages : 0; i < issued; ++i)
        if (!mbar_wait(&full[i % kStages], (uint32_t)((i / kStages) & 1))) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t qb = smem_u32(smem + L::OffQ);
      BlockCursor cur;
      cur.init(gb_lo, a.nblk);
      int seg = -1;
      bool ok = true;
      for (int i = 0; i < nb; ++i, cur.next(a.nblk)) {
        const int s = i & 1;
        const uint32_t u = (uint32_t)(i >> 1);
        if (i == 0 || cur.blk == 0) ++seg;
        if (!mbar_wait(&aqk_full[s], u & 1u) || !mbar_wait(&s_free[s], (u & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t q = qb + (uint32_t)((seg & 1) * kQBytes);
        const uint32_t acc = tmem + kColS + 32u * s, aa = tmem + kColA + 128u * s;
#pragma unroll
        for (int ks = 0; ks < 16; ++ks)
          mma_f16_ta(acc, aa + 8 * ks, sw128_kmajor_desc(q + (ks >> 2) * 4096 + (ks & 3) * 32), kIdesc,
                     ks ? 1u : 0u);
        mma_commit(&qk_done[s]);
        mma_commit(&s_full[s]);
        if (i + 1 == nb || cur.blk + 1 == a.nblk) mma_commit(&q_free[seg & 1]);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done);
    }
  } else if (warp < 6) {
    // ---------------- decoders: thread = token = TMEM lane
    const int quarter = warp & 3;
    const int t = quarter * 32 + lane;
    const uint32_t lb = (uint32_t)(quarter * 32) << 16;
    const uint32_t t3 = smem_u32(smem + L::OffT3) + (uint32_t)lane * 4u;
    const uint32_t t2 = smem_u32(smem + L::OffT2) + (uint32_t)(lane & 15) * 8u;
    BlockCursor cur;
    cur.init(gb_lo, a.nblk);
    bool ok = true;
    for (int i = 0; i < nb; ++i, cur.next(a.nblk)) {
      const int r = i % kStages, s = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      if (!mbar_wait_warp(&full[r], (uint32_t)((i / kStages) & 1)) || !mbar_wait_warp(&qk_done[s], (u & 1u) ^ 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint8_t* st = ring + r * L::Stage;
      const int64_t t0 = cur.blk * kTok;
      const int n = (int)min((int64_t)kTok, a.T - t0);
      const int n4 = n & ~3;
      uint32_t w0[L::W0], w1[L::W1], sg[4];
      if (t < n4) {
#pragma unroll
        for (int k = 0; k < L::W0; ++k) w0[k] = reinterpret_cast<const uint32_t*>(st + L::C0)[t * L::W0 + k];
#pragma unroll
        for (int k = 0; k < L::W1; ++k) w1[k] = reinterpret_cast<const uint32_t*>(st + L::C1)[t * L::W1 + k];
        const uint2 x0 = *reinterpret_cast<const uint2*>(st + L::S0 + t * 8);
        const uint2 x1 = *reinterpret_cast<const uint2*>(st + L::S1 + t * 8);
        sg[0] = x0.x, sg[1] = x0.y, sg[2] = x1.x, sg[3] = x1.y;
      } else if (t < n) {
        const int64_t row = cur.bh * a.kv_stride + t0 + t;
#pragma unroll
        for (int k = 0; k < L::W0; ++k) w0[k] = a.codes[0][row * L::W0 + k];
#pragma unroll
        for (int k = 0; k < L::W1; ++k) w1[k] = a.codes[1][row * L::W1 + k];
        sg[0] = a.signs[0][row * 2], sg[1] = a.signs[0][row * 2 + 1];
        sg[2] = a.signs[1][row * 2], sg[3] = a.signs[1][row * 2 + 1];
      } else {
#pragma unroll
        for (int k = 0; k < L::W0; ++k) w0[k] = 0u;
#pragma unroll
        for (int k = 0; k < L::W1; ++k) w1[k] = 0u;
        sg[0] = sg[1] = sg[2] = sg[3] = 0u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[r]);
      const uint32_t aa = tmem + lb + kColA + 128u * s;
      {
        uint32_t h[32];
        decode_group<BM0>(w0, t3, t2, h);
        tmem_st16(aa, *reinterpret_cast<const uint32_t(*)[16]>(h));
        tmem_st16(aa + 16, *reinterpret_cast<const uint32_t(*)[16]>(h + 16));
      }
      {
        uint32_t h[32];
        decode_group<BM1>(w1, t3, t2, h);
        tmem_st16(aa + 64, *reinterpret_cast<const uint32_t(*)[16]>(h));
        tmem_st16(aa + 80, *reinterpret_cast<const uint32_t(*)[16]>(h + 16));
      }
      // signs: group g word w (coordinates 32 w ..) -> columns 32 + 64 g + 16 w + c, pairing (c, c + 16)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t x = sg[k];
        uint32_t p[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) p[c] = 0xBC00BC00u ^ ((x << (15 - c)) & 0x80008000u);
        tmem_st16(aa + 32 + 64 * (k >> 1) + 16 * (k & 1), p);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aqk_full[s]);
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  } else {
    // ---------------- epilogue: thread = token
    const int quarter = warp & 3;
    const int t = quarter * 32 + lane;
    const uint32_t lb = (uint32_t)(quarter * 32) << 16;
    float c1[2][4], c2[2][4];  // [group][head]: alpha^-1 / s' and sqrt(pi/2)/64 / s''
    int64_t q0 = 0;
    BlockCursor cur;
    cur.init(gb_lo, a.nblk);
    bool ok = true;
    for (int i = 0; i < nb; ++i, cur.next(a.nblk)) {
      const int r = i % kStages, s = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      if (i == 0 || cur.blk == 0) {
        const int64_t b = cur.bh / a.Hkv, hh = cur.bh - b * a.Hkv;
        q0 = b * a.Hq + hh * 4;
#pragma unroll
        for (int g = 0; g < 2; ++g)
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float* qs = a.qscale + ((q0 + h) * 2 + g) * 2;
            c1[g][h] = qs[0] * a.inv_alpha[g] * a.scale;
            c2[g][h] = qs[1] * kQjl64 * a.scale;
          }
      }
      if (!mbar_wait_warp(&s_full[s], u & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[32];
      tmem_ld32(tmem + lb + kColS + 32u * s, sv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[s]);
      const int64_t t0 = cur.blk * kTok;
      const int n = (int)min((int64_t)kTok, a.T - t0);
      const int n4 = n & ~3;
      const uint8_t* st = ring + r * L::Stage;
      float nn[2] = {0.f, 0.f}, rr[2] = {0.f, 0.f};
      if (t < n) {
        if (t < n4) {
          nn[0] = reinterpret_cast<const float*>(st + L::N0)[t];
          rr[0] = reinterpret_cast<const float*>(st + L::R0)[t];
          nn[1] = reinterpret_cast<const float*>(st + L::N1)[t];
          rr[1] = reinterpret_cast<const float*>(st + L::R1)[t];
        } else {
          const int64_t row = cur.bh * a.kv_stride + t0 + t;
          nn[0] = a.norms[0][row];
          rr[0] = a.rnorms[0][row];
          nn[1] = a.norms[1][row];
          rr[1] = a.rnorms[1][row];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[r]);
      if (t < n) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float e = nn[0] * c1[0][h] * (sv[h] + sv[16 + h]);
          e = fmaf(rr[0] * c2[0][h], sv[4 + h] + sv[20 + h], e);
          e = fmaf(nn[1] * c1[1][h], sv[8 + h] + sv[24 + h], e);
          e = fmaf(rr[1] * c2[1][h], sv[12 + h] + sv[28 + h], e);
          a.logits[(q0 + h) * a.T + t0 + t] = e;
        }
      }
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  }
  __syncthreads();
  if (warp == 1) {
    if (!mbar_wait(done, 0) && lane == 0) atomicOr(a.status, kStatusTimeout);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The query tile of every (batch, kv-head), a [32 x 256] fp16 B operand in the
// 128B-swizzled K-major layout.  Row 4 p + h (p = 0: q'_A, 1: q''_A, 2: q'_B,
// 3: q''_B; h the head of the group) holds its copy, scaled by a power of two
// that puts the largest entry in (2^13, 2^14], on K = 64 p .. 64 p + 63 (q''
// coordinates paired as the sign columns), zeros elsewhere; row 16 + r holds
// the fp16 remainders of row r.  One 128-thread CTA per (batch, kv-head).
__global__ void __launch_bounds__(128) logits_tc_qtile_kernel(const float* qrot0, const float* qproj0,
                                                              const float* qrot1, const float* qproj1, int Hq,
                                                              int Hkv, uint8_t* qtiles, float* qscale) {
  __shared__ float v[4][4][64];   // [p][head][coordinate], scaled
  __shared__ float red[4][4][2];  // [p][head][half of the 64 coordinates]
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / Hkv, hh = bh % Hkv;
  const int64_t q0 = b * Hq + hh * 4;
  const int j = threadIdx.x, lane = j & 31;
  const float* src[4] = {qrot0, qproj0, qrot1, qproj1};
  // thread j: copies (p, h) of index 2 (j >> 6) .. + 1, coordinate j & 63
  for (int it = 0; it < 8; ++it) {
    const int pair = it * 2 + (j >> 6), p = pair >> 2, h = pair & 3, c = j & 63;
    const float x = src[p][(q0 + h) * 64 + c];
    float m = fabsf(x);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[p][h][(c >> 5)] = m;
    v[p][h][c] = x;
  }
  __syncthreads();
  __shared__ float sc[4][4];
  if (j < 16) {
    const int p = j >> 2, h = j & 3;
    const float mx = fmaxf(red[p][h][0], red[p][h][1]);
    int e = 0;
    if (mx > 0.f) (void)frexpf(mx, &e);
    const float s = mx > 0.f ? ldexpf(1.f, 14 - e) : 1.f;
    sc[p][h] = s;
    qscale[((q0 + h) * 2 + (p >> 1)) * 2 + (p & 1)] = 1.f / s;
  }
  __syncthreads();
  // thread j writes row j / 4, K elements 64 (j % 4) .. + 63 (eight 16-byte units)
  const int row = j >> 2, kq = (j & 3) * 64;
  const bool lo = row >= 16;
  const int r16 = row & 15, p = r16 >> 2, h = r16 & 3;
  uint8_t* tile = qtiles + bh * kQBytes;
  for (int uu = 0; uu < 8; ++uu) {
    const int k0 = kq + 8 * uu;
    uint32_t pk[4];
    for (int e = 0; e < 8; e += 2) {
      float x2[2];
      for (int f = 0; f < 2; ++f) {
        const int k = k0 + e + f;
        float x = 0.f;
        if ((k >> 6) == p) {
          const int kk = k & 63;
          const int c = (p & 1) ? 32 * (kk >> 5) + ((kk & 31) >> 1) + 16 * (kk & 1) : kk;
          x = v[p][h][c] * sc[p][h];
        }
        const __half hi = __float2half_rn(x);
        x2[f] = lo ? x - __half2float(hi) : x;
      }
      const __half2 hv = __floats2half2_rn(x2[0], x2[1]);
      pk[e >> 1] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    const int slab = k0 >> 6, unit = (k0 & 63) >> 3;
    *reinterpret_cast<uint4*>(tile + slab * 4096 + row * 128 + ((unit ^ (row & 7)) << 4)) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

}  // namespace

bool logits_tc_supported(const tq_ctx* const* hk, int ngroups, int64_t kv_stride) {
  return logits_mma_supported(hk, ngroups, kv_stride) && !hk[0]->debug_fixed_tables && hk[0]->tc_attn;
}

size_t logits_tc_workspace(int B, int Hkv) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  return al((size_t)B * Hkv * kQBytes) + al((size_t)B * Hkv * 4 * 2 * 2 * 4);
}

int launch_logits_tc(const tq_ctx* const* hk, const float* const* qrot, const float* const* qproj, int B, int Hq,
                     int Hkv, int64_t T, int64_t kv_stride, const uint32_t* const* kcodes,
                     const uint32_t* const* ksigns, const float* const* knorms, const float* const* krnorms,
                     float scale, float* logits, void* workspace, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  uint8_t* qt = static_cast<uint8_t*>(workspace);
  float* qs = reinterpret_cast<float*>(qt + al((size_t)B * Hkv * kQBytes));
  logits_tc_qtile_kernel<<<(unsigned)((int64_t)B * Hkv), 128, 0, s>>>(qrot[0], qproj[0], qrot[1], qproj[1], Hq, Hkv,
                                                                      qt, qs);
  if (cudaError_t e = cudaGetLastError()) return (int)e;
  LtArgs a;
  for (int g = 0; g < 2; ++g) {
    a.codes[g] = kcodes[g];
    a.signs[g] = ksigns[g];
    a.norms[g] = knorms[g];
    a.rnorms[g] = krnorms[g];
    for (int k = 0; k < 8; ++k)
      a.ctab[g][k] = (uint32_t)hk[g]->sc_tab[2 * k] | ((uint32_t)hk[g]->sc_tab[2 * k + 1] << 16);
    a.inv_alpha[g] = hk[g]->sc_inv_alpha;
  }
  a.qtiles = qt;
  a.qscale = qs;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.T = T;
  a.kv_stride = kv_stride;
  a.nblk = (T + kTok - 1) / kTok;
  a.total = (int64_t)B * Hkv * a.nblk;
  a.scale = scale;
  a.logits = logits;
  a.status = hk[0]->dev.status;
  const int grid = (int)(a.total < hk[0]->sm_count ? a.total : hk[0]->sm_count);
  auto go = [&](auto kern, int smem) -> int {
    if (int e = ensure_dyn_smem((const void*)kern, smem)) return e;
    kern<<<grid, kThreads, smem, s>>>(a);
    return (int)cudaGetLastError();
  };
  const int b0 = hk[0]->bm, b1 = hk[1]->bm;
  if (b0 == 3 && b1 == 2) return go(logits_tc_kernel<3, 2>, LtLayout<3, 2>::Smem);
  if (b0 == 2 && b1 == 3) return go(logits_tc_kernel<2, 3>, LtLayout<2, 3>::Smem);
  if (b0 == 3 && b1 == 3) return go(logits_tc_kernel<3, 3>, LtLayout<3, 3>::Smem);
  return go(logits_tc_kernel<2, 2>, LtLayout<2, 2>::Smem);
}

}  // namespace tqi
