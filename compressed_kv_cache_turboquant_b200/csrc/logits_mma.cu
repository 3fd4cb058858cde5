// Full-context attention logits over a key cache split into two d = 64
// TurboQuant_prod channel groups, on the tensor cores with mma.sync (sm_100a).
//
// Pages: ttakun.com/news/45354 ("KV缓存52GB瞬间爆内存？…", 为什么TurboQuant…): 3.5 bits
// per channel with the high-variance channels at more bits; tmdm.cn ("谷歌悄悄扔下
// 一颗“性能核弹”…", 双剑合璧 / ✦ QJL): the QJL estimator inside attention.
//
// The logit of query head h and token t is scale * (est_A + est_B) with, per group,
//   est = n <q', c[idx]> + rn sqrt(pi/2)/64 <q'', sigma>.
// A block of 16 tokens of one warp is the M side of m16n8k16 MMAs whose N = 8
// columns are (group A, heads 0-3) and (group B, heads 0-3).  Lane (g, c) of the
// warp decodes, for tokens g and g + 8, coordinates 16c .. 16c + 15 of both
// groups: k-steps 0-3 carry group A, k-steps 4-7 group B, and the query
// fragment of a column is zero on the other group's k-steps, so one
// accumulator holds both groups' codebook dots and another their sign dots.
// Codes become fp16 through byte-indexed tables (one copy per lane), the
// codebook values scaled by the handle's alpha so they are nearly exact fp16
// numbers; the rotated queries enter as two fp16 pieces (hi + lo), the
// projected queries as one; norms and scales are applied in fp32.
//
// Persistent CTAs own equal contiguous ranges of 240-token blocks over all
// (batch, kv-head) pairs; warp 0 bulk-copies each block (codes, signs and the
// four norm arrays of both groups) into a ring; 15 consumer warps take 16
// tokens each and write the block's 4 x 240 logits.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>

#include "mma_frag.cuh"
#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;
using namespace frag;

constexpr int kCons = 15;     // consumer warps (with the producer, four per SM sub-partition)
constexpr int kBlk = 16 * kCons;  // tokens per stage, 16 per consumer warp
constexpr int kStages = 4;
constexpr int kThreads = 32 * (1 + kCons);
constexpr int kTabBytes = 256 * 256;
constexpr float kQjl64 = 1.2533141373155003f / 64.f;

template <int BM0, int BM1>
struct LgLayout {
  static constexpr int W0 = 2 * BM0, W1 = 2 * BM1;  // code words per token of each group
  static constexpr int C0 = 0;
  static constexpr int S0 = C0 + kBlk * W0 * 4;
  static constexpr int C1 = S0 + kBlk * 2 * 4;
  static constexpr int S1 = C1 + kBlk * W1 * 4;
  static constexpr int N0 = S1 + kBlk * 2 * 4;
  static constexpr int R0 = N0 + kBlk * 4;
  static constexpr int N1 = R0 + kBlk * 4;
  static constexpr int R1 = N1 + kBlk * 4;
  static constexpr int Stage = R1 + kBlk * 4;
  static constexpr int TokBytes = (W0 + 2 + W1 + 2 + 4) * 4;
  static constexpr int Smem = kStages * Stage + 2 * kTabBytes + kCons * 64 * 4 + 256 + 1024;
  static_assert(Stage % 16 == 0, "stage offsets stay 16-byte aligned");
};

struct LgArgs {
  const uint32_t* codes[2];
  const uint32_t* signs[2];
  const float* norms[2];
  const float* rnorms[2];
  const uint32_t* qfrag;  // [B*Hq][2 groups][3 pieces: q' hi, q' lo, q'' hi][64] fp16, coordinate order
  const float* qscale;    // [B*Hq][2 groups][2]: 1/s of the q' pieces and of q''
  uint32_t ctab[2][8];    // per group: fp16 alpha c[k] pairs (k = 2i in the low half)
  float inv_alpha[2];
  int B, Hq, Hkv;
  int64_t T, kv_stride;
  int64_t nblk, total;    // blocks per (batch, kv-head); all blocks
  float scale;
  float* logits;          // [B][Hq][T]
  int* status;
  uint32_t dyn_base;      // where the host measured the dynamic window to start
};

__host__ __device__ __forceinline__ int64_t lg_first_block(int64_t i, int64_t total, int64_t G) {
  return i * total / G;
}

__device__ __forceinline__ uint32_t ctab_half(const uint32_t (&t)[8], uint32_t k) {
  return (t[k >> 1] >> (16 * (k & 1u))) & 0xFFFFu;
}

// 16 coordinates (one half of a 32-coordinate group) of a key -> 8 fp16 pairs
// in coordinate order.  3-bit layout: half 0 is in the nibbles of w0, w1; half 1
// in w2 and in the spare fourth bits of w0..w2.  2-bit layout: half h is word h,
// byte i holding coordinates 4i .. 4i+3.
template <int BM, uint32_t ADDR>
__device__ __forceinline__ void decode_half(const uint32_t* w, int half, uint32_t tab, uint32_t off3,
                                            uint32_t off2, uint32_t (&h)[8]) {
  if constexpr (BM == 3) {
    const uint32_t s3 = ((w[0] >> 3) & 0x11111111u) | ((w[1] >> 2) & 0x22222222u) | ((w[2] >> 1) & 0x44444444u);
    const uint32_t wa = half ? w[2] : w[0];
    const uint32_t wb = half ? s3 : w[1];
    lookup4<ADDR>(wa, tab, off3, h);
    lookup4<ADDR>(wb, tab, off3, h + 4);
  } else {
    // one byte = four 2-bit codes = two fp16 pairs: one 8-byte lookup per byte
    const uint32_t x = half ? w[1] : w[0];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint2 v = tab_ld64<ADDR>(tab, prmt(x, off2, 0x5504 | (i << 4)));
      h[2 * i] = v.x, h[2 * i + 1] = v.y;
    }
  }
}

// 16 sign bits (bits 0..15 of w) -> 8 fp16 pairs of +-1
template <uint32_t ADDR>
__device__ __forceinline__ void decode_signs16(uint32_t w, uint32_t tab, uint32_t s_off, uint32_t (&h)[8]) {
  const uint4 v0 = tab_ld128<ADDR>(tab, prmt(w, s_off, 0x5504));
  const uint4 v1 = tab_ld128<ADDR>(tab, prmt(w, s_off, 0x5514));
  h[0] = v0.x, h[1] = v0.y, h[2] = v0.z, h[3] = v0.w;
  h[4] = v1.x, h[5] = v1.y, h[6] = v1.z, h[7] = v1.w;
}

// DB: shared address of the dynamic window (table addresses become load
// immediates), or kDynRuntime
template <int BM0, int BM1, uint32_t DB>
__global__ void __launch_bounds__(kThreads, 1) logits_mma_kernel(LgArgs a) {
  using L = LgLayout<BM0, BM1>;
  constexpr uint32_t KT = tab_addr(DB, kStages * L::Stage);
  constexpr uint32_t SG = tab_addr(DB, kStages * L::Stage + kTabBytes);
  extern __shared__ __align__(1024) uint8_t smem[];
  // the instance built for the host's measurement of the window start (DB ==
  // a.dyn_base) finds the window elsewhere: report, write nothing
  if (DB != kDynRuntime && (smem_u32(smem) != DB || a.dyn_base != DB)) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusLayout);
    return;
  }
  uint8_t* stages = smem;
  uint8_t* ktab = smem + kStages * L::Stage;   // row B: [3-bit pair, one copy per lane][2-bit pair pair, 16 copies]
  uint8_t* sgtab = ktab + kTabBytes;           // row B: 16 copies of the four +-1 pairs of B's bits
  float* obuf = reinterpret_cast<float*>(sgtab + kTabBytes);  // [kCons][4 heads][16 tokens]
  uint64_t* full = reinterpret_cast<uint64_t*>(obuf + kCons * 64);
  uint64_t* empty = full + kStages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t gb_lo = lg_first_block(blockIdx.x, a.total, G);
  const int64_t gb_hi = lg_first_block(blockIdx.x + 1, a.total, G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCons);
    }
    fence_mbar_init();
  }
  {
    // the 3-bit table comes from a group with 3 mse bits, the 2-bit one from a group with 2
    const int g3 = (BM0 == 3) ? 0 : 1, g2 = (BM0 == 2) ? 0 : 1;
    uint32_t* kt = reinterpret_cast<uint32_t*>(ktab);
    for (int w = threadIdx.x; w < kTabBytes / 4; w += blockDim.x) {
      const uint32_t row = (uint32_t)w >> 6, col = (uint32_t)w & 63u;
      uint32_t v;
      if (col < 32) {
        v = ctab_half(a.ctab[g3], row & 7u) | (ctab_half(a.ctab[g3], (row >> 4) & 7u) << 16);
      } else {
        // (c[b0], c[b1]) in the low word, (c[b2], c[b3]) in the high word of each 8-byte copy
        const uint32_t sh = (col & 1u) ? 4u : 0u;
        v = ctab_half(a.ctab[g2], (row >> sh) & 3u) | (ctab_half(a.ctab[g2], (row >> (sh + 2)) & 3u) << 16);
      }
      kt[w] = v;
    }
    uint32_t* sg = reinterpret_cast<uint32_t*>(sgtab);
    for (int w = threadIdx.x; w < kTabBytes / 4; w += blockDim.x) {
      const uint32_t row = (uint32_t)w >> 6, pair = (uint32_t)w & 3u;
      const uint32_t lo = ((row >> (2 * pair)) & 1u) ? 0x3C00u : 0xBC00u;
      const uint32_t hi = ((row >> (2 * pair + 1)) & 1u) ? 0x3C00u : 0xBC00u;
      sg[w] = lo | (hi << 16);
    }
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      BlockCursor cur;
      cur.init(gb_lo, a.nblk);
      for (int64_t gb = gb_lo, i = 0; gb < gb_hi; ++gb, ++i, cur.next(a.nblk)) {
        const int s = (int)(i % kStages);
        if (!mbar_wait(&empty[s], (uint32_t)(((i / kStages) & 1) ^ 1))) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        const int64_t bh = cur.bh;
        const int64_t t0 = cur.blk * kBlk;
        const int n = (int)min((int64_t)kBlk, a.T - t0);
        const int n4 = n & ~3;  // whole 16-byte units; the consumers read the tail from global memory
        uint8_t* st = stages + s * L::Stage;
        const int64_t r = bh * a.kv_stride + t0;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(n4 * L::TokBytes));
        if (n4) {
          bulk_load(st + L::C0, a.codes[0] + r * L::W0, n4 * L::W0 * 4, &full[s]);
          bulk_load(st + L::S0, a.signs[0] + r * 2, n4 * 8, &full[s]);
          bulk_load(st + L::C1, a.codes[1] + r * L::W1, n4 * L::W1 * 4, &full[s]);
          bulk_load(st + L::S1, a.signs[1] + r * 2, n4 * 8, &full[s]);
          bulk_load(st + L::N0, a.norms[0] + r, n4 * 4, &full[s]);
          bulk_load(st + L::R0, a.rnorms[0] + r, n4 * 4, &full[s]);
          bulk_load(st + L::N1, a.norms[1] + r, n4 * 4, &full[s]);
          bulk_load(st + L::R1, a.rnorms[1] + r, n4 * 4, &full[s]);
        }
      }
    }
  } else {
    const int cw = warp - 1;
    const int g = lane >> 2, c = lane & 3;
    // coordinates 16c .. 16c + 15 of each channel group: code group c >> 1, half c & 1; the
    // lane's accumulator columns 2c, 2c + 1 belong to channel group c >> 1 as well
    const int half = c & 1, grp_of_c = c >> 1;
    const uint32_t kt = smem_u32(ktab), sgt = smem_u32(sgtab);
    const uint32_t off3 = (uint32_t)lane * 4u, off2 = 128u + (uint32_t)(lane & 15) * 8u;
    const uint32_t s_off = (uint32_t)(lane & 15) * 16u;
    float* ob = obuf + cw * 64;
    uint32_t qh[8][2], ql[8][2], qq[8][2];
    float isq[2][2];  // [head j][0: q' pieces, 1: q''] for this lane's accumulator columns
    // byte offsets within a stage of this lane's words for tokens g and g + 8
    uint32_t o_c0[2], o_c1[2], o_s0[2], o_s1[2], o_n[2], o_r[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int tok = cw * 16 + g + 8 * r;
      o_c0[r] = L::C0 + (tok * L::W0 + grp_of_c * BM0) * 4;
      o_c1[r] = L::C1 + (tok * L::W1 + grp_of_c * BM1) * 4;
      o_s0[r] = L::S0 + (tok * 2 + grp_of_c) * 4;
      o_s1[r] = L::S1 + (tok * 2 + grp_of_c) * 4;
      o_n[r] = (grp_of_c ? L::N1 : L::N0) + tok * 4;
      o_r[r] = (grp_of_c ? L::R1 : L::R0) + tok * 4;
    }
    int64_t cur_bh = -1, q0 = 0;
    int stg = 0;
    uint32_t phase = 0u;
    bool ok = true;
    BlockCursor cur;
    cur.init(gb_lo, a.nblk);
    for (int64_t gb = gb_lo, i = 0; ok && gb < gb_hi; ++gb, ++i, cur.next(a.nblk)) {
      const int64_t bh = cur.bh;
      if (bh != cur_bh) {
        cur_bh = bh;
        const int64_t b = bh / a.Hkv, hh = bh - b * a.Hkv;
        q0 = b * a.Hq + hh * 4;  // first query head of the kv-head
        // B fragments: column g = (group g >> 2, head g & 3); k-steps 0-3 belong to group 0,
        // 4-7 to group 1; coordinates 16c + 4 (kb & 3) .. + 3 of the lane's range
        const int colgrp = g >> 2, colhead = g & 3;
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
          const int kg = kb >> 2;
          const uint32_t* qf = a.qfrag + ((q0 + colhead) * 2 + kg) * 3 * 32 + 8 * c + 2 * (kb & 3);
          const bool on = colgrp == kg;
          const uint2 vh = *reinterpret_cast<const uint2*>(qf);
          const uint2 vl = *reinterpret_cast<const uint2*>(qf + 32);
          const uint2 vq = *reinterpret_cast<const uint2*>(qf + 64);
          qh[kb][0] = on ? vh.x : 0u, qh[kb][1] = on ? vh.y : 0u;
          ql[kb][0] = on ? vl.x : 0u, ql[kb][1] = on ? vl.y : 0u;
          qq[kb][0] = on ? vq.x : 0u, qq[kb][1] = on ? vq.y : 0u;
        }
        // accumulator columns 2c, 2c+1: group c >> 1, heads 2 (c & 1) + j
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float* qs = a.qscale + ((q0 + 2 * half + j) * 2 + grp_of_c) * 2;
          isq[j][0] = qs[0];
          isq[j][1] = qs[1] * kQjl64;
        }
      }
      const int s = stg;
      const uint32_t ph = phase;
      if (++stg == kStages) stg = 0, phase ^= 1u;
      if (!mbar_wait_warp(&full[s], ph)) {
        ok = false;
        break;
      }
      const uint8_t* st = stages + s * L::Stage;
      const int64_t t0 = cur.blk * kBlk;
      const int n = (int)min((int64_t)kBlk, a.T - t0);
      const int n4 = n & ~3;
      const int tb = cw * 16;
      const int64_t row0 = bh * a.kv_stride + t0;
      // the words of this lane's code groups for tokens g and g + 8
      uint32_t w0[2][3], w1[2][3], sw0[2], sw1[2];
      float nn[2], rr[2];  // [token], of the lane's accumulator group
      if (n4 == kBlk) {
        // whole block in the stage (every block but a context's last): fixed per-lane offsets
        const uint32_t sb = smem_u32(st);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            w0[r][k] = k < BM0 ? lds32(sb + o_c0[r] + 4 * k) : 0u;
            w1[r][k] = k < BM1 ? lds32(sb + o_c1[r] + 4 * k) : 0u;
          }
          sw0[r] = lds32(sb + o_s0[r]);
          sw1[r] = lds32(sb + o_s1[r]);
          nn[r] = __uint_as_float(lds32(sb + o_n[r]));
          rr[r] = __uint_as_float(lds32(sb + o_r[r]));
        }
      } else
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int tok = tb + g + 8 * r;
        if (tok < n4) {
          const uint32_t* c0 = reinterpret_cast<const uint32_t*>(st + L::C0) + tok * L::W0 + grp_of_c * BM0;
          const uint32_t* c1 = reinterpret_cast<const uint32_t*>(st + L::C1) + tok * L::W1 + grp_of_c * BM1;
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            w0[r][k] = k < BM0 ? c0[k] : 0u;
            w1[r][k] = k < BM1 ? c1[k] : 0u;
          }
          sw0[r] = reinterpret_cast<const uint32_t*>(st + L::S0)[tok * 2 + grp_of_c];
          sw1[r] = reinterpret_cast<const uint32_t*>(st + L::S1)[tok * 2 + grp_of_c];
          nn[r] = reinterpret_cast<const float*>(st + (grp_of_c ? L::N1 : L::N0))[tok];
          rr[r] = reinterpret_cast<const float*>(st + (grp_of_c ? L::R1 : L::R0))[tok];
        } else if (tok < n) {
          const int64_t rw = row0 + tok;
          const uint32_t* c0 = a.codes[0] + rw * L::W0 + grp_of_c * BM0;
          const uint32_t* c1 = a.codes[1] + rw * L::W1 + grp_of_c * BM1;
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            w0[r][k] = k < BM0 ? c0[k] : 0u;
            w1[r][k] = k < BM1 ? c1[k] : 0u;
          }
          sw0[r] = a.signs[0][rw * 2 + grp_of_c];
          sw1[r] = a.signs[1][rw * 2 + grp_of_c];
          nn[r] = (grp_of_c ? a.norms[1] : a.norms[0])[rw];
          rr[r] = (grp_of_c ? a.rnorms[1] : a.rnorms[0])[rw];
        } else {
#pragma unroll
          for (int k = 0; k < 3; ++k) w0[r][k] = w1[r][k] = 0u;
          sw0[r] = sw1[r] = 0u;
          nn[r] = rr[r] = 0.f;
        }
      }
      // codebook dots (k-steps 0-3 group 0, 4-7 group 1), q' as hi + lo
      float sm[4] = {0.f, 0.f, 0.f, 0.f}, sq[4] = {0.f, 0.f, 0.f, 0.f};
      {
        uint32_t ha[8], hb[8];
        decode_half<BM0, KT>(w0[0], half, kt, off3, off2, ha);
        decode_half<BM0, KT>(w0[1], half, kt, off3, off2, hb);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          mma16816(sm, ha[2 * kb], hb[2 * kb], ha[2 * kb + 1], hb[2 * kb + 1], qh[kb][0], qh[kb][1]);
          mma16816(sm, ha[2 * kb], hb[2 * kb], ha[2 * kb + 1], hb[2 * kb + 1], ql[kb][0], ql[kb][1]);
        }
        decode_half<BM1, KT>(w1[0], half, kt, off3, off2, ha);
        decode_half<BM1, KT>(w1[1], half, kt, off3, off2, hb);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          mma16816(sm, ha[2 * kb], hb[2 * kb], ha[2 * kb + 1], hb[2 * kb + 1], qh[4 + kb][0], qh[4 + kb][1]);
          mma16816(sm, ha[2 * kb], hb[2 * kb], ha[2 * kb + 1], hb[2 * kb + 1], ql[4 + kb][0], ql[4 + kb][1]);
        }
        // sign dots: bits 16 half .. 16 half + 15 of the group's sign word
        decode_signs16<SG>(sw0[0] >> (16 * half), sgt, s_off, ha);
        decode_signs16<SG>(sw0[1] >> (16 * half), sgt, s_off, hb);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
          mma16816(sq, ha[2 * kb], hb[2 * kb], ha[2 * kb + 1], hb[2 * kb + 1], qq[kb][0], qq[kb][1]);
        decode_signs16<SG>(sw1[0] >> (16 * half), sgt, s_off, ha);
        decode_signs16<SG>(sw1[1] >> (16 * half), sgt, s_off, hb);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
          mma16816(sq, ha[2 * kb], hb[2 * kb], ha[2 * kb + 1], hb[2 * kb + 1], qq[4 + kb][0], qq[4 + kb][1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // the stage is no longer read
      // est of this lane's group for tokens (g, g+8) x heads (2 half + j); add the other group's (lane c ^ 2)
      float est[4];
      const float ia = grp_of_c ? a.inv_alpha[1] : a.inv_alpha[0];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float nr = nn[r], rn = rr[r];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int e = 2 * r + j;
          est[e] = fmaf(nr * ia * isq[j][0], sm[e], rn * isq[j][1] * sq[e]);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) est[e] += __shfl_xor_sync(0xffffffffu, est[e], 2);
      if (c < 2) {
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int j = 0; j < 2; ++j) ob[(2 * half + j) * 16 + g + 8 * r] = est[2 * r + j] * a.scale;
      }
      __syncwarp();
      if (lane < 16) {
        const int hd = lane >> 2, qt = lane & 3;
        const int tok = tb + 4 * qt;
        float* dst = a.logits + (q0 + hd) * a.T + t0 + tok;
        const float4 v = *reinterpret_cast<const float4*>(ob + hd * 16 + 4 * qt);
        if (tok + 4 <= n && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
          *reinterpret_cast<float4*>(dst) = v;
        } else {
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (tok + k < n) dst[k] = vv[k];
        }
      }
      __syncwarp();
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  }
  __syncthreads();
}

// Query fragments: per query head and group, q' s as fp16 hi + lo and q'' s'' as
// fp16, each with its own power-of-two scale putting the largest entry in
// [2^13, 2^14); one warp per (query head, group).
__global__ void logits_qfrag_kernel(const float* qrot0, const float* qproj0, const float* qrot1, const float* qproj1,
                                    int64_t nq, __half* qfrag, float* qscale) {
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= nq * 2) return;
  const int64_t q = wid >> 1;
  const int grp = (int)(wid & 1);
  const float* qr = (grp ? qrot1 : qrot0) + q * 64;
  const float* qp = (grp ? qproj1 : qproj0) + q * 64;
  const float r0 = qr[lane], r1 = qr[lane + 32], p0 = qp[lane], p1 = qp[lane + 32];
  float mr = fmaxf(fabsf(r0), fabsf(r1)), mp = fmaxf(fabsf(p0), fabsf(p1));
  for (int o = 16; o > 0; o >>= 1) {
    mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
    mp = fmaxf(mp, __shfl_xor_sync(0xffffffffu, mp, o));
  }
  auto scale_of = [](float m) {
    if (!(m > 0.f)) return 1.f;
    int e;
    (void)frexpf(m, &e);
    return ldexpf(1.f, 14 - e);
  };
  const float sr = scale_of(mr), sp = scale_of(mp);
  __half* dst = qfrag + (q * 2 + grp) * 3 * 64;
  const float vr[2] = {r0 * sr, r1 * sr};  // exact: powers of two
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const __half hi = __float2half_rn(vr[k]);
    dst[lane + 32 * k] = hi;
    dst[64 + lane + 32 * k] = __float2half_rn(vr[k] - __half2float(hi));
  }
  dst[128 + lane] = __float2half_rn(p0 * sp);
  dst[128 + lane + 32] = __float2half_rn(p1 * sp);
  if (lane == 0) {
    qscale[(q * 2 + grp) * 2] = 1.f / sr;
    qscale[(q * 2 + grp) * 2 + 1] = 1.f / sp;
  }
}

}  // namespace

bool logits_mma_supported(const tq_ctx* const* hk, int ngroups, int64_t kv_stride) {
  if (ngroups != 2) return false;
  for (int g = 0; g < 2; ++g)
    if (hk[g]->d != 64 || hk[g]->bm < 2 || hk[g]->bm > 3) return false;
  // one table per bit width: two groups of the same width must share their codebook
  if (hk[0]->bm == hk[1]->bm)
    for (int k = 0; k < (1 << hk[0]->bm); ++k)
      if (hk[0]->sc_tab[k] != hk[1]->sc_tab[k]) return false;
  return (kv_stride % 4) == 0;
}

size_t logits_mma_workspace(int64_t nq) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  return al((size_t)nq * 2 * 3 * 64 * 2) + al((size_t)nq * 2 * 2 * 4);
}

int launch_logits_mma(const tq_ctx* const* hk, const float* const* qrot, const float* const* qproj, int B, int Hq,
                      int Hkv, int64_t T, int64_t kv_stride, const uint32_t* const* kcodes,
                      const uint32_t* const* ksigns, const float* const* knorms, const float* const* krnorms,
                      float scale, float* logits, void* workspace, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t nq = (int64_t)B * Hq;
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  __half* qf = static_cast<__half*>(workspace);
  float* qs = reinterpret_cast<float*>(static_cast<char*>(workspace) + al((size_t)nq * 2 * 3 * 64 * 2));
  {
    const int64_t threads = nq * 2 * 32;
    logits_qfrag_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(qrot[0], qproj[0], qrot[1], qproj[1], nq,
                                                                          qf, qs);
    int e = (int)cudaGetLastError();
    if (e) return e;
  }
  LgArgs a;
  for (int g = 0; g < 2; ++g) {
    a.codes[g] = kcodes[g];
    a.signs[g] = ksigns[g];
    a.norms[g] = knorms[g];
    a.rnorms[g] = krnorms[g];
    for (int k = 0; k < 8; ++k)
      a.ctab[g][k] = (uint32_t)hk[g]->sc_tab[2 * k] | ((uint32_t)hk[g]->sc_tab[2 * k + 1] << 16);
    a.inv_alpha[g] = hk[g]->sc_inv_alpha;
  }
  a.qfrag = reinterpret_cast<const uint32_t*>(qf);
  a.qscale = qs;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.T = T;
  a.kv_stride = kv_stride;
  a.nblk = (T + kBlk - 1) / kBlk;
  a.total = (int64_t)B * Hkv * a.nblk;
  a.scale = scale;
  a.logits = logits;
  a.status = hk[0]->dev.status;
  a.dyn_base = hk[0]->dyn_base;
  const int grid = (int)(a.total < hk[0]->sm_count ? a.total : hk[0]->sm_count);
  const bool fixed = hk[0]->dyn_base == kDynBaseSm100 || hk[0]->debug_fixed_tables;
  auto go = [&](auto kern, int smem) -> int {
    if (int e = ensure_dyn_smem((const void*)kern, smem)) return e;
    kern<<<grid, kThreads, smem, s>>>(a);
    return (int)cudaGetLastError();
  };
  const int b0 = hk[0]->bm, b1 = hk[1]->bm;
  constexpr uint32_t F = kDynBaseSm100, R = kDynRuntime;
  if (b0 == 3 && b1 == 2)
    return fixed ? go(logits_mma_kernel<3, 2, F>, LgLayout<3, 2>::Smem) : go(logits_mma_kernel<3, 2, R>, LgLayout<3, 2>::Smem);
  if (b0 == 2 && b1 == 3)
    return fixed ? go(logits_mma_kernel<2, 3, F>, LgLayout<2, 3>::Smem) : go(logits_mma_kernel<2, 3, R>, LgLayout<2, 3>::Smem);
  if (b0 == 3 && b1 == 3)
    return fixed ? go(logits_mma_kernel<3, 3, F>, LgLayout<3, 3>::Smem) : go(logits_mma_kernel<3, 3, R>, LgLayout<3, 3>::Smem);
  return fixed ? go(logits_mma_kernel<2, 2, F>, LgLayout<2, 2>::Smem) : go(logits_mma_kernel<2, 2, R>, LgLayout<2, 2>::Smem);
}

}  // namespace tqi
