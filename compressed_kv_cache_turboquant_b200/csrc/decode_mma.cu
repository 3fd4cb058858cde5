// Decode attention over a TurboQuant K/V cache, memory-bound path (sm_100a).
//
// turboquant.net/zh, "实现步骤草图", 集成到 attention: K and V are stored in
// TurboQuant form and QJL is used inside attention; tmdm.cn ("谷歌悄悄扔下一颗
// “性能核弹”…", 实测数据): attention logits computed directly over a 4-bit cache.
//
// Work split: one CTA per (batch, kv-head, context split).  The 4 query heads
// of the kv-head's group share every key and value read.
//   warp 0     producer: bulk copies of 64-token blocks (K codes, QJL signs,
//              V codes and the three norm arrays) into an 8-stage ring
//   warps 1-4  consumers, 16 tokens of every block each:
//     logits   mma.sync m16n8k16 (fp16 in, fp32 accumulate), keys as M, the
//              K dimension = 128 mse coordinates then 128 QJL coordinates,
//              N = 8 columns = 4 rotated queries (mse part) and 4 projected
//              queries (QJL part); est = n <q', c[idx]> + rn sqrt(pi/2)/d <q'', s>
//     softmax  online, per head, in base 2
//     values   mma.sync with M = 128 coordinates (rotated frame), K = 16 tokens,
//              N = 4 heads; the weights carry the value norms
//   the four warps' states merge in shared memory; partial (max, sum, acc[d])
//   per head goes to the workspace; the merge kernel combines the splits and
//   rotates back once.
// Decoding is register-only: 3-bit key indices and 4-bit value indices become
// fp16 through byte-permute lookups in 8-entry byte tables (the value
// codebook's symmetry c[15-i] = -c[i] keeps its table at 8 entries); QJL bits
// become +-1.0 with one shift and one logic op per pair.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>

#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int kBlk = 64;       // tokens per stage
constexpr int kStages = 8;
constexpr int kCons = 4;       // consumer warps
constexpr int kThreads = 32 * (1 + kCons);
constexpr int kKW = 12;        // K code words per token (3 bits x 128 / 32)
constexpr int kSW = 4;         // sign words
constexpr int kVW = 16;        // V code words (4 bits)
// stage layout (bytes)
constexpr int kOffK = 0;
constexpr int kOffS = kOffK + kBlk * kKW * 4;   // 3072
constexpr int kOffV = kOffS + kBlk * kSW * 4;   // 4096
constexpr int kOffN = kOffV + kBlk * kVW * 4;   // 8192
constexpr int kOffR = kOffN + kBlk * 4;
constexpr int kOffVN = kOffR + kBlk * 4;
constexpr int kStageBytes = kOffVN + kBlk * 4;  // 8960
constexpr float kLog2e = 1.4426950408889634f;

struct DecArgs {
  const uint32_t* kcodes;
  const uint32_t* ksigns;
  const float* knorms;
  const float* krnorms;
  const uint32_t* vcodes;
  const float* vnorms;
  const uint32_t* qfrag;   // [B*Hq][2][128] fp16 pairs: rotated (natural order), projected (QJL order)
  const float* qscale;     // [B*Hq][2]: 1/s for the two fp16 query copies
  const uint32_t* ktab;    // [4]: K centroid lo bytes c0..3, c4..7, hi bytes c0..3, c4..7
  const uint32_t* vtab;    // [4]: V magnitude table |c|[8..15], lo and hi bytes
  int B, Hq, Hkv;
  int64_t T, kv_stride;
  int64_t nblk;            // 64-token blocks per (batch, kv-head)
  int64_t total;           // B * Hkv * nblk
  int max_seg;             // partial slots per CTA
  float scale_log2;        // logit scale * log2(e)
  float qjl_coef;          // sqrt(pi/2) / d
  float* partials;         // [CTA][max_seg][4 heads][d + 2]: acc[d], m (natural log), l
  int* status;
};

// CTA i of G owns the global blocks [i*total/G, (i+1)*total/G); a global block
// gb is block gb % nblk of (batch, kv-head) gb / nblk
__host__ __device__ __forceinline__ int64_t cta_first_block(int64_t i, int64_t total, int64_t G) {
  return i * total / G;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) { return __byte_perm(a, b, s); }

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 8 coordinates whose 3-bit indices sit in the nibbles of `sel` (bit 3 clear)
// -> 4 fp16 pairs (coords 0-1, 2-3, 4-5, 6-7) from the 8-entry byte tables
__device__ __forceinline__ void lut8(uint32_t sel, uint32_t tl0, uint32_t tl1, uint32_t th0, uint32_t th1,
                                     uint32_t* out) {
  const uint32_t s1 = sel >> 16;
  const uint32_t la = prmt(tl0, tl1, sel), ha = prmt(th0, th1, sel);
  const uint32_t lb = prmt(tl0, tl1, s1), hb = prmt(th0, th1, s1);
  out[0] = prmt(la, ha, 0x5140);
  out[1] = prmt(la, ha, 0x7362);
  out[2] = prmt(lb, hb, 0x5140);
  out[3] = prmt(lb, hb, 0x7362);
}

// one 3-bit group of 32 coordinates (words w0..w2, layout of tq.h) -> 16 fp16 pairs in coordinate order
__device__ __forceinline__ void decode_k3(uint32_t w0, uint32_t w1, uint32_t w2, const uint32_t (&t)[4],
                                          uint32_t (&h)[16]) {
  const uint32_t s3 = ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
  lut8(w0 & 0x77777777u, t[0], t[1], t[2], t[3], h + 0);
  lut8(w1 & 0x77777777u, t[0], t[1], t[2], t[3], h + 4);
  lut8(w2 & 0x77777777u, t[0], t[1], t[2], t[3], h + 8);
  lut8(s3, t[0], t[1], t[2], t[3], h + 12);
}

// 8 coordinates of 4-bit value indices (one word) -> 4 fp16 pairs in coordinate order.
// c[i] = +T[i-8] for i >= 8, -T[7-i] for i < 8 (symmetric codebook), T = |c| of the upper half.
__device__ __forceinline__ void decode_v4(uint32_t w, const uint32_t (&t)[4], uint32_t* out) {
  const uint32_t neg = (~w >> 3) & 0x11111111u;        // 1 where the index is in the lower half
  const uint32_t mag = (w ^ (neg * 7u)) & 0x77777777u;  // magnitude index m
  const uint32_t sg = neg << 2;                         // selector 4 -> byte 0x80, 0 -> 0x00
  const uint32_t m1 = mag >> 16, g1 = sg >> 16;
  const uint32_t la = prmt(t[0], t[1], mag), ha = prmt(t[2], t[3], mag) ^ prmt(0u, 0x80u, sg);
  const uint32_t lb = prmt(t[0], t[1], m1), hb = prmt(t[2], t[3], m1) ^ prmt(0u, 0x80u, g1);
  out[0] = prmt(la, ha, 0x5140);
  out[1] = prmt(la, ha, 0x7362);
  out[2] = prmt(lb, hb, 0x5140);
  out[3] = prmt(lb, hb, 0x7362);
}

__global__ void __launch_bounds__(kThreads, 2) decode_mma_kernel(DecArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* pub = empty + kStages;                                        // consumers published their state
  __half* pbuf = reinterpret_cast<__half*>(pub + 2);                     // [kCons][4 heads][16 tokens]
  float* mrg = reinterpret_cast<float*>(pbuf + kCons * 64);               // [2][kCons][4][2 + D]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t gb_lo = cta_first_block(blockIdx.x, a.total, G);
  const int64_t gb_hi = cta_first_block(blockIdx.x + 1, a.total, G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCons);
    }
    mbar_init(pub, 32 * kCons);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      for (int64_t gb = gb_lo, i = 0; gb < gb_hi; ++gb, ++i) {
        const int s = (int)(i % kStages);
        const uint32_t u = (uint32_t)(i / kStages);
        if (!mbar_wait(&empty[s], (u & 1u) ^ 1u)) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        const int64_t bh = gb / a.nblk;
        const int64_t t0 = (gb % a.nblk) * kBlk;
        const int n = (int)min((int64_t)kBlk, a.T - t0);
        const int n4 = n & ~3;  // norms are copied in whole 16-byte units
        uint8_t* st = stages + s * kStageBytes;
        const int64_t r = bh * a.kv_stride + t0;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(n * (kKW + kSW + kVW) * 4 + 3 * n4 * 4));
        bulk_load(st + kOffK, a.kcodes + r * kKW, n * kKW * 4, &full[s]);
        bulk_load(st + kOffS, a.ksigns + r * kSW, n * kSW * 4, &full[s]);
        bulk_load(st + kOffV, a.vcodes + r * kVW, n * kVW * 4, &full[s]);
        if (n4) {
          bulk_load(st + kOffN, a.knorms + r, n4 * 4, &full[s]);
          bulk_load(st + kOffR, a.krnorms + r, n4 * 4, &full[s]);
          bulk_load(st + kOffVN, a.vnorms + r, n4 * 4, &full[s]);
        }
      }
    }
  } else {
    const int cw = warp - 1;           // consumer index
    const int ct = threadIdx.x - 32;   // consumer thread 0..127
    const int g = lane >> 2, c = lane & 3;
    const int cp = c & 1;              // heads 2cp, 2cp+1 handled by this lane
    const int group = a.Hq / a.Hkv;    // 4
    uint32_t kt[4], vt[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) kt[i] = a.ktab[i], vt[i] = a.vtab[i];
    uint32_t bm[8][2], bq[8][2];
    float inv_s1[2], inv_s2[2];
    float m_run[2], l_run[2];
    float acc[8][4];
    __half* pb = pbuf + cw * 64;
    int64_t cur_bh = -1;
    int seg = -1;
    bool ok = true;

    // publish this warp's state, combine the four warps, write one partial
    auto flush = [&](int sg, int64_t bhv) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 4);
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 8);
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 16);
      }
      float* mb = mrg + (sg & 1) * kCons * 4 * (2 + D);
      float* mw = mb + cw * 4 * (2 + D);
      if (c < 2) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float* mh = mw + (2 * c + j) * (2 + D);
          if (g == 0) mh[0] = m_run[j], mh[1] = l_run[j];
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            mh[2 + 16 * g + 2 * mt] = acc[mt][j];
            mh[2 + 16 * g + 2 * mt + 1] = acc[mt][2 + j];
          }
        }
      }
      mbar_arrive(pub);
      if (!mbar_wait(pub, (uint32_t)(sg & 1))) {
        ok = false;
        return;
      }
      float* dst = a.partials + ((int64_t)blockIdx.x * a.max_seg + sg) * 4 * (D + 2);
      for (int idx = ct; idx < 4 * (2 + D); idx += 32 * kCons) {
        const int hd = idx / (2 + D), k = idx % (2 + D);
        float M = -FLT_MAX;
#pragma unroll
        for (int w = 0; w < kCons; ++w) M = fmaxf(M, mb[(w * 4 + hd) * (2 + D)]);
        if (k == 0) {
          dst[hd * (D + 2) + D] = M / kLog2e;  // natural-log units for the merge
        } else {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kCons; ++w) {
            const float* mh = mb + (w * 4 + hd) * (2 + D);
            v += mh[k] * exp2f(mh[0] - M);
          }
          if (k == 1) dst[hd * (D + 2) + D + 1] = v;
          else dst[hd * (D + 2) + k - 2] = v;
        }
      }
      (void)bhv;
    };

    for (int64_t gb = gb_lo, i = 0; ok && gb < gb_hi; ++gb, ++i) {
      const int64_t bh = gb / a.nblk;
      if (bh != cur_bh) {
        if (seg >= 0) flush(seg, cur_bh);
        if (!ok) break;
        ++seg;
        cur_bh = bh;
        // queries of this (batch, kv-head): mse columns 0-3 (q' of head g), QJL columns 4-7 (q'' of head g-4)
        const int64_t b = bh / a.Hkv, hh = bh % a.Hkv;
        const int64_t q0 = b * a.Hq + hh * group;
        const uint32_t* qf = a.qfrag + (q0 + (g & 3)) * 2 * 64;
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
          const uint2 vm = *reinterpret_cast<const uint2*>(qf + 16 * c + 2 * kb);
          const uint2 vq = *reinterpret_cast<const uint2*>(qf + 64 + 16 * c + 2 * kb);
          bm[kb][0] = (g < 4) ? vm.x : 0u;
          bm[kb][1] = (g < 4) ? vm.y : 0u;
          bq[kb][0] = (g >= 4) ? vq.x : 0u;
          bq[kb][1] = (g >= 4) ? vq.y : 0u;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          inv_s1[j] = a.qscale[2 * (q0 + 2 * cp + j)];
          inv_s2[j] = a.qscale[2 * (q0 + 2 * cp + j) + 1];
          m_run[j] = -FLT_MAX;
          l_run[j] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
      }
      const int s = (int)(i % kStages);
      const uint32_t u = (uint32_t)(i / kStages);
      if (!mbar_wait(&full[s], u & 1u)) {
        ok = false;
        break;
      }
      const uint8_t* st = stages + s * kStageBytes;
      const int64_t t0 = (gb % a.nblk) * kBlk;
      const int n = (int)min((int64_t)kBlk, a.T - t0);
      const int n4 = n & ~3;
      const int64_t row0 = bh * a.kv_stride + t0;
      const int tb = cw * 16;  // this warp's 16 tokens within the block
      // ---------------- logits: keys g and g+8 of the sub-block
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      {
        uint32_t hk0[16], hk1[16], sg0, sg1;
        const uint32_t* kc0 = reinterpret_cast<const uint32_t*>(st + kOffK) + (tb + g) * kKW + 3 * c;
        const uint32_t* kc1 = kc0 + 8 * kKW;
        decode_k3(kc0[0], kc0[1], kc0[2], kt, hk0);
        decode_k3(kc1[0], kc1[1], kc1[2], kt, hk1);
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(st + kOffS);
        sg0 = sw[(tb + g) * kSW + c];
        sg1 = sw[(tb + g + 8) * kSW + c];
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) mma16816(sc, hk0[2 * kb], hk1[2 * kb], hk0[2 * kb + 1], hk1[2 * kb + 1],
                                                 bm[kb][0], bm[kb][1]);
        const uint32_t one = 0x3C003C00u;
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
          // sign pairs (coords m, m+16) for m = 2kb and 2kb+1; bit set -> +1.0
          const uint32_t a0 = (~(sg0 << (15 - 2 * kb)) & 0x80008000u) | one;
          const uint32_t a1 = (~(sg1 << (15 - 2 * kb)) & 0x80008000u) | one;
          const uint32_t a2 = (~(sg0 << (14 - 2 * kb)) & 0x80008000u) | one;
          const uint32_t a3 = (~(sg1 << (14 - 2 * kb)) & 0x80008000u) | one;
          mma16816(sc, a0, a1, a2, a3, bq[kb][0], bq[kb][1]);
        }
      }
      // exchange: lanes c and c^2 hold the mse and QJL dots of the same heads
      float ot[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) ot[e] = __shfl_xor_sync(0xffffffffu, sc[e], 2);
      const float* mse = (c < 2) ? sc : ot;
      const float* qjl = (c < 2) ? ot : sc;
      // norms of keys g and g+8 (tail tokens past the copied multiple of 4 come from global memory)
      float kn[2], kr[2], vn[2];
      bool valid[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int tok = tb + g + 8 * r;
        valid[r] = tok < n;
        if (tok < n4) {
          kn[r] = reinterpret_cast<const float*>(st + kOffN)[tok];
          kr[r] = reinterpret_cast<const float*>(st + kOffR)[tok];
          vn[r] = reinterpret_cast<const float*>(st + kOffVN)[tok];
        } else if (tok < n) {
          const int64_t gi = row0 + tok;
          kn[r] = a.knorms[gi];
          kr[r] = a.krnorms[gi];
          vn[r] = a.vnorms[gi];
        } else {
          kn[r] = kr[r] = vn[r] = 0.f;
        }
      }
      // logits (base 2): [token r][head j]
      float lg[2][2];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float est = kn[r] * mse[2 * r + j] * inv_s1[j] + kr[r] * a.qjl_coef * qjl[2 * r + j] * inv_s2[j];
          lg[r][j] = valid[r] ? est * a.scale_log2 : -FLT_MAX;
        }
      // online softmax per head over the 16 tokens
      float alpha[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float mx = fmaxf(lg[0][j], lg[1][j]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float mn = fmaxf(m_run[j], mx);
        alpha[j] = exp2f(m_run[j] - mn);
        m_run[j] = mn;
        const float p0 = valid[0] ? exp2f(lg[0][j] - mn) : 0.f;
        const float p1 = valid[1] ? exp2f(lg[1][j] - mn) : 0.f;
        l_run[j] = l_run[j] * alpha[j] + p0 + p1;
        // weights carry the value norms
        if (c < 2) {
          pb[(2 * cp + j) * 16 + g] = __float2half_rn(p0 * vn[0]);
          pb[(2 * cp + j) * 16 + g + 8] = __float2half_rn(p1 * vn[1]);
        }
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        acc[mt][0] *= alpha[0];
        acc[mt][1] *= alpha[1];
        acc[mt][2] *= alpha[0];
        acc[mt][3] *= alpha[1];
      }
      __syncwarp();
      uint32_t pw0 = 0u, pw1 = 0u;
      if (g < 4) {
        pw0 = *reinterpret_cast<const uint32_t*>(pb + g * 16 + 2 * c);
        pw1 = *reinterpret_cast<const uint32_t*>(pb + g * 16 + 2 * c + 8);
      }
      // ---------------- values: tokens 2c, 2c+1, 2c+8, 2c+9; coordinates 16g .. 16g+15
      {
        const uint32_t* vc = reinterpret_cast<const uint32_t*>(st + kOffV);
        uint32_t xa[8], xb[8], xc[8], xd[8];
        const uint2 wa = *reinterpret_cast<const uint2*>(vc + (tb + 2 * c) * kVW + 2 * g);
        const uint2 wb = *reinterpret_cast<const uint2*>(vc + (tb + 2 * c + 1) * kVW + 2 * g);
        const uint2 wc = *reinterpret_cast<const uint2*>(vc + (tb + 2 * c + 8) * kVW + 2 * g);
        const uint2 wd = *reinterpret_cast<const uint2*>(vc + (tb + 2 * c + 9) * kVW + 2 * g);
        decode_v4(wa.x, vt, xa);
        decode_v4(wa.y, vt, xa + 4);
        decode_v4(wb.x, vt, xb);
        decode_v4(wb.y, vt, xb + 4);
        decode_v4(wc.x, vt, xc);
        decode_v4(wc.y, vt, xc + 4);
        decode_v4(wd.x, vt, xd);
        decode_v4(wd.y, vt, xd + 4);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          // rows (coords 16g + 2mt, 16g + 2mt + 1), token pairs (2c, 2c+1) and (2c+8, 2c+9)
          const uint32_t a0 = prmt(xa[mt], xb[mt], 0x5410), a1 = prmt(xa[mt], xb[mt], 0x7632);
          const uint32_t a2 = prmt(xc[mt], xd[mt], 0x5410), a3 = prmt(xc[mt], xd[mt], 0x7632);
          mma16816(acc[mt], a0, a1, a2, a3, pw0, pw1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (ok && seg >= 0) flush(seg, cur_bh);
    if (!ok) atomicOr(a.status, kStatusTimeout);
  }
  __syncthreads();
}

// Combine the partials of every CTA that covered a (batch, kv-head) and rotate
// back once: out = Pi_V^T (sum_s acc_s e^(m_s - M)) / (sum_s l_s e^(m_s - M)).
// One CTA per (batch, q-head).
__global__ void __launch_bounds__(128) decode_merge_persistent_kernel(const float* partials, int64_t G, int max_seg,
                                                                      int64_t nblk, int64_t total, int Hq, int Hkv,
                                                                      const float* PiV, float* out) {
  __shared__ float orot[D];
  __shared__ float ML[2];
  __shared__ int64_t range[2];
  const int64_t bq = blockIdx.x;
  const int64_t b = bq / Hq, hq = bq % Hq;
  const int group = Hq / Hkv;
  const int64_t bh = b * Hkv + hq / group;
  const int hd = (int)(hq % group);
  const int64_t lo = bh * nblk, hi = lo + nblk;
  if (threadIdx.x == 0) {
    // first CTA whose block range meets [lo, hi)
    int64_t i = lo * G / total;
    while (i > 0 && cta_first_block(i, total, G) > lo) --i;
    while (i < G && cta_first_block(i + 1, total, G) <= lo) ++i;
    int64_t i1 = i;
    float M = -FLT_MAX;
    for (; i1 < G && cta_first_block(i1, total, G) < hi; ++i1) {
      const int64_t sg = bh - cta_first_block(i1, total, G) / nblk;
      M = fmaxf(M, partials[((i1 * max_seg + sg) * 4 + hd) * (D + 2) + D]);
    }
    float L = 0.f;
    for (int64_t k = i; k < i1; ++k) {
      const int64_t sg = bh - cta_first_block(k, total, G) / nblk;
      const float* p = partials + ((k * max_seg + sg) * 4 + hd) * (D + 2);
      L += p[D + 1] * __expf(p[D] - M);
    }
    range[0] = i;
    range[1] = i1;
    ML[0] = M;
    ML[1] = L;
  }
  __syncthreads();
  const float M = ML[0], invL = 1.f / ML[1];
  for (int j = threadIdx.x; j < D; j += blockDim.x) {
    float v = 0.f;
    for (int64_t k = range[0]; k < range[1]; ++k) {
      const int64_t sg = bh - cta_first_block(k, total, G) / nblk;
      const float* p = partials + ((k * max_seg + sg) * 4 + hd) * (D + 2);
      v += p[j] * __expf(p[D] - M);
    }
    orot[j] = v * invL;
  }
  __syncthreads();
  for (int i2 = threadIdx.x; i2 < D; i2 += blockDim.x) {
    float v = 0.f;
    for (int j = 0; j < D; ++j) v = fmaf(PiV[(int64_t)j * D + i2], orot[j], v);
    out[bq * D + i2] = v;
  }
}

}  // namespace

bool decode_mma_supported(const tq_ctx* hk, const tq_ctx* hv, int Hq, int Hkv, int64_t kv_stride) {
  return hk->d == 128 && hv->d == 128 && hk->bm == 3 && hv->bm == 4 && Hq == 4 * Hkv && (kv_stride % 4) == 0 &&
         hk->dev.ktab != nullptr && hv->dev.vtab != nullptr;
}

// grid of the persistent kernel (2 CTAs per SM) and the partial slots each CTA needs
int decode_mma_grid(int B, int Hkv, int64_t T, int sm_count) {
  const int64_t total = (int64_t)B * Hkv * ((T + kBlk - 1) / kBlk);
  const int64_t g = 2 * (int64_t)sm_count;
  return (int)(total < g ? total : g);
}

int decode_mma_max_seg(int B, int Hkv, int64_t T, int sm_count) {
  const int64_t nblk = (T + kBlk - 1) / kBlk;
  const int64_t total = (int64_t)B * Hkv * nblk;
  const int64_t G = decode_mma_grid(B, Hkv, T, sm_count);
  const int64_t per = (total + G - 1) / G;
  return (int)((per + nblk - 1) / nblk + 1);
}

int launch_decode_mma(const tq_ctx* hk, const tq_ctx* hv, const uint32_t* qfrag, const float* qscale, int B,
                      int Hq, int Hkv, int64_t T, int64_t kv_stride, const uint32_t* kcodes,
                      const uint32_t* ksigns, const float* knorms, const float* krnorms, const uint32_t* vcodes,
                      const float* vnorms, float scale, float* partials, float* out, void* stream) {
  DecArgs a;
  a.kcodes = kcodes;
  a.ksigns = ksigns;
  a.knorms = knorms;
  a.krnorms = krnorms;
  a.vcodes = vcodes;
  a.vnorms = vnorms;
  a.qfrag = qfrag;
  a.qscale = qscale;
  a.ktab = hk->dev.ktab;
  a.vtab = hv->dev.vtab;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.T = T;
  a.kv_stride = kv_stride;
  a.nblk = (T + kBlk - 1) / kBlk;
  a.total = (int64_t)B * Hkv * a.nblk;
  a.max_seg = decode_mma_max_seg(B, Hkv, T, hk->sm_count);
  a.scale_log2 = scale * kLog2e;
  a.qjl_coef = 1.2533141373155003f / 128.0f;
  a.partials = partials;
  a.status = hk->dev.status;
  const int G = decode_mma_grid(B, Hkv, T, hk->sm_count);
  const int smem = kStages * kStageBytes + (2 * kStages + 2) * 8 + kCons * 64 * 2 + 2 * kCons * 4 * (2 + D) * 4;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    attr = true;
  }
  cudaStream_t s = (cudaStream_t)stream;
  decode_mma_kernel<<<G, kThreads, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  decode_merge_persistent_kernel<<<B * Hq, 128, 0, s>>>(partials, G, a.max_seg, a.nblk, a.total, Hq, Hkv,
                                                        hv->dev.Pi, out);
  return (int)cudaGetLastError();
}

}  // namespace tqi

namespace tqi {
namespace {

// Rotated / projected queries (fp32, from query_prep) -> scaled fp16 MMA B
// operands.  Per query: s = 2^(14 - ceil(log2 max|v|)) so the largest entry
// lands in (2^13, 2^14]; 1/s is kept to undo it.  The rotated copy stays in
// coordinate order; the projected copy is permuted within each group of 32 so
// that position 4kb + e holds coordinate 2kb, 2kb+16, 2kb+1, 2kb+17 (e = 0..3),
// the order in which the decode kernel pairs QJL sign bits.
__global__ void qfrag_kernel(const float* qrot, const float* qproj, int64_t nq, __half* qfrag, float* qscale) {
  const int64_t qi = blockIdx.x;
  if (qi >= nq) return;
  __shared__ float red[2][4];
  const int t = threadIdx.x;  // 128 threads, one coordinate each
  for (int which = 0; which < 2; ++which) {
    const float* src = (which ? qproj : qrot) + qi * D;
    float m = fabsf(src[t]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & 31) == 0) red[which][t >> 5] = m;
    __syncthreads();
    const float mx = fmaxf(fmaxf(red[which][0], red[which][1]), fmaxf(red[which][2], red[which][3]));
    int e = 0;
    if (mx > 0.f) (void)frexpf(mx, &e);  // mx in [2^(e-1), 2^e)
    const float s = (mx > 0.f) ? ldexpf(1.f, 14 - e) : 1.f;
    int coord = t;
    if (which) {
      const int grp = t >> 5, pp = t & 31, kb = pp >> 2, el = pp & 3;
      const int off = (el == 0) ? 2 * kb : (el == 1) ? 2 * kb + 16 : (el == 2) ? 2 * kb + 1 : 2 * kb + 17;
      coord = 32 * grp + off;
    }
    qfrag[qi * 2 * D + which * D + t] = __float2half_rn(src[coord] * s);
    if (t == 0) qscale[2 * qi + which] = 1.f / s;
    __syncthreads();
  }
}

}  // namespace

int launch_qfrag(const float* qrot, const float* qproj, int64_t nq, void* qfrag, float* qscale, void* stream) {
  qfrag_kernel<<<(unsigned)nq, 128, 0, (cudaStream_t)stream>>>(qrot, qproj, nq, (__half*)qfrag, qscale);
  return (int)cudaGetLastError();
}

}  // namespace tqi
