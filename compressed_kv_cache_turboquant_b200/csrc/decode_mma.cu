// Decode attention over a TurboQuant K/V cache, memory-bound path (sm_100a).
//
// turboquant.net/zh, "实现步骤草图", 集成到 attention: K and V are stored in
// TurboQuant form and QJL is used inside attention; tmdm.cn ("谷歌悄悄扔下一颗
// “性能核弹”…", 实测数据): attention logits computed directly over a 4-bit cache.
//
// Work split: persistent CTAs own equal contiguous ranges of 192-token blocks
// over all (batch, kv-head) pairs; the 4 query heads of a kv-head's group share
// every key and value read.
//   warp 0      producer: bulk copies of each block (K codes, QJL signs, V codes
//               and the three norm arrays) into a 4-stage ring (three blocks in
//               flight while the consumers work on the fourth)
//   warps 1-12  consumers (three per SM sub-partition), 16 tokens of every block each:
//     logits   mma.sync m16n8k16 (fp16 in, fp32 accumulate), keys as M, the
//              K dimension = 128 mse coordinates then 128 QJL coordinates,
//              N = 8 columns = 4 rotated queries (mse part) and 4 projected
//              queries (QJL part); est = n <q', c[idx]> + rn sqrt(pi/2)/d <q'', s>
//     softmax  online, per head, in base 2
//     values   mma.sync with M = 128 coordinates (rotated frame), K = 16 tokens,
//              N = 4 heads; the weights carry the value norms
//   the consumer warps' states merge in shared memory when a CTA leaves a
//   (batch, kv-head); partial (max, sum, acc[d]) per head goes to the workspace;
//   the merge kernel combines the CTAs that covered it and rotates back once.
// Decoding: every byte of key or value codes holds two indices and is turned
// into an fp16 pair by one lookup in a 256-entry table in shared memory (one
// table replica per lane, so the 32 lookups of a warp never share a bank); QJL
// bits become +-1.0 with one shift and one logic op per pair.
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

constexpr int D = 128;
constexpr int kCons = 12;      // consumer warps (three per SM sub-partition)
constexpr int kBlk = 16 * kCons;  // tokens per stage (16 per consumer warp)
constexpr int kStages = 4;
constexpr int kThreads = 32 * (1 + kCons);
constexpr int kKW = 12;        // K code words per token (3 bits x 128 / 32)
constexpr int kSW = 4;         // sign words
constexpr int kVW = 16;        // V code words (4 bits)
// stage layout (bytes)
constexpr int kOffK = 0;
constexpr int kOffS = kOffK + kBlk * kKW * 4;
constexpr int kOffV = kOffS + kBlk * kSW * 4;
constexpr int kOffN = kOffV + kBlk * kVW * 4;
constexpr int kOffR = kOffN + kBlk * 4;
constexpr int kOffVN = kOffR + kBlk * 4;
constexpr int kStageBytes = kOffVN + kBlk * 4;  // 26880
static_assert(kStageBytes % 16 == 0 && kOffS % 16 == 0 && kOffV % 16 == 0 && kOffN % 16 == 0, "bulk-copy alignment");
// Decode tables in shared memory, 256 rows of 256 bytes each, indexed by one
// byte of codes (two indices, or eight sign bits):
//   KV table, row B: [K entry, one 4-byte copy per lane][V entry, one per lane]
//     K entry = fp16 pair (cK[B & 7], cK[(B >> 4) & 7])   (3-bit codes; bits 3, 7 ignored)
//     V entry = fp16 pair (cV[B & 15], cV[B >> 4])         (4-bit codes)
//   sign table, row B: 8 copies of 16 bytes = four fp16 pairs (s0,s1)..(s6,s7),
//     s_i = +1.0 if bit i of B is set, else -1.0
// With a copy per lane the 32-bit lookups of a warp never meet in a bank, and
// the address of a lookup is one byte permute: (code byte) << 8 | (lane
// offset).  A 16-byte load is served a quarter-warp at a time, so 8 copies of
// a sign row (one per lane of a quarter) are enough; its address is
// (sign byte) << 7 | (lane offset), a shift and a masked merge.
constexpr int kTabBytes = 256 * 256;
constexpr int kSgTabBytes = 256 * 128;
constexpr int kSmemBytes = kStages * kStageBytes + kTabBytes + kSgTabBytes + (2 * kStages + 2) * 8 + kCons * 64 * 2 +
                           kCons * 4 * (2 + D) * 4;
static_assert(kSmemBytes <= 227 * 1024, "shared memory of one CTA");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 4.0f;        // rescale only when a logit passes the running max by 2^4
constexpr float kPScale = 0.0625f;   // fp16 weights p * ||v|| / 16 stay below ||v||

struct DecArgs {
  const uint32_t* kcodes;
  const uint32_t* ksigns;
  const float* knorms;
  const float* krnorms;
  const uint32_t* vcodes;
  const float* vnorms;
  const uint32_t* qfrag;   // [B*Hq][2][128] fp16: rotated and projected queries, coordinate order
  const float* qscale;     // [B*Hq][2]: 1/s for the two fp16 query copies
  const uint32_t* klut;    // [16]: fp16 of the key codebook c0..c7 in the low halves
  const uint32_t* vlut;    // [16]: fp16 of the value codebook c0..c15 in the low halves
  int B, Hq, Hkv;
  int64_t T, kv_stride;
  int64_t nblk;            // token blocks per (batch, kv-head)
  int64_t total;           // B * Hkv * nblk
  int max_seg;             // partial slots per CTA
  float scale_log2;        // logit scale * log2(e)
  float qjl_coef;          // sqrt(pi/2) / d
  float* partials;         // [CTA][max_seg][4 heads][d + 2]: acc[d], m (natural log), l
  int* status;
  uint32_t dyn_base;       // where the host measured the dynamic window to start
  uint64_t wait_ns;        // limit of every pipeline wait
  int stall;               // diagnostic: consumers first wait on a barrier nothing completes
  // paged cache (page > 0): token t of (batch, kv-head) bh is row
  // block_table[bh * max_pages + t / page] * page + t % page of every array
  const int32_t* block_table;
  int max_pages, page;
  int rn16;                // residual norms stored as fp16
};

// cache row of token t of (batch, kv-head) bh
__device__ __forceinline__ int64_t cache_row(const DecArgs& a, int64_t bh, int64_t t) {
  if (a.page == 0) return bh * a.kv_stride + t;
  return (int64_t)a.block_table[bh * a.max_pages + t / a.page] * a.page + t % a.page;
}

__device__ __forceinline__ float rnorm_at(const DecArgs& a, int64_t row) {
  return a.rn16 ? __half2float(reinterpret_cast<const __half*>(a.krnorms)[row]) : a.krnorms[row];
}

// CTA i of G owns the global blocks [i*total/G, (i+1)*total/G); a global block
// gb is block gb % nblk of (batch, kv-head) gb / nblk
__host__ __device__ __forceinline__ int64_t cta_first_block(int64_t i, int64_t total, int64_t G) {
  return i * total / G;
}

// one 3-bit group of 32 coordinates (words w0..w2, layout of tq.h) -> 16 fp16 pairs in coordinate order
template <uint32_t ADDR>
__device__ __forceinline__ void decode_k3(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t tab, uint32_t lane_off,
                                          uint32_t (&h)[16]) {
  // coordinates 24..31 live in the fourth bit of every nibble of w0..w2
  const uint32_t s3 = ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
  lookup4<ADDR>(w0, tab, lane_off, h + 0);
  lookup4<ADDR>(w1, tab, lane_off, h + 4);
  lookup4<ADDR>(w2, tab, lane_off, h + 8);
  lookup4<ADDR>(s3, tab, lane_off, h + 12);
}

// 32 QJL sign bits -> 16 fp16 pairs (+-1.0) in coordinate order; `lane_off` =
// (lane & 7) * 16, the lane's copy within a 128-byte sign row
template <uint32_t ADDR>
__device__ __forceinline__ void decode_signs(uint32_t w, uint32_t tab, uint32_t lane_off, uint32_t (&h)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t row = (i == 0) ? (w << 7) : (w >> (8 * i - 7));  // byte i at bits 7..14
    const uint4 v = tab_ld128<ADDR>(tab, (row & 0x7F80u) | lane_off);
    h[4 * i + 0] = v.x, h[4 * i + 1] = v.y, h[4 * i + 2] = v.z, h[4 * i + 3] = v.w;
  }
}

// DB: shared address of the dynamic window (the tables' addresses become load
// immediates), or kDynRuntime (table addresses added at run time)
template <uint32_t DB>
__global__ void __launch_bounds__(kThreads, 1) decode_mma_kernel(DecArgs a) {
  constexpr uint32_t KV = tab_addr(DB, kStages * kStageBytes);
  constexpr uint32_t SG = tab_addr(DB, kStages * kStageBytes + kTabBytes);
  extern __shared__ __align__(1024) uint8_t smem[];
  // the instance built for the host's measurement of the window start (DB ==
  // a.dyn_base) finds the window elsewhere: report, write nothing
  if (DB != kDynRuntime && (smem_u32(smem) != DB || a.dyn_base != DB)) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusLayout);
    return;
  }
  uint8_t* stages = smem;
  uint8_t* kvtab = smem + kStages * kStageBytes;
  uint8_t* sgtab = kvtab + kTabBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sgtab + kSgTabBytes);
  uint64_t* empty = full + kStages;
  uint64_t* pub = empty + kStages;                                        // consumer sync at segment ends
  uint64_t* never = pub + 1;                                              // diagnostic: nothing arrives
  __half* pbuf = reinterpret_cast<__half*>(pub + 2);                     // [kCons][4 heads][16 tokens]
  float* mrg = reinterpret_cast<float*>(pbuf + kCons * 64);               // [kCons][4][2 + D]

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
    mbar_init(never, 1);
    fence_mbar_init();
  }
  // tables
  {
    uint32_t* kv = reinterpret_cast<uint32_t*>(kvtab);
    for (int w = threadIdx.x; w < kTabBytes / 4; w += blockDim.x) {
      const uint32_t row = (uint32_t)w >> 6, col = (uint32_t)w & 63u;
      kv[w] = (col < 32) ? ((a.klut[row & 7u] & 0xFFFFu) | (a.klut[(row >> 4) & 7u] << 16))
                         : ((a.vlut[row & 15u] & 0xFFFFu) | (a.vlut[row >> 4] << 16));
    }
    uint32_t* sg = reinterpret_cast<uint32_t*>(sgtab);
    for (int w = threadIdx.x; w < kSgTabBytes / 4; w += blockDim.x) {
      const uint32_t row = (uint32_t)w >> 5, pair = (uint32_t)w & 3u;
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
      int64_t issued = 0;
      for (int64_t gb = gb_lo, i = 0; gb < gb_hi; ++gb, ++i, cur.next(a.nblk)) {
        const int s = (int)(i % kStages);
        const uint32_t u = (uint32_t)(i / kStages);
        if (!mbar_wait_ns(&empty[s], (u & 1u) ^ 1u, a.wait_ns)) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        issued = i + 1;
        const int64_t bh = cur.bh;
        const int64_t t0 = cur.blk * kBlk;
        const int n = (int)min((int64_t)kBlk, a.T - t0);
        uint8_t* st = stages + s * kStageBytes;
        // The block's rows come in contiguous pieces: the whole block of a dense
        // cache, or its part in each page.  Norms move in whole 16-byte units
        // (4 fp32 or 8 fp16 rows); piece starts are multiples of 8 rows, so only
        // the block's last few rows can be left for the consumers to read
        // from global memory.
        const int rnu = a.rn16 ? 8 : 4;
        for (int pass = 0; pass < 2; ++pass) {
          uint32_t tx = 0;
          for (int off = 0; off < n;) {
            const int64_t t = t0 + off;
            const int len = a.page ? (int)min((int64_t)(n - off), (int64_t)(a.page - t % a.page)) : n;
            const int64_t r = cache_row(a, bh, t);
            const int l4 = len & ~3, lr = len & ~(rnu - 1);
            if (pass == 0) {
              tx += (uint32_t)(len * (kKW + kSW + kVW) * 4 + 2 * l4 * 4 + lr * (a.rn16 ? 2 : 4));
            } else {
              bulk_load(st + kOffK + off * kKW * 4, a.kcodes + r * kKW, len * kKW * 4, &full[s]);
              bulk_load(st + kOffS + off * kSW * 4, a.ksigns + r * kSW, len * kSW * 4, &full[s]);
              bulk_load(st + kOffV + off * kVW * 4, a.vcodes + r * kVW, len * kVW * 4, &full[s]);
              if (l4) {
                bulk_load(st + kOffN + off * 4, a.knorms + r, l4 * 4, &full[s]);
                bulk_load(st + kOffVN + off * 4, a.vnorms + r, l4 * 4, &full[s]);
              }
              if (lr) {
                const int esz = a.rn16 ? 2 : 4;
                bulk_load(st + kOffR + off * esz, reinterpret_cast<const uint8_t*>(a.krnorms) + r * esz, lr * esz,
                          &full[s]);
              }
            }
            off += len;
          }
          if (pass == 0) mbar_arrive_expect_tx(&full[s], tx);
        }
      }
      // Before the CTA may exit, every copy issued into its shared memory must
      // have landed, also when the consumers gave up early: wait (bounded) for
      // the last phase of each stage that received a block.
      for (int64_t i = issued - kStages > 0 ? issued - kStages : 0; i < issued; ++i) {
        if (!mbar_wait(&full[i % kStages], (uint32_t)((i / kStages) & 1))) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
      }
    }
  } else {
    const int cw = warp - 1;           // consumer index
    const int ct = threadIdx.x - 32;   // consumer thread 0..255
    const int g = lane >> 2, c = lane & 3;
    const int cp = c & 1;              // heads 2cp, 2cp+1 handled by this lane
    const int group = a.Hq / a.Hkv;    // 4
    const uint32_t kvt = smem_u32(kvtab), sgt = smem_u32(sgtab);
    const uint32_t k_off = (uint32_t)lane * 4u, v_off = 128u + (uint32_t)lane * 4u;
    const uint32_t s_off = (uint32_t)(lane & 7) * 16u;
    // Value MMA k index -> token: k and k ^ 1 trade places in the pairs that
    // lanes c = 2, 3 hold, so that at each value-code load half the lanes of
    // a half-warp read even tokens and half odd ones (64-byte rows: two bank
    // groups instead of one).  The weights are stored in the same order.
    const int vsw = c >> 1;
    const int pslot = g ^ ((g >> 2) & 1);  // position of tokens g, g + 8 among the k indices
    // this lane's byte offsets within a stage (tokens of warp cw start at 16 cw)
    const int tb = cw * 16;
    const uint32_t o_k = kOffK + (uint32_t)((tb + g) * kKW + 3 * c) * 4u;    // +0, +4, +8; key g + 8 at +8 kKW words
    const uint32_t o_s = kOffS + (uint32_t)((tb + g) * kSW + c) * 4u;        // key g + 8 at +8 kSW words
    const uint32_t o_va = kOffV + (uint32_t)((tb + 2 * c + vsw) * kVW + 2 * g) * 4u;      // +8 tokens: +8 kVW words
    const uint32_t o_vb = kOffV + (uint32_t)((tb + 2 * c + 1 - vsw) * kVW + 2 * g) * 4u;
    const uint32_t o_n = kOffN + (uint32_t)(tb + g) * 4u;                   // R and VN follow at +kBlk floats
    const uint32_t st0 = smem_u32(stages);
    int stg = 0;
    uint32_t phase = 0u;
    uint32_t bf[8][2];  // query B fragments: q' of head g (g < 4), q'' of head g - 4 (g >= 4)
    float inv_s1[2], inv_s2[2];
    float m_ref[2], l_run[2];
    float acc[8][4];
    __half* pb = pbuf + cw * 64;
    int seg = -1;
    bool ok = true;

    // publish this warp's state, combine the consumer warps, write one partial
    auto flush = [&](int sg) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 4);
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 8);
        l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], 16);
      }
      float* mw = mrg + cw * 4 * (2 + D);
      if (c < 2) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float* mh = mw + (2 * c + j) * (2 + D);
          if (g == 0) mh[0] = m_ref[j], mh[1] = l_run[j];
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            mh[2 + 16 * g + 2 * mt] = acc[mt][j];
            mh[2 + 16 * g + 2 * mt + 1] = acc[mt][2 + j];
          }
        }
      }
      mbar_arrive(pub);
      if (!mbar_wait_warp(pub, 0u, a.wait_ns)) {
        ok = false;
        return;
      }
      float* dst = a.partials + ((int64_t)blockIdx.x * a.max_seg + sg) * 4 * (D + 2);
      for (int idx = ct; idx < 4 * (2 + D); idx += 32 * kCons) {
        const int hd = idx / (2 + D), k = idx % (2 + D);
        float M = -FLT_MAX;
#pragma unroll
        for (int w = 0; w < kCons; ++w) M = fmaxf(M, mrg[(w * 4 + hd) * (2 + D)]);
        if (k == 0) {
          dst[hd * (D + 2) + D] = M / kLog2e;  // natural-log units for the merge
        } else {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kCons; ++w) {
            const float* mh = mrg + (w * 4 + hd) * (2 + D);
            v += mh[k] * exp2f(mh[0] - M);
          }
          if (k == 1) dst[hd * (D + 2) + D + 1] = v;
          else dst[hd * (D + 2) + k - 2] = v;
        }
      }
      // second phase: everyone has read the merge buffer before it is written again
      mbar_arrive(pub);
      if (!mbar_wait_warp(pub, 1u, a.wait_ns)) ok = false;
    };

    if (a.stall && !mbar_wait_warp(never, 0u, a.wait_ns)) ok = false;
    BlockCursor cur;
    cur.init(gb_lo, a.nblk);
    const int nblocks = (int)(gb_hi - gb_lo);
    for (int it = 0; ok && it < nblocks; ++it, cur.next(a.nblk)) {
      const int64_t bh = cur.bh;
      if (it == 0 || cur.blk == 0) {  // a new (batch, kv-head) segment
        if (seg >= 0) flush(seg);
        if (!ok) break;
        ++seg;
        // queries of this (batch, kv-head): columns 0-3 q' of the 4 heads, columns 4-7 q''; both MMA passes
        // take all 8 columns, the code pass is read from columns 0-3 and the sign pass from columns 4-7
        const int64_t b = bh / a.Hkv, hh = bh - b * a.Hkv;
        const int64_t q0 = b * a.Hq + hh * group;
        const uint32_t* qf = a.qfrag + (q0 + (g & 3)) * 2 * 64;
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
          const uint2 v = *reinterpret_cast<const uint2*>(qf + (g < 4 ? 0 : 64) + 16 * c + 2 * kb);
          bf[kb][0] = v.x;
          bf[kb][1] = v.y;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          inv_s1[j] = a.qscale[2 * (q0 + 2 * cp + j)];
          inv_s2[j] = a.qscale[2 * (q0 + 2 * cp + j) + 1] * a.qjl_coef;
          m_ref[j] = -FLT_MAX;
          l_run[j] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
      }
      const int s = stg;
      if (!mbar_wait_ns(&full[s], phase, a.wait_ns)) {
        ok = false;
        break;
      }
      if (++stg == kStages) stg = 0, phase ^= 1u;
      const uint8_t* st = stages + s * kStageBytes;
      const uint32_t sb = st0 + (uint32_t)(s * kStageBytes);
      const int64_t t0 = cur.blk * kBlk;
      const int n = (int)min((int64_t)kBlk, a.T - t0);
      // ---------------- logits: keys g and g+8 of the sub-block
      float sm[4] = {0.f, 0.f, 0.f, 0.f}, sq[4] = {0.f, 0.f, 0.f, 0.f};
      {
        uint32_t h0[16], h1[16];
        const uint32_t ka = sb + o_k, kb8 = ka + 8 * kKW * 4;
        decode_k3<KV>(lds32(ka), lds32(ka + 4), lds32(ka + 8), kvt, k_off, h0);
        decode_k3<KV>(lds32(kb8), lds32(kb8 + 4), lds32(kb8 + 8), kvt, k_off, h1);
#pragma unroll
        for (int kb = 0; kb < 8; ++kb)
          mma16816(sm, h0[2 * kb], h1[2 * kb], h0[2 * kb + 1], h1[2 * kb + 1], bf[kb][0], bf[kb][1]);
        decode_signs<SG>(lds32(sb + o_s), sgt, s_off, h0);
        decode_signs<SG>(lds32(sb + o_s + 8 * kSW * 4), sgt, s_off, h1);
#pragma unroll
        for (int kb = 0; kb < 8; ++kb)
          mma16816(sq, h0[2 * kb], h1[2 * kb], h0[2 * kb + 1], h1[2 * kb + 1], bf[kb][0], bf[kb][1]);
      }
      // lane c < 2 holds the code dots of heads 2c, 2c+1 (columns 2c, 2c+1 of sm), lane c + 2 their sign dots
      // (columns 4 + 2c, 5 + 2c of sq): each sends the half the other needs
      float ot[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) ot[e] = __shfl_xor_sync(0xffffffffu, (c < 2) ? sm[e] : sq[e], 2);
      const float* mse = (c < 2) ? sm : ot;
      const float* qjl = (c < 2) ? ot : sq;
      // norms of keys g and g+8; a partial last block reads its tail from global memory
      float kn[2], kr[2], vn[2];
      if (n == kBlk) {
        const uint32_t na = sb + o_n;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          kn[r] = __uint_as_float(lds32(na + 32 * r));
          vn[r] = __uint_as_float(lds32(na + (kOffVN - kOffN) + 32 * r));
        }
        if (a.rn16) {
          const __half* rh = reinterpret_cast<const __half*>(st + kOffR);
          kr[0] = __half2float(rh[tb + g]);
          kr[1] = __half2float(rh[tb + g + 8]);
        } else {
#pragma unroll
          for (int r = 0; r < 2; ++r) kr[r] = __uint_as_float(lds32(na + (kOffR - kOffN) + 32 * r));
        }
      } else {
        const int n4 = n & ~3, nr = a.rn16 ? (n & ~7) : n4;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int tok = tb + g + 8 * r;
          if (tok < n4) {
            kn[r] = reinterpret_cast<const float*>(st + kOffN)[tok];
            vn[r] = reinterpret_cast<const float*>(st + kOffVN)[tok];
          } else if (tok < n) {
            const int64_t row = cache_row(a, bh, t0 + tok);
            kn[r] = a.knorms[row];
            vn[r] = a.vnorms[row];
          } else {
            kn[r] = vn[r] = 0.f;
          }
          if (tok < nr)
            kr[r] = a.rn16 ? __half2float(reinterpret_cast<const __half*>(st + kOffR)[tok])
                           : reinterpret_cast<const float*>(st + kOffR)[tok];
          else
            kr[r] = tok < n ? rnorm_at(a, cache_row(a, bh, t0 + tok)) : 0.f;
        }
      }
      // logits in base 2: [token r][head j]; tokens past the context end are -inf
      float lg[2][2];
      bool grow = false;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const bool valid = (tb + g + 8 * r) < n;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float est = fmaf(kn[r] * inv_s1[j], mse[2 * r + j], kr[r] * inv_s2[j] * qjl[2 * r + j]);
          lg[r][j] = valid ? est * a.scale_log2 : -FLT_MAX;
          grow |= lg[r][j] > m_ref[j] + kLazy;
        }
      }
      // lazy rescale: the reference max moves only when some logit passes it by kLazy
      if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float mx = fmaxf(lg[0][j], lg[1][j]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float mn = fmaxf(m_ref[j], mx);
          const float alpha = exp2f(m_ref[j] - mn);
          m_ref[j] = mn;
          l_run[j] *= alpha;
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            acc[mt][j] *= alpha;
            acc[mt][2 + j] *= alpha;
          }
        }
      }
      const bool v0 = (tb + g) < n, v1 = (tb + g + 8) < n;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float p0 = v0 ? exp2f(lg[0][j] - m_ref[j]) : 0.f;
        const float p1 = v1 ? exp2f(lg[1][j] - m_ref[j]) : 0.f;
        l_run[j] += (p0 + p1) * kPScale;
        if (c < 2) {
          pb[(2 * cp + j) * 16 + pslot] = __float2half_rn(p0 * vn[0] * kPScale);
          pb[(2 * cp + j) * 16 + pslot + 8] = __float2half_rn(p1 * vn[1] * kPScale);
        }
      }
      __syncwarp();
      uint32_t pw0 = 0u, pw1 = 0u;
      if (g < 4) {
        pw0 = *reinterpret_cast<const uint32_t*>(pb + g * 16 + 2 * c);
        pw1 = *reinterpret_cast<const uint32_t*>(pb + g * 16 + 2 * c + 8);
      }
      // ---------------- values: k indices 2c, 2c+1, 2c+8, 2c+9 (tokens k ^ vsw); coordinates 16g .. 16g+15
      {
        uint32_t xa[8], xb[8], xc[8], xd[8];
        const uint2 wa = lds64(sb + o_va);
        const uint2 wb = lds64(sb + o_vb);
        const uint2 wc = lds64(sb + o_va + 8 * kVW * 4);
        const uint2 wd = lds64(sb + o_vb + 8 * kVW * 4);
        lookup4<KV>(wa.x, kvt, v_off, xa);
        lookup4<KV>(wa.y, kvt, v_off, xa + 4);
        lookup4<KV>(wb.x, kvt, v_off, xb);
        lookup4<KV>(wb.y, kvt, v_off, xb + 4);
        lookup4<KV>(wc.x, kvt, v_off, xc);
        lookup4<KV>(wc.y, kvt, v_off, xc + 4);
        lookup4<KV>(wd.x, kvt, v_off, xd);
        lookup4<KV>(wd.y, kvt, v_off, xd + 4);
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
    if (ok && seg >= 0) flush(seg);
    if (!ok) atomicOr(a.status, kStatusTimeout);
  }
  __syncthreads();
}

// Combine the partials of every CTA that covered a (batch, kv-head) and rotate
// back once: out = Pi_V^T (sum_s acc_s e^(m_s - M)) / (sum_s l_s e^(m_s - M)).
// One CTA per (batch, q-head).
__global__ void __launch_bounds__(128) decode_merge_persistent_kernel(const float* partials, int64_t G, int max_seg,
                                                                      int64_t nblk, int64_t total, int Hq, int Hkv,
                                                                      const float* PiV, float* out, int partial_out) {
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
    orot[j] = partial_out ? v : v * invL;
  }
  if (partial_out) {  // the merged record (acc, m, l) in the rotated frame, at true scale:
    // the kernel's sums carry the fp16 weight scaling kPScale, which cancels in
    // its own quotient but not against records of other slices
    float* o = out + bq * (D + 2);
    for (int j = threadIdx.x; j < D; j += blockDim.x) o[j] = orot[j] * (1.f / kPScale);
    if (threadIdx.x == 0) o[D] = M, o[D + 1] = ML[1] * (1.f / kPScale);
    return;
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
         hk->dev.lut_dq != nullptr && hv->dev.lut_dq != nullptr;
}

// grid of the persistent kernel (2 CTAs per SM) and the partial slots each CTA needs
int decode_mma_grid(int B, int Hkv, int64_t T, int sm_count) {
  const int64_t total = (int64_t)B * Hkv * ((T + kBlk - 1) / kBlk);
  const int64_t g = (int64_t)sm_count;  // one CTA per SM
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
                      const float* vnorms, float scale, float* partials, float* out, void* stream,
                      int partial_out, PagedCache pg) {
  DecArgs a;
  a.kcodes = kcodes;
  a.ksigns = ksigns;
  a.knorms = knorms;
  a.krnorms = krnorms;
  a.vcodes = vcodes;
  a.vnorms = vnorms;
  a.qfrag = qfrag;
  a.qscale = qscale;
  a.klut = hk->dev.lut_dq;
  a.vlut = hv->dev.lut_dq;
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
  a.dyn_base = hk->dyn_base;
  a.wait_ns = hk->debug_stall_ns ? hk->debug_stall_ns : kWaitLimitNs;
  a.stall = hk->debug_stall_ns ? 1 : 0;
  a.block_table = pg.block_table;
  a.max_pages = pg.max_pages;
  a.page = pg.page;
  a.rn16 = pg.rn16;
  const int G = decode_mma_grid(B, Hkv, T, hk->sm_count);
  const int smem = kSmemBytes;
  const bool fixed = hk->dyn_base == kDynBaseSm100 || hk->debug_fixed_tables;
  auto kern = fixed ? decode_mma_kernel<kDynBaseSm100> : decode_mma_kernel<kDynRuntime>;
  if (int e = ensure_dyn_smem((const void*)kern, smem)) return e;
  cudaStream_t s = (cudaStream_t)stream;
  kern<<<G, kThreads, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  return launch_decode_merge_records(partials, G, a.max_seg, a.nblk, a.total, B, Hq, Hkv, hv, out, partial_out, s);
}

int launch_decode_merge_records(const float* partials, int64_t G, int max_seg, int64_t nblk, int64_t total, int B,
                                int Hq, int Hkv, const tq_ctx* hv, float* out, int partial_out, void* stream) {
  decode_merge_persistent_kernel<<<B * Hq, 128, 0, (cudaStream_t)stream>>>(partials, G, max_seg, nblk, total, Hq,
                                                                           Hkv, hv->dev.Pi, out, partial_out);
  return (int)cudaGetLastError();
}

}  // namespace tqi

namespace tqi {
namespace {

// Rotated / projected queries (fp32, from query_prep) -> scaled fp16 MMA B
// operands, both in coordinate order.  Per query copy: s = 2^(14 - ceil(log2
// max|v|)) so the largest entry lands in (2^13, 2^14]; 1/s is kept to undo it.
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
    qfrag[qi * 2 * D + which * D + t] = __float2half_rn(src[t] * s);
    if (t == 0) qscale[2 * qi + which] = 1.f / s;
    __syncthreads();
  }
}

// Shared-memory address at which the dynamic window of a kernel without
// static shared memory starts (written by one thread into `out`).
__global__ void dyn_smem_base_kernel(uint32_t* out) {
  extern __shared__ __align__(16) uint8_t dsm[];
  if (threadIdx.x == 0) out[0] = sm100::smem_u32(dsm);
}

}  // namespace

int launch_qfrag(const float* qrot, const float* qproj, int64_t nq, void* qfrag, float* qscale, void* stream) {
  qfrag_kernel<<<(unsigned)nq, 128, 0, (cudaStream_t)stream>>>(qrot, qproj, nq, (__half*)qfrag, qscale);
  return (int)cudaGetLastError();
}

// One launch of a 32-thread kernel with 16 bytes of dynamic shared memory;
// `scratch` is 4 bytes of device memory.  Synchronous.  Returns a CUDA error
// code; on success *base holds the address.
int probe_dyn_smem_base(uint32_t* scratch, uint32_t* base) {
  dyn_smem_base_kernel<<<1, 32, 16>>>(scratch);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpy(base, scratch, 4, cudaMemcpyDeviceToHost);
  return (int)e;
}

}  // namespace tqi
