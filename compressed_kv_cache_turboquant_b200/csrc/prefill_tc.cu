// Prefill (multi-query) attention over a TurboQuant K/V cache on the tensor
// cores (sm_100a).
//
// turboquant.net/zh, "实现步骤草图", 集成到 attention: K and V are stored in
// TurboQuant form and QJL is used inside attention; tmdm.cn ("谷歌悄悄扔下一颗
// “性能核弹”…", 实测数据): attention logits over a 4-bit cache.  A block of nq new
// tokens (already appended to the cache) attends causally: token i sits at
// position T - nq + i and sees keys t <= T - nq + i.
//
// With many queries per key the work is a pair of GEMMs per key tile, so every
// product runs on tcgen05 with the decoded cache as the shared-memory operand.
// The estimator's two terms share one accumulator:
//   S = Q' C^T + Q'' Sg^T
//     Q'  = s Pi_K q                     C  = n_k c[idx]        (fp16)
//     Q'' = s sqrt(pi/2)/d S_K q         Sg = rn_k sign(S_K r)  (fp16)
//   with s a power of two per query row (the larger of the two rows' maxima
//   placed at 2^13..2^14), so logit = scale S / s
//   O += P V^T-tile   P = 2^(log2e logit - m) (fp16, written back into tensor
//                     memory), V = n_v c_V[idx] (fp16) in the rotated value frame
// One CTA per (batch, kv-head, tile of 128 query rows, slice of the context);
// a query row is a (token, head of the kv-head's group) pair.  Q' and Q'' live
// in tensor memory as the A operands of the logit product, P overwrites the
// first half of its logit buffer as the A operand of the value product; the
// decoded key and value tiles are the B operands in shared memory.  Two logit
// buffers let the product of key tile i + 1 run while the softmax warps work
// on tile i.  Each CTA writes its rows' softmax records (acc in the rotated
// frame, m, l); the merge kernel combines the slices and applies Pi_V^T once.
//
// Warps (320 threads, one CTA per SM):
//   0      bulk copies of each 128-token tile of packed K codes, QJL signs,
//          V codes and the three norms into a three-stage ring
//   1      TMEM allocation and the single-thread MMA issuer
//   2-5    decoders: thread t decodes key t of tile i + 1 into the centroid and
//          sign tiles (centroids from register byte tables by byte permutes,
//          the norms multiplied in), then key t of tile i into its row of one
//          of two value tiles (an MN-major B operand, so each key's decoded row
//          is stored whole; byte-table lookups in a per-lane copy of the table)
//          once the value product of tile i - 2 is done with that tile
//   6-9    softmax: thread = query row (TMEM lane); a tile's logits are read
//          twice from tensor memory (the row max, 64 columns per wait; then
//          the weights, the next 32 columns' load in flight while a chunk is
//          weighted), online softmax in base 2 with a lazy rescale of O
// Tensor memory: Q' [0, 64) | Q'' [64, 128) | S/P buffer 0 [128, 256) |
// S/P buffer 1 [256, 384) | O [384, 512).  The sign tile pairs coordinates
// (32g + c, 32g + 16 + c) in each 32-bit element, and Q'' is written with the
// same pairing (a consistent reordering of the K dimension of one product).
//
// Range: the fp16 key and value tiles hold n_k c, rn_k and n_v c_V, so key and
// value norms must stay below 65504 / max|c| (about 3e5 for these codebooks).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cfloat>
#include <cmath>

#include "sm100_common.cuh"
#include "tq_internal.h"

namespace tqi {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int kTK = 128;                 // keys per tile
constexpr int kRows = 128;               // query rows per CTA
constexpr int kThreads = 320;
constexpr int kStages = 3;               // ring stages of packed tiles
constexpr int kKW = 12, kSW = 4, kVW = 16;
constexpr int kOffK = 0, kOffS = kOffK + kTK * kKW * 4, kOffV = kOffS + kTK * kSW * 4;
// the three norm arrays of the tile follow the codes (whole groups of 4 tokens)
constexpr int kOffKN = kOffV + kTK * kVW * 4, kOffKR = kOffKN + kTK * 4, kOffVN = kOffKR + kTK * 4;
constexpr int kStage = kOffVN + kTK * 4;   // 17920
constexpr int kTile = 2 * kTK * 128;             // one [128 x 128] fp16 operand (two 64-wide slabs)
constexpr uint32_t kColQ1 = 0, kColQ2 = 64, kColS = 128, kColO = 384;   // S/P buffers at 128 and 256
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;            // rescale O only when the max grows by 2^8
// shared layout: the swizzled operand tiles first (1024-byte aligned)
constexpr int kOffC = 0;
constexpr int kOffSg = kOffC + kTile;
constexpr int kOffVt = kOffSg + kTile;                 // two value tiles
constexpr int kOffRing = kOffVt + 2 * kTile;
constexpr int kOffTab = kOffRing + kStages * kStage;   // value byte table, one copy per lane: [256][32]
constexpr int kOffBar = kOffTab + 256 * 32 * 4;
constexpr int kSmem = kOffBar + 256 + 1024;

struct PfArgs {
  const uint32_t* kcodes;
  const uint32_t* ksigns;
  const float* knorms;
  const float* krnorms;
  const uint32_t* vcodes;
  const float* vnorms;
  const float* qrot;       // [rows][d] fp32, rows = (b nq + i) Hq + j
  const float* qproj;
  uint32_t ktab[4];        // key codebook (8 entries) as fp16 byte tables: lo bytes c0-3, c4-7, hi bytes c0-3, c4-7
  const float* vcent;      // [16]
  int B, nq, Hq, Hkv, g;   // g = Hq / Hkv query heads per kv-head
  int64_t T, kv_stride;
  int qtiles, splits;
  int64_t ktiles;          // key tiles of the whole context
  float scale_log2;        // logit scale * log2(e)
  float qjl_coef;          // sqrt(pi/2) / d
  float* partials;         // [rows][splits][d + 2]
  int* status;
};

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// 2^x by the hardware's approximate exponential (subnormal results flush to 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// An empty statement that the compiler sees as redefining r: placed right after
// tcgen05.wait::ld, it keeps every use of the loaded registers behind the wait
// (the load's results are asynchronous, which the compiler does not know).
__device__ __forceinline__ void regs_after_wait(float (&r)[32]) {
  asm volatile(""
               : "+f"(r[0]), "+f"(r[1]), "+f"(r[2]), "+f"(r[3]), "+f"(r[4]), "+f"(r[5]), "+f"(r[6]), "+f"(r[7]), "+f"(r[8]), "+f"(r[9]), "+f"(r[10]), "+f"(r[11]), "+f"(r[12]), "+f"(r[13]), "+f"(r[14]), "+f"(r[15]), "+f"(r[16]), "+f"(r[17]), "+f"(r[18]), "+f"(r[19]), "+f"(r[20]), "+f"(r[21]), "+f"(r[22]), "+f"(r[23]), "+f"(r[24]), "+f"(r[25]), "+f"(r[26]), "+f"(r[27]), "+f"(r[28]), "+f"(r[29]), "+f"(r[30]), "+f"(r[31])::"memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// eight 3-bit codes in the nibbles of x (bit 3 of each nibble ignored) -> four
// fp16 pairs (codes 0,1 | 2,3 | 4,5 | 6,7) through register byte tables: one
// byte permute picks the low bytes of four centroids, another the high bytes
__device__ __forceinline__ void decode8(uint32_t x, const uint32_t (&t)[4], uint32_t* out) {
  const uint32_t s0 = x & 0x7777u, s1 = (x >> 16) & 0x7777u;
  const uint32_t l0 = prmt(t[0], t[1], s0), h0 = prmt(t[2], t[3], s0);
  const uint32_t l1 = prmt(t[0], t[1], s1), h1 = prmt(t[2], t[3], s1);
  out[0] = prmt(l0, h0, 0x5140);
  out[1] = prmt(l0, h0, 0x7362);
  out[2] = prmt(l1, h1, 0x5140);
  out[3] = prmt(l1, h1, 0x7362);
}

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzled
// canonical layout: 64-element (128-byte) rows along N, 8-row atoms along K
// `sbo` bytes apart, the next 64 N elements `lbo` bytes further.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// byte offset of 16-byte unit u (8 fp16) of row r in slab s of a [128 x 128] K-major 128B-swizzled tile
__device__ __forceinline__ uint32_t tile_off(int s, int r, int u) {
  return (uint32_t)(s * kTK * 128 + r * 128 + ((u ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(PfArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem + kOffRing;
  uint8_t* ctile = smem + kOffC;
  uint8_t* stile = smem + kOffSg;
  uint8_t* vtile = smem + kOffVt;
  uint32_t* vtab = reinterpret_cast<uint32_t*>(smem + kOffTab);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;          // [kStages] ring, tx
  uint64_t* empty = bars + 3;     // [kStages] ring, 4 decoder warps
  uint64_t* cs_ready = bars + 6;  // 4 decoder warps: centroid and sign tiles written
  uint64_t* cs_free = bars + 7;   // MMA commit: logit product done with them
  uint64_t* v_ready = bars + 8;   // [2] 4 decoder warps: value tile written
  uint64_t* v_free = bars + 10;   // [2] MMA commit: the value product done with the value tile
  uint64_t* pv_done = bars + 12;  // MMA commit: value product done
  uint64_t* s_full = bars + 13;   // [2] MMA commit: logit buffer holds S
  uint64_t* p_ready = bars + 15;  // [2] 4 softmax warps: P written into the buffer
  uint64_t* q_ready = bars + 17;  // 4 softmax warps
  uint64_t* done = bars + 18;     // MMA commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's (batch, kv-head, query tile, context slice)
  int64_t cid = blockIdx.x;
  const int split = (int)(cid % a.splits);
  cid /= a.splits;
  const int qt = (int)(cid % a.qtiles);
  cid /= a.qtiles;
  const int h = (int)(cid % a.Hkv);
  const int b = (int)(cid / a.Hkv);
  const int64_t bh = (int64_t)b * a.Hkv + h;
  const int tok_per_tile = kRows / a.g;
  const int i0 = qt * tok_per_tile;                      // first token of the tile
  const int i_last = min(a.nq, i0 + tok_per_tile) - 1;
  const int64_t pos_max = a.T - a.nq + i_last;           // last visible key of the tile
  const int64_t kt_lo = split * a.ktiles / a.splits;
  const int64_t kt_end = (split + 1) * a.ktiles / a.splits;
  const int64_t kt_hi = min(kt_end, pos_max / kTK + 1);
  const int nkt = kt_hi > kt_lo ? (int)(kt_hi - kt_lo) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    mbar_init(cs_ready, 4);
    mbar_init(cs_free, 1);
    mbar_init(pv_done, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&v_ready[s], 4);
      mbar_init(&v_free[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_ready[s], 4);
    }
    mbar_init(q_ready, 4);
    mbar_init(done, 1);
    fence_mbar_init();
  }
  // value byte table: byte B -> (c[B & 15], c[B >> 4]) as an fp16 pair, one
  // copy per lane (entry B of lane l at word 32 B + l), so that lookups of a
  // warp never share a bank
  for (int e = threadIdx.x; e < 256 * 32; e += blockDim.x) {
    const int byte = e >> 5;
    vtab[e] = h2u(__floats2half2_rn(a.vcent[byte & 15], a.vcent[byte >> 4]));
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nkt; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&empty[s], (uint32_t)(((it / kStages) & 1) ^ 1))) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        const int64_t t0 = (kt_lo + it) * kTK;
        const int n = (int)min((int64_t)kTK, a.T - t0);
        const int64_t r = bh * a.kv_stride + t0;
        uint8_t* st = ring + s * kStage;
        const int n4 = n & ~3;  // norms in whole 16-byte units; a tail of up to 3 comes from global memory
        mbar_arrive_expect_tx(&full[s], (uint32_t)(n * (kKW + kSW + kVW) * 4 + 3 * n4 * 4));
        bulk_load(st + kOffK, a.kcodes + r * kKW, n * kKW * 4, &full[s]);
        bulk_load(st + kOffS, a.ksigns + r * kSW, n * kSW * 4, &full[s]);
        bulk_load(st + kOffV, a.vcodes + r * kVW, n * kVW * 4, &full[s]);
        if (n4) {
          bulk_load(st + kOffKN, a.knorms + r, n4 * 4, &full[s]);
          bulk_load(st + kOffKR, a.krnorms + r, n4 * 4, &full[s]);
          bulk_load(st + kOffVN, a.vnorms + r, n4 * 4, &full[s]);
        }
        issued = it + 1;
      }
      // no bulk copy may still be in flight when the CTA exits
      for (int it = issued - kStages > 0 ? issued - kStages : 0; it < issued; ++it)
        if (!mbar_wait(&full[it % kStages], (uint32_t)((it / kStages) & 1))) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kRows, kTK, false);
      const uint32_t idesc_pv = idesc | (1u << 16);   // B (the value tile) MN-major
      const uint32_t cbase = smem_u32(ctile), sbase = smem_u32(stile), vbase = smem_u32(vtile);
      // S(i) = Q' C^T + Q'' Sg^T into buffer i & 1: K = 2 x 128 in 16 steps of 16
      auto logit_product = [&](int it) {
        const uint32_t sc = tmem + kColS + (uint32_t)(it & 1) * 128;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t boff = (uint32_t)((ks >> 2) * kTK * 128 + (ks & 3) * 32);
          mma_f16_ta(sc, tmem + kColQ1 + 8 * ks, sw128_kmajor_desc(cbase + boff), idesc, ks ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t boff = (uint32_t)((ks >> 2) * kTK * 128 + (ks & 3) * 32);
          mma_f16_ta(sc, tmem + kColQ2 + 8 * ks, sw128_kmajor_desc(sbase + boff), idesc, 1u);
        }
        mma_commit(&s_full[it & 1]);
        mma_commit(cs_free);
      };
      bool ok = nkt == 0 || (mbar_wait(q_ready, 0u) && mbar_wait(cs_ready, 0u));
      if (ok && nkt > 0) {
        tc_fence_after();
        logit_product(0);
      }
      for (int it = 0; ok && it < nkt; ++it) {
        if (it + 1 < nkt) {
          // buffer (it + 1) & 1 last held P(it - 1): the value product of tile it - 1 must be done with it
          if (!mbar_wait(cs_ready, (uint32_t)((it + 1) & 1)) ||
              (it > 0 && !mbar_wait(pv_done, (uint32_t)((it - 1) & 1)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          logit_product(it + 1);
        }
        if (!mbar_wait(&p_ready[it & 1], (uint32_t)((it >> 1) & 1)) ||
            !mbar_wait(&v_ready[it & 1], (uint32_t)((it >> 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // O += P V: K = 128 keys in 8 steps of 16 (P pairs keys 2m, 2m+1 in
        // column m); the value tile is MN-major (key rows of 128 bytes, 8-row
        // atoms 1024 bytes apart, coordinates 64..127 one slab further)
        const uint32_t pc = tmem + kColS + (uint32_t)(it & 1) * 128;
        const uint32_t vt = vbase + (uint32_t)(it & 1) * kTile;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_f16_ta(tmem + kColO, pc + 8 * ks, sw128_mnmajor_desc(vt + ks * 2048, kTK * 128, 1024), idesc_pv,
                     (it | ks) ? 1u : 0u);
        mma_commit(&v_free[it & 1]);
        mma_commit(pv_done);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done);
    }
  } else if (warp < 6) {
    // ---------------- decoders: thread t = key t of the tile
    const int t = threadIdx.x - 64;
    const uint32_t rb = smem_u32(ring);
    const uint32_t ctb = smem_u32(ctile), stb = smem_u32(stile), vtb = smem_u32(vtile);
    const uint32_t tab = smem_u32(vtab) + (uint32_t)lane * 4u;
    const uint32_t ktab[4] = {a.ktab[0], a.ktab[1], a.ktab[2], a.ktab[3]};
    // centroid row n_k c[idx] and sign row rn_k sign of key t (zeros past the context end)
    auto decode_keys = [&](int it) -> bool {
      const int s = it % kStages;
      const int64_t t0 = (kt_lo + it) * kTK;
      const int n = (int)min((int64_t)kTK, a.T - t0);
      const int64_t row0 = bh * a.kv_stride + t0;
      if (!mbar_wait_warp(&full[s], (uint32_t)((it / kStages) & 1)) ||
          (it > 0 && !mbar_wait_warp(cs_free, (uint32_t)((it - 1) & 1))))
        return false;
      const uint8_t* st = ring + s * kStage;
      const uint32_t sb = rb + (uint32_t)(s * kStage);
      const int n4 = n & ~3;
      const bool kin = t < n;
      const float kn = t < n4 ? reinterpret_cast<const float*>(st + kOffKN)[t] : (kin ? a.knorms[row0 + t] : 0.f);
      const float kr = t < n4 ? reinterpret_cast<const float*>(st + kOffKR)[t] : (kin ? a.krnorms[row0 + t] : 0.f);
      const __half2 kn2 = __float2half2_rn(kn);
      // -rn_k in both halves; a set sign bit of the code flips a half to +rn_k
      const uint32_t neg_rn = 0x80008000u | (0x00010001u * (uint32_t)__half_as_ushort(__float2half_rn(kr)));
      uint32_t w[kKW], sg[kSW];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const uint4 v = kin ? lds128(sb + kOffK + (uint32_t)(t * kKW * 4 + 16 * q)) : make_uint4(0u, 0u, 0u, 0u);
        w[4 * q] = v.x, w[4 * q + 1] = v.y, w[4 * q + 2] = v.z, w[4 * q + 3] = v.w;
      }
      {
        const uint4 v = kin ? lds128(sb + kOffS + (uint32_t)(t * kSW * 4)) : make_uint4(0u, 0u, 0u, 0u);
        sg[0] = v.x, sg[1] = v.y, sg[2] = v.z, sg[3] = v.w;
      }
#pragma unroll
      for (int gq = 0; gq < 4; ++gq) {  // 32-coordinate groups
        // nibbles of w0, w1, w2 hold coordinates 0-23, their fourth bits coordinates 24-31
        const uint32_t w0 = w[3 * gq], w1 = w[3 * gq + 1], w2 = w[3 * gq + 2];
        const uint32_t s3 = ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
        uint32_t pr[16];
        decode8(w0, ktab, pr);
        decode8(w1, ktab, pr + 4);
        decode8(w2, ktab, pr + 8);
        decode8(s3, ktab, pr + 12);
#pragma unroll
        for (int e = 0; e < 16; ++e) pr[e] = h2u(__hmul2(u2h(pr[e]), kn2));
        // 32 coordinates = 4 units of 8; group gq is slab gq / 2, units 4 (gq & 1) .. + 3
#pragma unroll
        for (int u = 0; u < 4; ++u)
          sts128(ctb + tile_off(gq >> 1, t, 4 * (gq & 1) + u), pr[4 * u], pr[4 * u + 1], pr[4 * u + 2],
                 pr[4 * u + 3]);
        // signs: element c of the group pairs coordinates (c, c + 16)
        uint32_t sp[16];
        const uint32_t x = sg[gq];
#pragma unroll
        for (int c = 0; c < 16; ++c) sp[c] = neg_rn ^ ((x << (15 - c)) & 0x80008000u);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          sts128(stb + tile_off(gq >> 1, t, 4 * (gq & 1) + u), sp[4 * u], sp[4 * u + 1], sp[4 * u + 2],
                 sp[4 * u + 3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(cs_ready);
      return true;
    };
    // row t of value tile it & 1 (MN-major: key rows of 128 bytes, 8-row atoms
    // 1024 bytes apart, coordinates 64..127 one slab further): n_v c_V[idx]
    const uint32_t row_off = (uint32_t)((t >> 3) * 1024 + (t & 7) * 128);
    const uint32_t sw = (uint32_t)(t & 7);
    auto decode_values = [&](int it) -> bool {
      // the tile's buffer was last read by the value product of tile it - 2
      if (it > 1 && !mbar_wait_warp(&v_free[it & 1], (uint32_t)(((it >> 1) - 1) & 1))) return false;
      const int s = it % kStages;
      const int64_t t0 = (kt_lo + it) * kTK;
      const int n = (int)min((int64_t)kTK, a.T - t0);
      const int64_t row0 = bh * a.kv_stride + t0;
      const uint8_t* st = ring + s * kStage;
      const uint32_t sb = rb + (uint32_t)(s * kStage) + kOffV + (uint32_t)(t * kVW * 4);
      const int n4 = n & ~3;
      const bool kin = t < n;
      const float vn = t < n4 ? reinterpret_cast<const float*>(st + kOffVN)[t] : (kin ? a.vnorms[row0 + t] : 0.f);
      const __half2 vn2 = __float2half2_rn(vn);
      uint32_t w[kVW];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = kin ? lds128(sb + 16 * q) : make_uint4(0u, 0u, 0u, 0u);
        w[4 * q] = v.x, w[4 * q + 1] = v.y, w[4 * q + 2] = v.z, w[4 * q + 3] = v.w;
      }
      const uint32_t vt = vtb + (uint32_t)((it & 1) * kTile) + row_off;
#pragma unroll
      for (int q = 0; q < kVW; ++q) {
        // word q: coordinates 8 q .. 8 q + 7, two per byte
        const uint32_t x = w[q];
        const uint32_t e0 = h2u(__hmul2(u2h(lds32(tab + ((x << 7) & 0x7F80u))), vn2));
        const uint32_t e1 = h2u(__hmul2(u2h(lds32(tab + ((x >> 1) & 0x7F80u))), vn2));
        const uint32_t e2 = h2u(__hmul2(u2h(lds32(tab + ((x >> 9) & 0x7F80u))), vn2));
        const uint32_t e3 = h2u(__hmul2(u2h(lds32(tab + ((x >> 17) & 0x7F80u))), vn2));
        const uint32_t m = (uint32_t)(q >> 3), j = (uint32_t)(q & 7);
        sts128(vt + m * (kTK * 128) + ((j ^ sw) << 4), e0, e1, e2, e3);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&v_ready[it & 1]);
        mbar_arrive(&empty[s]);
      }
      return true;
    };
    // keys run one tile ahead of values: the logit product of tile i + 1 needs
    // only the logit product of tile i to be done, and with two value tiles
    // the value tile of tile i waits for the value product of tile i - 2
    bool ok = nkt == 0 || decode_keys(0);
    for (int it = 0; ok && it < nkt; ++it) {
      if (it + 1 < nkt) ok = decode_keys(it + 1);
      if (ok) ok = decode_values(it);
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  } else {
    // ---------------- softmax: thread = query row (TMEM lane)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lb = (uint32_t)(quarter * 32) << 16;
    const int il = r / a.g, jl = r % a.g;
    const int tok = i0 + il;
    const bool live = il < tok_per_tile && tok < a.nq;
    const int64_t qrow = ((int64_t)b * a.nq + tok) * a.Hq + (int64_t)h * a.g + jl;   // global query row
    const int64_t pos = a.T - a.nq + tok;                                            // this row's position
    // queries into tensor memory: Q' natural pairs, Q'' pairs (32 g + c, 32 g + 16 + c), both with the
    // row's power-of-two scale s so that the two products add in one accumulator
    float inv;
    {
      const float* q1 = a.qrot + qrow * D;
      const float* q2 = a.qproj + qrow * D;
      const float cq = a.qjl_coef;
      float mx = 0.f;
      if (live)
        for (int j = 0; j < D; ++j) mx = fmaxf(mx, fmaxf(fabsf(q1[j]), fabsf(q2[j]) * cq));
      int e1 = 0;
      if (mx > 0.f) (void)frexpf(mx, &e1);
      const float s1 = mx > 0.f ? ldexpf(1.f, 14 - e1) : 1.f, s2 = s1 * cq;
      inv = 1.f / s1;
      for (int c0 = 0; c0 < 64; c0 += 16) {
        uint32_t u1[16], u2[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int col = c0 + c;                          // column 0..63
          const int j1 = 2 * col;                          // Q': coordinates 2 col, 2 col + 1
          const int gq = col >> 4, cc = col & 15;          // Q'': group gq, element cc
          const int j2a = 32 * gq + cc, j2b = j2a + 16;
          u1[c] = live ? h2u(__floats2half2_rn(q1[j1] * s1, q1[j1 + 1] * s1)) : 0u;
          u2[c] = live ? h2u(__floats2half2_rn(q2[j2a] * s2, q2[j2b] * s2)) : 0u;
        }
        tmem_st16(tmem + lb + kColQ1 + c0, u1);
        tmem_st16(tmem + lb + kColQ2 + c0, u2);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    const float cl = inv * a.scale_log2;    // base-2 logit = cl S
    float m_run = -FLT_MAX, l_run = 0.f;
    bool ok = true;
    for (int it = 0; ok && it < nkt; ++it) {
      const int64_t t0 = (kt_lo + it) * kTK;
      const uint32_t sc = tmem + lb + kColS + (uint32_t)(it & 1) * 128;
      if (!mbar_wait_warp(&s_full[it & 1], (uint32_t)((it >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // keys past this row's position (or the context end) take no part; only
      // a tile that some row of the warp does not see whole needs the test
      const int64_t rel = pos - t0;
      const int lim = live ? (int)(rel < 0 ? -1 : (rel > kTK - 1 ? kTK - 1 : rel)) : -1;
      const bool masked = __any_sync(0xffffffffu, lim < kTK - 1);
      // pass 1: the row max of the tile (four independent chains), 64 columns per tensor-memory wait
      float m4[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        float v[2][32];
        tmem_ld32(sc + 64 * hf, v[0]);
        tmem_ld32(sc + 64 * hf + 32, v[1]);
        tmem_wait_ld();
        regs_after_wait(v[0]);
        regs_after_wait(v[1]);
        if (masked) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) v[c][e] = 64 * hf + 32 * c + e <= lim ? v[c][e] : -FLT_MAX;
        }
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) m4[e & 3] = fmaxf(m4[e & 3], v[c][e]);
      }
      const float smx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      const float mx = smx > -FLT_MAX ? smx * cl : -FLT_MAX;
      // lazy rescale: a row's reference max moves only when one of its logits
      // passes it by kLazy (or on its first visible key)
      const bool grow = mx > m_run + kLazy || (m_run == -FLT_MAX && mx > -FLT_MAX);
      float alpha = 1.f;
      if (grow) {
        alpha = m_run > -FLT_MAX ? ex2(m_run - mx) : 0.f;
        l_run *= alpha;
        m_run = mx;
      }
      // pass 2: P = 2^(cl S - m) as fp16 pairs of consecutive keys, written over
      // the first 64 columns of the buffer (chunk c of 32 keys goes to columns
      // 16 c .. 16 c + 15, which hold logits already read); the load of the next
      // chunk is in flight while a chunk is weighted
      const float mref = m_run > -FLT_MAX ? m_run : 0.f;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      auto weights = [&](const float (&x)[32], int c) {
        float p[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) p[e] = ex2(fmaf(cl, x[e], -mref));
        if (masked) {
#pragma unroll
          for (int e = 0; e < 32; ++e) p[e] = 32 * c + e <= lim ? p[e] : 0.f;
        }
        uint32_t pu[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          ls[e & 3] += p[2 * e] + p[2 * e + 1];
          pu[e] = h2u(__floats2half2_rn(p[2 * e], p[2 * e + 1]));
        }
        tmem_st16(sc + 16 * c, pu);
      };
      {
        float va[32], vb[32];
        tmem_ld32(sc, va);
        tmem_wait_ld();
        regs_after_wait(va);
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          tmem_ld32(sc + 32 * (c + 1), vb);
          weights(va, c);
          tmem_wait_ld();
          regs_after_wait(vb);
          if (c + 2 < 4) tmem_ld32(sc + 32 * (c + 2), va);
          weights(vb, c + 1);
          if (c + 2 < 4) {
            tmem_wait_ld();
            regs_after_wait(va);
          }
        }
      }
      l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // O carries the value products of tiles before this one: once the last
      // of them is done, the rows whose reference max moved scale it by alpha.
      // The loads and stores are warp-collective, so the whole warp takes the
      // step when any of its rows needs it (the others scale by 1).
      if (it > 0 && __any_sync(0xffffffffu, grow)) {
        if (!mbar_wait_warp(pv_done, (uint32_t)((it - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32];
          tmem_ld32(tmem + lb + kColO + c0, o);
          tmem_wait_ld();
          regs_after_wait(o);
          uint32_t ou[16];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int e = 0; e < 16; ++e) ou[e] = __float_as_uint(o[16 * hh + e] * alpha);
            tmem_st16(tmem + lb + kColO + c0 + 16 * hh, ou);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[it & 1]);
    }
    // the record of this row: acc (rotated frame), m (natural units), l.  The
    // last value products are awaited through the issuer's final commit: the
    // parity of pv_done alone cannot tell phase nkt - 1 from phase nkt - 3 when
    // the value product of tile nkt - 2 is still running
    if (ok && nkt > 0 && !mbar_wait_warp(done, 0u)) ok = false;
    if (!ok) atomicOr(a.status, kStatusTimeout);
    tc_fence_after();
    // records are d + 2 = 130 floats apart, so a record starts on an 8-byte
    // (not always a 16-byte) boundary: two-float stores
    float* rec = a.partials + (qrow * a.splits + split) * (D + 2);
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      float o[32];
      if (nkt > 0) {
        tmem_ld32(tmem + lb + kColO + c0, o);
        tmem_wait_ld();
        regs_after_wait(o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0.f;
      }
      if (live)
#pragma unroll
        for (int e = 0; e < 32; e += 2) *reinterpret_cast<float2*>(rec + c0 + e) = make_float2(o[e], o[e + 1]);
    }
    if (live) {
      rec[D] = m_run > -FLT_MAX ? m_run / kLog2e : -FLT_MAX;
      rec[D + 1] = l_run;
    }
  }
  __syncthreads();
  if (warp == 1) {
    if (!mbar_wait(done, 0) && lane == 0) atomicOr(a.status, kStatusTimeout);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool prefill_supported(const tq_ctx* hk, const tq_ctx* hv, int Hq, int Hkv, int64_t kv_stride) {
  const int g = Hkv > 0 ? Hq / Hkv : 0;
  return hk->d == 128 && hv->d == 128 && hk->bm == 3 && hv->bm == 4 && g >= 1 && g <= 128 && (128 % g) == 0 &&
         Hq == g * Hkv && (kv_stride % 4) == 0;
}

// splits of the context per query tile: enough CTAs for two waves of the
// machine, at least 4 key tiles per slice
int prefill_splits(int B, int nq, int Hq, int Hkv, int64_t T, int sm_count) {
  const int g = Hq / Hkv;
  const int64_t qtiles = ((int64_t)nq * g + 127) / 128;
  const int64_t base = (int64_t)B * Hkv * qtiles;
  const int64_t ktiles = (T + kTK - 1) / kTK;
  int64_t s = (2 * (int64_t)sm_count + base - 1) / base;
  s = std::min<int64_t>(s, std::max<int64_t>(1, ktiles / 4));
  return (int)std::max<int64_t>(1, std::min<int64_t>(s, 64));
}

size_t prefill_partials_bytes(int B, int nq, int Hq, int Hkv, int64_t T, int sm_count) {
  return (size_t)B * nq * Hq * prefill_splits(B, nq, Hq, Hkv, T, sm_count) * (D + 2) * 4;
}

int launch_prefill(const tq_ctx* hk, const tq_ctx* hv, const float* qrot, const float* qproj, int B, int nq, int Hq,
                   int Hkv, int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                   const float* knorms, const float* krnorms, const uint32_t* vcodes, const float* vnorms, float scale,
                   float* partials, float* out, void* stream) {
  PfArgs a;
  a.kcodes = kcodes;
  a.ksigns = ksigns;
  a.knorms = knorms;
  a.krnorms = krnorms;
  a.vcodes = vcodes;
  a.vnorms = vnorms;
  a.qrot = qrot;
  a.qproj = qproj;
  for (int k = 0; k < 4; ++k) a.ktab[k] = hk->host_ktab[k];
  a.vcent = hv->dev.centroids;
  a.B = B;
  a.nq = nq;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.g = Hq / Hkv;
  a.T = T;
  a.kv_stride = kv_stride;
  a.qtiles = (int)(((int64_t)nq * a.g + kRows - 1) / kRows);
  a.splits = prefill_splits(B, nq, Hq, Hkv, T, hk->sm_count);
  a.ktiles = (T + kTK - 1) / kTK;
  a.scale_log2 = scale * kLog2e;
  a.qjl_coef = 1.2533141373155003f / 128.0f;
  a.partials = partials;
  a.status = hk->dev.status;
  if (int e = ensure_dyn_smem((const void*)prefill_kernel, kSmem)) return e;
  const int64_t grid = (int64_t)B * Hkv * a.qtiles * a.splits;
  cudaStream_t s = (cudaStream_t)stream;
  prefill_kernel<<<(unsigned)grid, kThreads, kSmem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  const int64_t rows = (int64_t)B * nq * Hq;
  return launch_decode_merge(partials, rows, a.splits, hv, out, stream, D + 2, (int64_t)a.splits * (D + 2), 0);
}

}  // namespace tqi

using namespace tqi;

static size_t pf_align(size_t v) { return (v + 255) / 256 * 256; }

extern "C" size_t tq_attn_prefill_workspace(tq_handle hk, int B, int nq, int Hq, int Hkv, int64_t T) {
  if (!hk || B < 0 || nq < 0 || Hq < 0 || Hkv <= 0 || T < 1 || Hq % Hkv != 0) return 0;
  const size_t rows = (size_t)B * nq * Hq;
  return 2 * pf_align(rows * hk->d * 4) + pf_align(prefill_partials_bytes(B, nq, Hq, Hkv, T, hk->sm_count));
}

extern "C" int tq_attn_prefill(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int nq, int Hq, int Hkv,
                               int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                               const float* knorms, const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                               float scale, float* out, void* workspace, size_t ws_bytes, void* stream) {
  TQ_TRACE("tq_attn_prefill");
  const char* fn = "tq_attn_prefill";
  if (!hk || !hv) return set_error(TQ_EINVAL, "%s: NULL handle", fn);
  if (hk->variant != TQ_PROD || hv->variant != TQ_MSE)
    return set_error(TQ_EINVAL, "%s: need a TQ_PROD key handle and a TQ_MSE value handle", fn);
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return set_error(TQ_EUNSUPPORTED, "%s: q_dtype %d", fn, q_dtype);
  if (B < 0 || nq < 0 || Hq < 0 || Hkv <= 0 || (Hq % Hkv) != 0 || T < 1 || nq > T || kv_stride < T)
    return set_error(TQ_EINVAL, "%s: bad shape (B=%d nq=%d Hq=%d Hkv=%d T=%lld stride=%lld)", fn, B, nq, Hq, Hkv,
                     (long long)T, (long long)kv_stride);
  if (!prefill_supported(hk, hv, Hq, Hkv, kv_stride))
    return set_error(TQ_EUNSUPPORTED,
                     "%s: the tensor-core prefill takes d = 128, keys TQ_PROD b = 4, values TQ_MSE b = 4, "
                     "Hq / Hkv dividing 128 and kv_stride %% 4 == 0", fn);
  if (!std::isfinite(scale)) return set_error(TQ_EINVAL, "%s: scale is not finite", fn);
  if (B == 0 || nq == 0 || Hq == 0) return clear_error();
  if (!q || !kcodes || !ksigns || !knorms || !krnorms || !vcodes || !vnorms || !out)
    return set_error(TQ_EINVAL, "%s: NULL pointer", fn);
  for (const void* p : {(const void*)q, (const void*)kcodes, (const void*)ksigns, (const void*)knorms,
                        (const void*)krnorms, (const void*)vcodes, (const void*)vnorms, (const void*)out,
                        (const void*)workspace})
    if (reinterpret_cast<uintptr_t>(p) & 15u) return set_error(TQ_EALIGN, "%s: a device pointer is not 16-byte aligned", fn);
  const size_t need = tq_attn_prefill_workspace(hk, B, nq, Hq, Hkv, T);
  if (!workspace || ws_bytes < need) return set_error(TQ_EWORKSPACE, "%s: workspace %zu < %zu bytes", fn, ws_bytes, need);
  const int64_t rows = (int64_t)B * nq * Hq;
  char* ws = static_cast<char*>(workspace);
  float* qrot = reinterpret_cast<float*>(ws);
  float* qproj = reinterpret_cast<float*>(ws + pf_align((size_t)rows * hk->d * 4));
  float* partials = reinterpret_cast<float*>(ws + 2 * pf_align((size_t)rows * hk->d * 4));
  int e = launch_query_prep(hk, static_cast<const float*>(q), q_dtype, rows, qrot, qproj, stream);
  if (!e)
    e = launch_prefill(hk, hv, qrot, qproj, B, nq, Hq, Hkv, T, kv_stride, kcodes, ksigns, knorms, krnorms, vcodes,
                       vnorms, scale, partials, out, stream);
  return e ? set_error(TQ_ECUDA, "%s: %s", fn, cudaGetErrorString((cudaError_t)e)) : clear_error();
}
