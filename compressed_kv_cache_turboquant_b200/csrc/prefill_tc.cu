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
// product runs on tcgen05 with the decoded cache as the shared-memory operand:
//   S1 = Q' C^T      Q' = Pi_K q (fp16, per-row power-of-two scale), C = the
//                    key centroids c[idx] (fp16)
//   S2 = Q'' Sg^T    Q'' = S_K q, Sg = the QJL signs as +-1
//   logit = scale (n_k S1 / s' + rn_k sqrt(pi/2)/d S2 / s'')
//   O   += P V^T-tile  P = e^(logit - m) (fp16, written back into tensor memory),
//                    V = n_v c_V[idx] (fp16) in the rotated value frame
// One CTA per (batch, kv-head, tile of 128 query rows, slice of the context);
// a query row is a (token, head of the kv-head's group) pair.  Q' and Q'' live
// in tensor memory as the A operands of the two logit products, P overwrites
// S1 as the A operand of the value product; the decoded key and value tiles
// are the B operands in shared memory.  Each CTA writes its rows' softmax
// records (acc in the rotated frame, m, l); the merge kernel combines the
// slices and applies Pi_V^T once.
//
// Warps (320 threads, one CTA per SM):
//   0      bulk copies of each 128-token tile of packed K codes, QJL signs and
//          V codes into a two-stage ring
//   1      TMEM allocation and the single-thread MMA issuer
//   2-5    decoders: thread t decodes key t into the centroid and sign tiles
//          (byte-table lookups, one shift and one logic op per sign pair), then
//          key pairs into the transposed value tile (keys as the K dimension)
//   6-9    softmax: thread = query row (TMEM lane), online softmax in base 2
//          with a lazy rescale of O
// Tensor memory: Q' [0, 64) | Q'' [64, 128) | S1 / P [128, 256) | S2 [256, 384)
// | O [384, 512).  The sign tile pairs coordinates (32g + c, 32g + 16 + c) in
// each 32-bit element, and Q'' is written with the same pairing (a consistent
// reordering of the K dimension of one product).
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
constexpr int kKW = 12, kSW = 4, kVW = 16;
constexpr int kOffK = 0, kOffS = kOffK + kTK * kKW * 4, kOffV = kOffS + kTK * kSW * 4;
// the three norm arrays of the tile follow the codes (whole groups of 4 tokens)
constexpr int kOffKN = kOffV + kTK * kVW * 4, kOffKR = kOffKN + kTK * 4, kOffVN = kOffKR + kTK * 4;
constexpr int kStage = kOffVN + kTK * 4;   // 17920
constexpr int kTile = 2 * kTK * 128;             // one [128 x 128] fp16 operand (two 64-wide slabs)
constexpr uint32_t kColQ1 = 0, kColQ2 = 64, kColS1 = 128, kColS2 = 256, kColO = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;            // rescale O only when the max grows by 2^8
// shared layout
constexpr int kOffRing = 0;
constexpr int kOffC = kOffRing + 2 * kStage;
constexpr int kOffSg = kOffC + kTile;
constexpr int kOffVt = kOffSg + kTile;
constexpr int kOffTab = kOffVt + kTile;          // K table [256] + V table [256] fp16 pairs
constexpr int kOffNorm = kOffTab + 2 * 1024;     // [2][2][128] kn, kr
constexpr int kOffBar = kOffNorm + 2 * 2 * kTK * 4;
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
  const float* kcent;      // [8]
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
  uint32_t* ktab = reinterpret_cast<uint32_t*>(smem + kOffTab);
  uint32_t* vtab = ktab + 256;
  float* nrm = reinterpret_cast<float*>(smem + kOffNorm);     // [2 buffers][kn 128 | kr 128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;          // [2] ring, tx
  uint64_t* empty = bars + 2;     // [2] ring, 4 decoder warps
  uint64_t* cs_ready = bars + 4;  // 4 decoder warps
  uint64_t* cs_free = bars + 5;   // MMA commit
  uint64_t* v_ready = bars + 6;   // 4 decoder warps
  uint64_t* pv_done = bars + 7;   // MMA commit
  uint64_t* s_full = bars + 8;    // MMA commit
  uint64_t* p_ready = bars + 9;   // 4 softmax warps
  uint64_t* q_ready = bars + 10;  // 4 softmax warps
  uint64_t* done = bars + 11;     // MMA commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);

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
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    mbar_init(cs_ready, 4);
    mbar_init(cs_free, 1);
    mbar_init(v_ready, 4);
    mbar_init(pv_done, 1);
    mbar_init(s_full, 1);
    mbar_init(p_ready, 4);
    mbar_init(q_ready, 4);
    mbar_init(done, 1);
    fence_mbar_init();
  }
  // byte tables: K byte -> (c[B & 7], c[(B >> 4) & 7]), V byte -> (c[B & 15], c[B >> 4]) as fp16 pairs
  for (int e = threadIdx.x; e < 256; e += blockDim.x) {
    ktab[e] = h2u(__floats2half2_rn(a.kcent[e & 7], a.kcent[(e >> 4) & 7]));
    vtab[e] = h2u(__floats2half2_rn(a.vcent[e & 15], a.vcent[e >> 4]));
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
        const int s = it & 1;
        if (!mbar_wait(&empty[s], (uint32_t)(((it >> 1) & 1) ^ 1))) {
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
      for (int it = issued - 2 > 0 ? issued - 2 : 0; it < issued; ++it)
        if (!mbar_wait(&full[it & 1], (uint32_t)((it >> 1) & 1))) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kRows, kTK, false);
      const uint32_t cbase = smem_u32(ctile), sbase = smem_u32(stile), vbase = smem_u32(vtile);
      bool ok = mbar_wait(q_ready, 0u);
      for (int it = 0; ok && it < nkt; ++it) {
        if (!mbar_wait(cs_ready, (uint32_t)(it & 1)) || (it > 0 && !mbar_wait(pv_done, (uint32_t)((it - 1) & 1)))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // S1 = Q' C^T, S2 = Q'' Sg^T: K = 128 coordinates in 8 steps of 16
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t boff = (uint32_t)((ks >> 2) * kTK * 128 + (ks & 3) * 32);
          mma_f16_ta(tmem + kColS1, tmem + kColQ1 + 8 * ks, sw128_kmajor_desc(cbase + boff), idesc, ks ? 1u : 0u);
          mma_f16_ta(tmem + kColS2, tmem + kColQ2 + 8 * ks, sw128_kmajor_desc(sbase + boff), idesc, ks ? 1u : 0u);
        }
        mma_commit(s_full);
        mma_commit(cs_free);
        if (!mbar_wait(p_ready, (uint32_t)(it & 1)) || !mbar_wait(v_ready, (uint32_t)(it & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // O += P Vt: K = 128 keys in 8 steps of 16 (P pairs keys 2m, 2m+1 in column m)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t boff = (uint32_t)((ks >> 2) * kTK * 128 + (ks & 3) * 32);
          mma_f16_ta(tmem + kColO, tmem + kColS1 + 8 * ks, sw128_kmajor_desc(vbase + boff), idesc,
                 (it | ks) ? 1u : 0u);
        }
        mma_commit(pv_done);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done);
    }
  } else if (warp < 6) {
    // ---------------- decoders
    const int t = threadIdx.x - 64;          // key of the tile (centroid and sign rows)
    const int m = t & 63, ch = t >> 6;       // key pair (2m, 2m+1) and coordinate half for the value tile
    bool ok = true;
    for (int it = 0; ok && it < nkt; ++it) {
      const int s = it & 1;
      const int64_t t0 = (kt_lo + it) * kTK;
      const int n = (int)min((int64_t)kTK, a.T - t0);
      const int64_t row0 = bh * a.kv_stride + t0;
      if (!mbar_wait_warp(&full[s], (uint32_t)((it >> 1) & 1)) ||
          (it > 0 && !mbar_wait_warp(cs_free, (uint32_t)((it - 1) & 1)))) {
        ok = false;
        break;
      }
      const uint8_t* st = ring + s * kStage;
      // centroid row and sign row of key t (zeros past the context end)
      {
        uint32_t w[kKW], sg[kSW];
        if (t < n) {
#pragma unroll
          for (int q = 0; q < kKW; ++q) w[q] = reinterpret_cast<const uint32_t*>(st + kOffK)[t * kKW + q];
#pragma unroll
          for (int q = 0; q < kSW; ++q) sg[q] = reinterpret_cast<const uint32_t*>(st + kOffS)[t * kSW + q];
        } else {
#pragma unroll
          for (int q = 0; q < kKW; ++q) w[q] = 0u;
#pragma unroll
          for (int q = 0; q < kSW; ++q) sg[q] = 0u;
        }
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {  // 32-coordinate groups
          const uint32_t w0 = w[3 * gq], w1 = w[3 * gq + 1], w2 = w[3 * gq + 2];
          const uint32_t s3 = ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
          const uint32_t src[4] = {w0, w1, w2, s3};
          uint32_t pr[16];
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int by = 0; by < 4; ++by) pr[4 * q + by] = t < n ? ktab[(src[q] >> (8 * by)) & 0xFFu] : 0u;
          // 32 coordinates = 4 units of 8; group gq is slab gq / 2, units 4 (gq & 1) .. + 3
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(ctile + tile_off(gq >> 1, t, 4 * (gq & 1) + u)) =
                make_uint4(pr[4 * u], pr[4 * u + 1], pr[4 * u + 2], pr[4 * u + 3]);
          // signs: element c of the group pairs coordinates (c, c + 16): +1.0 = 0x3C00, -1.0 = 0xBC00
          uint32_t sp[16];
          const uint32_t x = sg[gq];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            sp[c] = t < n ? (0xBC00BC00u ^ ((x << (15 - c)) & 0x80008000u)) : 0u;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(stile + tile_off(gq >> 1, t, 4 * (gq & 1) + u)) =
                make_uint4(sp[4 * u], sp[4 * u + 1], sp[4 * u + 2], sp[4 * u + 3]);
        }
        float* nb = nrm + (it & 1) * 2 * kTK;
        const int n4 = n & ~3;
        const float* skn = reinterpret_cast<const float*>(st + kOffKN);
        const float* skr = reinterpret_cast<const float*>(st + kOffKR);
        nb[t] = t < n4 ? skn[t] : (t < n ? a.knorms[row0 + t] : 0.f);
        nb[kTK + t] = t < n4 ? skr[t] : (t < n ? a.krnorms[row0 + t] : 0.f);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(cs_ready);
      // transposed value tile: row = coordinate, K = keys; thread (m, ch) writes
      // the words (v[2m][c], v[2m+1][c]) for coordinates c of half ch
      if (it > 0 && !mbar_wait_warp(pv_done, (uint32_t)((it - 1) & 1))) {
        ok = false;
        break;
      }
      {
        const int k0 = 2 * m, k1 = 2 * m + 1;
        const int n4 = n & ~3;
        const float* svn = reinterpret_cast<const float*>(st + kOffVN);
        const __half2 n0 = __float2half2_rn(k0 < n4 ? svn[k0] : (k0 < n ? a.vnorms[row0 + k0] : 0.f));
        const __half2 n1 = __float2half2_rn(k1 < n4 ? svn[k1] : (k1 < n ? a.vnorms[row0 + k1] : 0.f));
        const uint32_t* v0 = reinterpret_cast<const uint32_t*>(st + kOffV) + k0 * kVW + 8 * ch;
        const uint32_t* v1 = v0 + kVW;
        const int slab = m >> 5, unit = (m & 31) >> 2, sub = (m & 3) * 4;
#pragma unroll
        for (int q = 0; q < 8; ++q) {           // code word q: coordinates 64 ch + 8 q .. + 7
          const uint32_t a0 = k0 < n ? v0[q] : 0u, a1 = k1 < n ? v1[q] : 0u;
#pragma unroll
          for (int by = 0; by < 4; ++by) {      // byte: coordinates 2 by, 2 by + 1 of the word
            const uint32_t p0 = h2u(__hmul2(u2h(vtab[(a0 >> (8 * by)) & 0xFFu]), n0));
            const uint32_t p1 = h2u(__hmul2(u2h(vtab[(a1 >> (8 * by)) & 0xFFu]), n1));
            const int c = 64 * ch + 8 * q + 2 * by;
            *reinterpret_cast<uint32_t*>(vtile + tile_off(slab, c, unit) + sub) = __byte_perm(p0, p1, 0x5410);
            *reinterpret_cast<uint32_t*>(vtile + tile_off(slab, c + 1, unit) + sub) = __byte_perm(p0, p1, 0x7632);
          }
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(v_ready);
        mbar_arrive(&empty[s]);
      }
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
    const int64_t grow = ((int64_t)b * a.nq + tok) * a.Hq + (int64_t)h * a.g + jl;   // global query row
    const int64_t pos = a.T - a.nq + tok;                                            // this row's position
    // queries into tensor memory: Q' natural pairs, Q'' pairs (32 g + c, 32 g + 16 + c)
    float inv1, inv2;
    {
      const float* q1 = a.qrot + grow * D;
      const float* q2 = a.qproj + grow * D;
      float mx1 = 0.f, mx2 = 0.f;
      if (live)
        for (int j = 0; j < D; ++j) mx1 = fmaxf(mx1, fabsf(q1[j])), mx2 = fmaxf(mx2, fabsf(q2[j]));
      int e1 = 0, e2 = 0;
      if (mx1 > 0.f) (void)frexpf(mx1, &e1);
      if (mx2 > 0.f) (void)frexpf(mx2, &e2);
      const float s1 = mx1 > 0.f ? ldexpf(1.f, 14 - e1) : 1.f, s2 = mx2 > 0.f ? ldexpf(1.f, 14 - e2) : 1.f;
      inv1 = 1.f / s1;
      inv2 = 1.f / s2;
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
    const float c1 = inv1 * a.scale_log2, c2 = inv2 * a.qjl_coef * a.scale_log2;
    float m_run = -FLT_MAX, l_run = 0.f;
    bool ok = true;
    for (int it = 0; ok && it < nkt; ++it) {
      const int64_t t0 = (kt_lo + it) * kTK;
      if (!mbar_wait_warp(s_full, (uint32_t)(it & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* nb = nrm + (it & 1) * 2 * kTK;
      // logits (base 2) of 32 keys from the two accumulators, one tensor-memory
      // wait for both 32-column loads; keys past this row's position (or the
      // context end) are -FLT_MAX
      auto logits32 = [&](int c0, float (&x)[32]) {
        float v1[32], v2[32];
        tmem_ld32(tmem + lb + kColS1 + c0, v1);
        tmem_ld32(tmem + lb + kColS2 + c0, v2);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int k = c0 + e;
          const bool vis = live && t0 + k <= pos && t0 + k < a.T;
          x[e] = vis ? fmaf(nb[k] * c1, v1[e], nb[kTK + k] * c2 * v2[e]) : -FLT_MAX;
        }
      };
      // pass 1: the row max of the tile
      float mx = -FLT_MAX;
#pragma unroll 1
      for (int c0 = 0; c0 < kTK; c0 += 32) {
        float x[32];
        logits32(c0, x);
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, x[e]);
      }
      // lazy rescale: a row's reference max moves only when one of its logits
      // passes it by kLazy.  The O rescale goes through warp-collective tensor
      // memory loads and stores, so the whole warp takes it when any row needs
      // it (rows that do not rescale by 1).
      const bool grow = mx > m_run + kLazy || (it == 0 && mx > -FLT_MAX);
      const float mn = grow ? mx : m_run;
      if (it > 0 && __any_sync(0xffffffffu, grow)) {
        const float alpha = grow ? exp2f(m_run - mn) : 1.f;
        if (!mbar_wait_warp(pv_done, (uint32_t)((it - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32];
          tmem_ld32(tmem + lb + kColO + c0, o);
          tmem_wait_ld();
          uint32_t ou[16];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int e = 0; e < 16; ++e) ou[e] = __float_as_uint(o[16 * hh + e] * alpha);
            tmem_st16(tmem + lb + kColO + c0 + 16 * hh, ou);
          }
        }
        tmem_wait_st();
      }
      if (grow) {
        l_run *= (it > 0) ? exp2f(m_run - mn) : 0.f;
        m_run = mn;
      }
      // pass 2: P (fp16 pairs of consecutive keys), 32 keys at a time; the 16
      // columns written hold keys the earlier reads have consumed
#pragma unroll 1
      for (int c0 = 0; c0 < kTK; c0 += 32) {
        float x[32];
        logits32(c0, x);
        uint32_t pu[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float xa = x[2 * e];
          const float xb = x[2 * e + 1];
          const float p0 = xa > -FLT_MAX ? exp2f(xa - m_run) : 0.f;
          const float p1 = xb > -FLT_MAX ? exp2f(xb - m_run) : 0.f;
          const __half2 ph = __floats2half2_rn(p0, p1);
          l_run += __low2float(ph) + __high2float(ph);
          pu[e] = h2u(ph);
        }
        tmem_st16(tmem + lb + kColS1 + c0 / 2, pu);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready);
    }
    // the record of this row: acc (rotated frame), m (natural units), l
    if (ok && nkt > 0 && !mbar_wait_warp(pv_done, (uint32_t)((nkt - 1) & 1))) ok = false;
    if (!ok) atomicOr(a.status, kStatusTimeout);
    tc_fence_after();
    // records are d + 2 = 130 floats apart, so a record starts on an 8-byte
    // (not always a 16-byte) boundary: two-float stores
    float* rec = a.partials + (grow * a.splits + split) * (D + 2);
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      float o[32];
      if (nkt > 0) {
        tmem_ld32(tmem + lb + kColO + c0, o);
        tmem_wait_ld();
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
  a.kcent = hk->dev.centroids;
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
