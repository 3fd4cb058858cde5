// Decode attention over a TurboQuant K/V cache on the tcgen05 tensor cores
// (sm_100a).
//
// turboquant.net/zh, "实现步骤草图", 集成到 attention: K and V are stored in
// TurboQuant form and QJL is used inside attention; tmdm.cn ("谷歌悄悄扔下一颗
// “性能核弹”…", 实测数据): attention logits computed directly over a 4-bit cache.
//
// One query token, the Hq = 4 Hkv heads of a kv-head's group sharing every key
// and value read.  Per tile of 128 tokens, two products on the tensor cores:
//   S[128 tok x 16] = [C | Sg] . Bq^T     C = key centroids c[idx] (fp16),
//                                          Sg = QJL signs as +-1, K = 256;
//                    Bq rows 0-3: q' of the 4 heads, 4-7: S q (each scaled by
//                    a power of two), rows 8-15 their fp16 remainders, so
//                    S[:, h] + S[:, 8 + h] = <c, q'_h> to ~22 bits
//   O[128 coord x 16] = Vt . P             Vt = value centroids (fp16, rotated
//                    frame) as an MN-major A operand (keys as K), P = the
//                    softmax weights times the value norms (fp16), 4 of 16 columns
// The key side of the first product lives in tensor memory (A operand, lane =
// token), the value tile in shared memory; S and O are tcgen05 accumulators.
// est = n <q', c> + rn sqrt(pi/2)/d <S q, sigma>, logits in base 2, the
// softmax max exact per tile; each tile's O is added into registers with the
// rescale of the running max, so tensor memory is never rescaled.
//
// Work split (as the mma.sync kernel): persistent CTAs own equal contiguous
// ranges of 128-token blocks over all (batch, kv-head) pairs; a CTA writes one
// softmax record (acc[d] in the rotated value frame, m, l) per head for each
// (batch, kv-head) it touches, and the merge kernel combines the CTAs and
// rotates back once.
//
// Warps (448 threads, one CTA per SM):
//   0      producer: bulk copies of each block (K codes, QJL signs, V codes,
//          the three norm arrays) into a 4-stage ring, and of the (batch,
//          kv-head)'s query tile when a new one starts
//   1      TMEM allocation and the single-thread MMA issuer
//   2-5    key decoders: thread = token = TMEM lane; 3-bit codes become fp16
//          pairs through byte permutes of a register table, QJL bits +-1.0
//          with one shift and one logic op per pair; tcgen05.st into the A stage
//   6-9    value decoders: thread = token; byte-indexed table in shared memory
//          (one copy per lane), rows of the MN-major value tile
//   10-13  softmax: thread = token (S lane) and coordinate (O lane)
// Tensor memory (512 columns): A stage s at 128 s (64 columns of centroid
// pairs, 64 of sign pairs), S[s] at 256 + 16 s, O[s] at 288 + 16 s.  The sign
// columns pair coordinates (32 g + c, 32 g + 16 + c); the S q rows of the query
// tile use the same pairing.
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

constexpr int D = 128;
constexpr int kTok = 128;                  // tokens per block
constexpr int kStages = 4;
constexpr int kThreads = 448;
constexpr int kKW = 12, kSW = 4, kVW = 16;
// ring stage
constexpr int kOffK = 0;
constexpr int kOffS = kOffK + kTok * kKW * 4;
constexpr int kOffV = kOffS + kTok * kSW * 4;
constexpr int kOffN = kOffV + kTok * kVW * 4;
constexpr int kOffR = kOffN + kTok * 4;
constexpr int kOffVN = kOffR + kTok * 4;
constexpr int kStageBytes = kOffVN + kTok * 4;  // 17920
// shared memory (1024-aligned base)
constexpr int kVtBytes = kTok * D * 2;           // one value tile: 32 KB
constexpr int kPBytes = 2 * 16 * 128;            // one weight tile: 2 slabs x 16 rows x 128 B
constexpr int kQBytes = 4 * 16 * 128;            // one query tile: 4 slabs x 16 rows x 128 B
constexpr int kTabBytes = 256 * 128;             // value table: row = code byte, one 4-byte copy per lane
constexpr int kOffRing = 0;
constexpr int kOffVt = kOffRing + kStages * kStageBytes;
constexpr int kOffP = kOffVt + 2 * kVtBytes;
constexpr int kOffQ = kOffP + 2 * kPBytes;
constexpr int kOffTab = kOffQ + 2 * kQBytes;
constexpr int kOffRed = kOffTab + kTabBytes;     // [2][4 warps][4 heads] tile maxima, [4][4] l partials
constexpr int kOffBar = kOffRed + 64 * 4;
constexpr int kSmem = kOffBar + 256 + 1024;
static_assert(kOffVt % 1024 == 0 && kOffP % 1024 == 0 && kOffQ % 1024 == 0 && kOffTab % 1024 == 0, "atoms");
static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
// tensor memory columns
constexpr uint32_t kColA = 0, kColS = 256, kColO = 288;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kPScale = 0.0625f;  // fp16 weights p |v| / 16 (the merge kernel undoes it)

struct TcDecArgs {
  const uint32_t* kcodes;
  const uint32_t* ksigns;
  const float* knorms;
  const float* krnorms;
  const uint32_t* vcodes;
  const float* vnorms;
  const uint8_t* qtiles;   // [B*Hkv][kQBytes]: the query tile of every (batch, kv-head)
  const float* qscale;     // [B*Hq][2]: 1/s of q' and of S q
  uint32_t ktab[4];        // key codebook as fp16 byte tables: lo bytes c0-3, c4-7, hi bytes c0-3, c4-7
  const uint32_t* vlut;    // [16]: fp16 of the value codebook in the low halves
  int B, Hq, Hkv;
  int64_t T, kv_stride;
  int64_t nblk, total;
  int max_seg;
  float scale_log2;
  float qjl_coef;
  float* partials;         // [CTA][max_seg][4 heads][d + 2]
  int* status;
  uint64_t wait_ns;
  int stall;
  int rn16;
};

// instruction descriptors: M = 128, N = 16, fp16, f32 accumulate; the value
// product's A operand is MN-major (bit 15)
constexpr uint32_t kIdescQK = idesc_f16(128, 16, false);
constexpr uint32_t kIdescPV = idesc_f16(128, 16, false) | (1u << 15);

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzled
// canonical layout: 64-element (128-byte) rows along M, 8-row atoms along K
// `sbo` bytes apart, the next 64 M elements `lbo` bytes further.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&r)[4]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
               : "r"(taddr));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
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

// eight 3-bit codes in the nibbles of x (bit 3 of each nibble ignored) -> four
// fp16 pairs (codes 0,1 | 2,3 | 4,5 | 6,7) through the register byte tables
__device__ __forceinline__ void decode8(uint32_t x, const uint32_t (&t)[4], uint32_t* out) {
  const uint32_t s0 = x & 0x7777u, s1 = (x >> 16) & 0x7777u;
  const uint32_t l0 = prmt(t[0], t[1], s0), h0 = prmt(t[2], t[3], s0);
  const uint32_t l1 = prmt(t[0], t[1], s1), h1 = prmt(t[2], t[3], s1);
  out[0] = prmt(l0, h0, 0x5140);
  out[1] = prmt(l0, h0, 0x7362);
  out[2] = prmt(l1, h1, 0x5140);
  out[3] = prmt(l1, h1, 0x7362);
}

__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(TcDecArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem + kOffRing;
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;            // [4] producer (tx)
  uint64_t* empty = bars + 4;       // [4] 12 consumer warps
  uint64_t* aqk_full = bars + 8;    // [2] 4 key-decoder warps
  uint64_t* qk_done = bars + 10;    // [2] MMA commit: A stage free
  uint64_t* s_full = bars + 12;     // [2] MMA commit
  uint64_t* s_free = bars + 14;     // [2] 4 softmax warps
  uint64_t* v_full = bars + 16;     // [2] 4 value-decoder warps
  uint64_t* p_full = bars + 18;     // [2] 4 softmax warps
  uint64_t* pv_done = bars + 20;    // [2] MMA commit: value and weight tiles free
  uint64_t* o_full = bars + 22;     // [2] MMA commit
  uint64_t* o_free = bars + 24;     // [2] 4 softmax warps
  uint64_t* q_free = bars + 26;     // [2] MMA commit after a (batch, kv-head)'s last key product
  uint64_t* done = bars + 28;       // MMA: everything issued has completed
  uint64_t* never = bars + 29;      // diagnostic: nothing arrives
  uint64_t* xbar = bars + 30;       // [2] 4 softmax warps: tile maxima written
  uint64_t* fbar = bars + 32;       // 4 softmax warps: l partials written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 34);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t gb_lo = blockIdx.x * a.total / G;
  const int64_t gb_hi = (blockIdx.x + 1) * a.total / G;
  const int nb = (int)(gb_hi - gb_lo);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 12);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&aqk_full[s], 4);
      mbar_init(&qk_done[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
      mbar_init(&v_full[s], 4);
      mbar_init(&p_full[s], 4);
      mbar_init(&pv_done[s], 1);
      mbar_init(&o_full[s], 1);
      mbar_init(&o_free[s], 4);
      mbar_init(&q_free[s], 1);
    }
    mbar_init(done, 1);
    mbar_init(never, 1);
    mbar_init(&xbar[0], 4);
    mbar_init(&xbar[1], 4);
    mbar_init(fbar, 4);
    fence_mbar_init();
  }
  // value table; weight tiles start at zero (rows 4-15 stay zero)
  {
    uint32_t* vt = reinterpret_cast<uint32_t*>(smem + kOffTab);
    for (int w = threadIdx.x; w < kTabBytes / 4; w += blockDim.x) {
      const uint32_t row = (uint32_t)w >> 5;
      vt[w] = (a.vlut[row & 15u] & 0xFFFFu) | (a.vlut[row >> 4] << 16);
    }
    uint32_t* pz = reinterpret_cast<uint32_t*>(smem + kOffP);
    for (int w = threadIdx.x; w < 2 * kPBytes / 4; w += blockDim.x) pz[w] = 0u;
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t wl = a.wait_ns;

  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      BlockCursor cur;
      cur.init(gb_lo, a.nblk);
      int issued = 0, seg = -1;
      for (int i = 0; i < nb; ++i, cur.next(a.nblk)) {
        const int r = i % kStages;
        if (!mbar_wait_ns(&empty[r], (uint32_t)(((i / kStages) & 1) ^ 1), wl)) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        const bool first = (i == 0 || cur.blk == 0);
        if (first) {
          ++seg;
          if (!mbar_wait_ns(&q_free[seg & 1], (uint32_t)(((seg >> 1) & 1) ^ 1), wl)) {
            atomicOr(a.status, kStatusTimeout);
            break;
          }
        }
        const int64_t t0 = cur.blk * kTok;
        const int n = (int)min((int64_t)kTok, a.T - t0);
        const int l4 = n & ~3, lr = a.rn16 ? (n & ~7) : l4;
        const int64_t row = cur.bh * a.kv_stride + t0;
        uint8_t* st = ring + r * kStageBytes;
        const uint32_t tx = (uint32_t)(n * (kKW + kSW + kVW) * 4 + 2 * l4 * 4 + lr * (a.rn16 ? 2 : 4)) +
                            (first ? (uint32_t)kQBytes : 0u);
        mbar_arrive_expect_tx(&full[r], tx);
        if (first) bulk_load(smem + kOffQ + (seg & 1) * kQBytes, a.qtiles + cur.bh * kQBytes, kQBytes, &full[r]);
        bulk_load(st + kOffK, a.kcodes + row * kKW, n * kKW * 4, &full[r]);
        bulk_load(st + kOffS, a.ksigns + row * kSW, n * kSW * 4, &full[r]);
        bulk_load(st + kOffV, a.vcodes + row * kVW, n * kVW * 4, &full[r]);
        if (l4) {
          bulk_load(st + kOffN, a.knorms + row, l4 * 4, &full[r]);
          bulk_load(st + kOffVN, a.vnorms + row, l4 * 4, &full[r]);
        }
        if (lr) {
          const int esz = a.rn16 ? 2 : 4;
          bulk_load(st + kOffR, reinterpret_cast<const uint8_t*>(a.krnorms) + row * esz, lr * esz, &full[r]);
        }
        issued = i + 1;
      }
      // every copy issued into this CTA's shared memory must land before it exits
      for (int i = issued - kStages > 0 ? issued - kStages : 0; i < issued; ++i)
        if (!mbar_wait(&full[i % kStages], (uint32_t)((i / kStages) & 1))) {
          atomicOr(a.status, kStatusTimeout);
          break;
        }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t qb = smem_u32(smem + kOffQ), vb = smem_u32(smem + kOffVt), pb = smem_u32(smem + kOffP);
      bool ok = true;
      BlockCursor cq;
      cq.init(gb_lo, a.nblk);
      int seg_q = -1;
      auto issue_qk = [&](int i) -> bool {
        const int s = i & 1;
        const uint32_t u = (uint32_t)(i >> 1);
        if (i == 0 || cq.blk == 0) ++seg_q;
        if (!mbar_wait_ns(&aqk_full[s], u & 1u, wl) || !mbar_wait_ns(&s_free[s], (u & 1u) ^ 1u, wl)) return false;
        tc_fence_after();
        const uint32_t q = qb + (uint32_t)((seg_q & 1) * kQBytes);
        const uint32_t acc = tmem + kColS + 16u * s, aa = tmem + kColA + 128u * s;
#pragma unroll
        for (int ks = 0; ks < 16; ++ks)
          mma_f16_ta(acc, aa + 8 * ks, sw128_kmajor_desc(q + (ks >> 2) * 2048 + (ks & 3) * 32), kIdescQK,
                     ks ? 1u : 0u);
        mma_commit(&qk_done[s]);
        mma_commit(&s_full[s]);
        const bool last = (i + 1 == nb) || (cq.blk + 1 == a.nblk);
        if (last) mma_commit(&q_free[seg_q & 1]);
        cq.next(a.nblk);
        return true;
      };
      if (nb > 0) ok = issue_qk(0);
      for (int i = 0; ok && i < nb; ++i) {
        if (i + 1 < nb && !issue_qk(i + 1)) {
          ok = false;
          break;
        }
        const int s = i & 1;
        const uint32_t u = (uint32_t)(i >> 1);
        if (!mbar_wait_ns(&v_full[s], u & 1u, wl) || !mbar_wait_ns(&p_full[s], u & 1u, wl) ||
            !mbar_wait_ns(&o_free[s], (u & 1u) ^ 1u, wl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + kColO + 16u * s;
        const uint32_t vt = vb + (uint32_t)(s * kVtBytes), pt = pb + (uint32_t)(s * kPBytes);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_f16(acc, sw128_mnmajor_desc(vt + ks * 2048, kTok * 128, 1024),
                  sw128_kmajor_desc(pt + (ks >> 2) * 2048 + (ks & 3) * 32), kIdescPV, ks ? 1u : 0u);
        mma_commit(&pv_done[s]);
        mma_commit(&o_full[s]);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      mma_commit(done);
    }
  } else if (warp < 6) {
    // ---------------- key decoders: thread = token = TMEM lane
    const int quarter = warp & 3;
    const int t = quarter * 32 + lane;
    const uint32_t lb = (uint32_t)(quarter * 32) << 16;
    const uint32_t tk[4] = {a.ktab[0], a.ktab[1], a.ktab[2], a.ktab[3]};
    const uint32_t rb = smem_u32(ring);
    bool ok = true;
    for (int i = 0; i < nb; ++i) {
      const int r = i % kStages, s = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      if (!mbar_wait_warp(&full[r], (uint32_t)((i / kStages) & 1), wl) ||
          !mbar_wait_warp(&qk_done[s], (u & 1u) ^ 1u, wl)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sb = rb + (uint32_t)(r * kStageBytes);
      uint32_t w[kKW], sg[kSW];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const uint4 v = lds128(sb + kOffK + (uint32_t)(t * kKW * 4 + 16 * q));
        w[4 * q] = v.x, w[4 * q + 1] = v.y, w[4 * q + 2] = v.z, w[4 * q + 3] = v.w;
      }
      {
        const uint4 v = lds128(sb + kOffS + (uint32_t)(t * kSW * 4));
        sg[0] = v.x, sg[1] = v.y, sg[2] = v.z, sg[3] = v.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[r]);
      const uint32_t aa = tmem + lb + kColA + 128u * s;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        // 32 coordinates: nibbles of w0, w1, w2 hold coordinates 0-23, their
        // fourth bits coordinates 24-31
        const uint32_t w0 = w[3 * g], w1 = w[3 * g + 1], w2 = w[3 * g + 2];
        const uint32_t s3 = ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
        uint32_t h[16];
        decode8(w0, tk, h);
        decode8(w1, tk, h + 4);
        decode8(w2, tk, h + 8);
        decode8(s3, tk, h + 12);
        tmem_st16(aa + 16 * g, h);
        // signs: column c pairs coordinates (32 g + c, 32 g + 16 + c); bit set = +1.0
        const uint32_t x = sg[g];
        uint32_t p[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) p[c] = 0xBC00BC00u ^ ((x << (15 - c)) & 0x80008000u);
        tmem_st16(aa + 64 + 16 * g, p);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aqk_full[s]);
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  } else if (warp < 10) {
    // ---------------- value decoders: thread = token, one row of the MN-major value tile
    const int t = (warp - 6) * 32 + lane;
    const uint32_t rb = smem_u32(ring);
    const uint32_t tab = smem_u32(smem + kOffTab) + (uint32_t)lane * 4u;
    // row t of the tile: 8-token atom t / 8 (1024 B apart), row t % 8 in it;
    // coordinates 64 m .. 64 m + 63 are 16 KB further for m = 1
    const uint32_t row_off = (uint32_t)((t >> 3) * 1024 + (t & 7) * 128);
    const uint32_t sw = (uint32_t)(t & 7);
    bool ok = true;
    for (int i = 0; i < nb; ++i) {
      const int r = i % kStages, s = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      if (!mbar_wait_warp(&full[r], (uint32_t)((i / kStages) & 1), wl) ||
          !mbar_wait_warp(&pv_done[s], (u & 1u) ^ 1u, wl)) {
        ok = false;
        break;
      }
      const uint32_t sb = rb + (uint32_t)(r * kStageBytes) + kOffV + (uint32_t)(t * kVW * 4);
      uint32_t w[kVW];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = lds128(sb + 16 * q);
        w[4 * q] = v.x, w[4 * q + 1] = v.y, w[4 * q + 2] = v.z, w[4 * q + 3] = v.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[r]);
      const uint32_t vt = smem_u32(smem + kOffVt + s * kVtBytes) + row_off;
#pragma unroll
      for (int q = 0; q < kVW; ++q) {
        // word q: coordinates 8 q .. 8 q + 7, two per byte
        const uint32_t x = w[q];
        const uint32_t e0 = lds32(tab + ((x << 7) & 0x7F80u));
        const uint32_t e1 = lds32(tab + ((x >> 1) & 0x7F80u));
        const uint32_t e2 = lds32(tab + ((x >> 9) & 0x7F80u));
        const uint32_t e3 = lds32(tab + ((x >> 17) & 0x7F80u));
        const uint32_t m = (uint32_t)(q >> 3), j = (uint32_t)(q & 7);
        sts128(vt + m * (kTok * 128) + ((j ^ sw) << 4), e0, e1, e2, e3);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_full[s]);
    }
    if (!ok) atomicOr(a.status, kStatusTimeout);
  } else {
    // ---------------- softmax: thread = token (S lane) and coordinate (O lane)
    const int quarter = warp & 3;
    const int sw_idx = warp - 10;              // slot in the exchange buffer
    const int t = quarter * 32 + lane;
    const uint32_t lb = (uint32_t)(quarter * 32) << 16;
    const int tid = threadIdx.x - 320;
    const int group = a.Hq / a.Hkv;            // 4
    bool ok = true;
    if (a.stall && !mbar_wait_warp(never, 0u, wl)) ok = false;
    float inv1[4] = {0.f, 0.f, 0.f, 0.f}, inv2[4] = {0.f, 0.f, 0.f, 0.f};
    float m_run[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX}, lsum[4] = {0.f, 0.f, 0.f, 0.f};
    float oreg[4] = {0.f, 0.f, 0.f, 0.f}, alpha_prev[4] = {1.f, 1.f, 1.f, 1.f};
    BlockCursor cur;
    cur.init(gb_lo, a.nblk);
    int seg = -1;
    const uint32_t pbase = smem_u32(smem + kOffP);
    // one softmax record per head of the segment: acc (lane = coordinate), m, l.
    // The warps exchange through mbarriers with bounded waits (a warp that gave
    // up must not leave the others waiting without a limit).
    int nflush = 0;
    auto flush = [&](int sg) -> bool {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float v = lsum[h];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        lsum[h] = v;
      }
      float* rl = red + 32;
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < 4; ++h) rl[sw_idx * 4 + h] = lsum[h];
        mbar_arrive(fbar);
      }
      if (!mbar_wait_warp(fbar, (uint32_t)(nflush & 1), wl)) return false;
      ++nflush;
      float* dst = a.partials + ((int64_t)blockIdx.x * a.max_seg + sg) * 4 * (D + 2);
#pragma unroll
      for (int h = 0; h < 4; ++h) dst[h * (D + 2) + t] = oreg[h];
      if (tid < 4) {
        const float l = rl[tid] + rl[4 + tid] + rl[8 + tid] + rl[12 + tid];
        float mr = m_run[0];
#pragma unroll
        for (int h = 1; h < 4; ++h) mr = tid == h ? m_run[h] : mr;
        dst[tid * (D + 2) + D] = mr > -FLT_MAX ? mr / kLog2e : -FLT_MAX;
        dst[tid * (D + 2) + D + 1] = l;
      }
      return true;
    };
    for (int i = 0; ok && i < nb; ++i, cur.next(a.nblk)) {
      const int r = i % kStages, s = i & 1;
      const uint32_t u = (uint32_t)(i >> 1);
      const bool first = (i == 0 || cur.blk == 0);
      const bool last = (i + 1 == nb) || (cur.blk + 1 == a.nblk);
      if (first) {
        ++seg;
        const int64_t b = cur.bh / a.Hkv, hh = cur.bh - b * a.Hkv;
        const int64_t q0 = b * a.Hq + hh * group;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          inv1[h] = a.qscale[2 * (q0 + h)] * a.scale_log2;
          inv2[h] = a.qscale[2 * (q0 + h) + 1] * a.qjl_coef * a.scale_log2;
          m_run[h] = -FLT_MAX;
          lsum[h] = 0.f;
          oreg[h] = 0.f;
          alpha_prev[h] = 1.f;
        }
      }
      const int64_t t0 = cur.blk * kTok;
      const int n = (int)min((int64_t)kTok, a.T - t0);
      if (!mbar_wait_warp(&s_full[s], u & 1u, wl)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[16];
      tmem_ld16(tmem + lb + kColS + 16u * s, sv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[s]);
      // norms of token t (whole 16-byte units were copied; a tail comes from global memory)
      const uint8_t* st = ring + r * kStageBytes;
      float kn = 0.f, kr = 0.f, vn = 0.f;
      const int l4 = n & ~3, lr = a.rn16 ? (n & ~7) : l4;
      if (t < n) {
        const int64_t row = cur.bh * a.kv_stride + t0 + t;
        kn = t < l4 ? reinterpret_cast<const float*>(st + kOffN)[t] : a.knorms[row];
        vn = t < l4 ? reinterpret_cast<const float*>(st + kOffVN)[t] : a.vnorms[row];
        if (a.rn16)
          kr = __half2float(t < lr ? reinterpret_cast<const __half*>(st + kOffR)[t]
                                   : reinterpret_cast<const __half*>(a.krnorms)[row]);
        else
          kr = t < lr ? reinterpret_cast<const float*>(st + kOffR)[t] : a.krnorms[row];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[r]);
      float lg[4], mx[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float e = fmaf(kn * inv1[h], sv[h] + sv[8 + h], kr * inv2[h] * (sv[4 + h] + sv[12 + h]));
        lg[h] = t < n ? e : -FLT_MAX;
        mx[h] = lg[h];
      }
      // the tile's max of every head over the 128 tokens
#pragma unroll
      for (int h = 0; h < 4; ++h)
        for (int o = 16; o > 0; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
      float* rx = red + s * 16;
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < 4; ++h) rx[sw_idx * 4 + h] = mx[h];
        mbar_arrive(&xbar[s]);
      }
      if (!mbar_wait_warp(&xbar[s], u & 1u, wl)) {
        ok = false;
        break;
      }
      float alpha[4], p[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float tm = fmaxf(fmaxf(rx[h], rx[4 + h]), fmaxf(rx[8 + h], rx[12 + h]));
        const float mn = fmaxf(m_run[h], tm);
        alpha[h] = exp2f(m_run[h] - mn);
        m_run[h] = mn;
        p[h] = t < n ? exp2f(lg[h] - mn) : 0.f;
        lsum[h] = fmaf(lsum[h], alpha[h], p[h] * kPScale);
      }
      // weights p |v| / 16 into row h of the weight tile (K-major, keys as K)
      if (!mbar_wait_warp(&pv_done[s], (u & 1u) ^ 1u, wl)) {
        ok = false;
        break;
      }
      {
        const uint32_t base = pbase + (uint32_t)(s * kPBytes) + (uint32_t)((t >> 6) * 2048) + (uint32_t)((t & 7) * 2);
        const uint32_t unit = (uint32_t)((t & 63) >> 3);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const __half wv = __float2half_rn(p[h] * vn * kPScale);
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(base + (uint32_t)(h * 128) + ((unit ^ (uint32_t)h) << 4)),
                       "h"(__half_as_ushort(wv))
                       : "memory");
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[s]);
      // fold the previous tile's O (same segment) into the registers: lane = coordinate t
      auto absorb = [&](int j, const float (&al)[4]) -> bool {
        const int sj = j & 1;
        if (!mbar_wait_warp(&o_full[sj], (uint32_t)((j >> 1) & 1), wl)) return false;
        tc_fence_after();
        float o[4];
        tmem_ld4(tmem + lb + kColO + 16u * sj, o);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[sj]);
#pragma unroll
        for (int h = 0; h < 4; ++h) oreg[h] = fmaf(oreg[h], al[h], o[h]);
        return true;
      };
      if (!first && !absorb(i - 1, alpha_prev)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int h = 0; h < 4; ++h) alpha_prev[h] = alpha[h];
      if (last) {
        if (!absorb(i, alpha)) {
          ok = false;
          break;
        }
        if (!flush(seg)) {
          ok = false;
          break;
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

// The query tile of every (batch, kv-head), in the 128B-swizzled K-major
// layout of a [16 x 256] fp16 B operand: rows 0-3 q' s' of the group's heads
// (K 0..127), rows 4-7 (S q) s'' (K 128..255, coordinates paired as the sign
// columns), rows 8-15 the fp16 remainders of rows 0-7; zeros elsewhere.  s',
// s'' put each copy's largest entry in (2^13, 2^14]; 1/s' and 1/s'' go to qscale.
// One 128-thread CTA per (batch, kv-head).
__global__ void __launch_bounds__(128) decode_tc_qtile_kernel(const float* qrot, const float* qproj, int Hq, int Hkv,
                                                              uint8_t* qtiles, float* qscale) {
  __shared__ float v[2][4][D];
  __shared__ float red[2][4][4];
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / Hkv, hh = bh % Hkv;
  const int group = Hq / Hkv;
  const int64_t q0 = b * Hq + hh * group;
  const int j = threadIdx.x, lane = j & 31, wp = j >> 5;
  for (int part = 0; part < 2; ++part)
    for (int h = 0; h < 4; ++h) {
      const float x = (part ? qproj : qrot)[(q0 + h) * D + j];
      float m = fabsf(x);
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[part][h][wp] = m;
      v[part][h][j] = x;
    }
  __syncthreads();
  __shared__ float sc[2][4];
  if (j < 8) {
    const int part = j >> 2, h = j & 3;
    const float mx = fmaxf(fmaxf(red[part][h][0], red[part][h][1]), fmaxf(red[part][h][2], red[part][h][3]));
    int e = 0;
    if (mx > 0.f) (void)frexpf(mx, &e);
    const float s = mx > 0.f ? ldexpf(1.f, 14 - e) : 1.f;
    sc[part][h] = s;
    qscale[2 * (q0 + h) + part] = 1.f / s;
  }
  __syncthreads();
  // thread j writes row j / 8, K elements 32 (j % 8) .. + 31 (four 16-byte units)
  const int row = j >> 3, kq = (j & 7) * 32;
  const bool lo = row >= 8;
  const int r8 = row & 7;
  const int part = r8 >> 2, h = r8 & 3;
  uint8_t* tile = qtiles + bh * (4 * 16 * 128);
  for (int uu = 0; uu < 4; ++uu) {
    const int k0 = kq + 8 * uu;
    uint32_t pk[4];
    for (int e = 0; e < 8; e += 2) {
      float x2[2];
      for (int f = 0; f < 2; ++f) {
        const int k = k0 + e + f;
        float x = 0.f;
        if (part == 0 && k < D) {
          x = v[0][h][k] * sc[0][h];
        } else if (part == 1 && k >= D) {
          const int kk = k - D, g = kk >> 5, ee = kk & 31;
          x = v[1][h][32 * g + (ee >> 1) + 16 * (ee & 1)] * sc[1][h];
        }
        const __half hi = __float2half_rn(x);
        x2[f] = lo ? x - __half2float(hi) : x;
      }
      const __half2 hv = __floats2half2_rn(x2[0], x2[1]);
      pk[e >> 1] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    const int slab = k0 >> 6, unit = (k0 & 63) >> 3;
    *reinterpret_cast<uint4*>(tile + slab * 2048 + row * 128 + ((unit ^ (row & 7)) << 4)) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

}  // namespace

bool decode_tc_supported(const tq_ctx* hk, const tq_ctx* hv, int Hq, int Hkv, int64_t kv_stride, int rn16) {
  return decode_mma_supported(hk, hv, Hq, Hkv, kv_stride) && hk->dev.ktab != nullptr && (!rn16 || kv_stride % 8 == 0) &&
         !hk->debug_fixed_tables && hk->tc_attn;
}

int decode_tc_grid(int B, int Hkv, int64_t T, int sm_count) {
  const int64_t total = (int64_t)B * Hkv * ((T + kTok - 1) / kTok);
  return (int)(total < sm_count ? total : sm_count);
}

int decode_tc_max_seg(int B, int Hkv, int64_t T, int sm_count) {
  const int64_t nblk = (T + kTok - 1) / kTok;
  const int64_t total = (int64_t)B * Hkv * nblk;
  const int64_t G = decode_tc_grid(B, Hkv, T, sm_count);
  const int64_t per = (total + G - 1) / G;
  return (int)((per + nblk - 1) / nblk + 1);
}

size_t decode_tc_qtile_bytes(int B, int Hkv) { return (size_t)B * Hkv * kQBytes; }

int launch_decode_tc(const tq_ctx* hk, const tq_ctx* hv, const float* qrot, const float* qproj, uint8_t* qtiles,
                     float* qscale, int B, int Hq, int Hkv, int64_t T, int64_t kv_stride, const uint32_t* kcodes,
                     const uint32_t* ksigns, const float* knorms, const float* krnorms, const uint32_t* vcodes,
                     const float* vnorms, float scale, float* partials, float* out, void* stream, int partial_out,
                     int rn16) {
  cudaStream_t s = (cudaStream_t)stream;
  decode_tc_qtile_kernel<<<(unsigned)((int64_t)B * Hkv), 128, 0, s>>>(qrot, qproj, Hq, Hkv, qtiles, qscale);
  if (cudaError_t e = cudaGetLastError()) return (int)e;
  TcDecArgs a;
  a.kcodes = kcodes;
  a.ksigns = ksigns;
  a.knorms = knorms;
  a.krnorms = krnorms;
  a.vcodes = vcodes;
  a.vnorms = vnorms;
  a.qtiles = qtiles;
  a.qscale = qscale;
  for (int k = 0; k < 4; ++k) a.ktab[k] = hk->host_ktab[k];
  a.vlut = hv->dev.lut_dq;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.T = T;
  a.kv_stride = kv_stride;
  a.nblk = (T + kTok - 1) / kTok;
  a.total = (int64_t)B * Hkv * a.nblk;
  a.max_seg = decode_tc_max_seg(B, Hkv, T, hk->sm_count);
  a.scale_log2 = scale * kLog2e;
  a.qjl_coef = 1.2533141373155003f / 128.0f;
  a.partials = partials;
  a.status = hk->dev.status;
  a.wait_ns = hk->debug_stall_ns ? hk->debug_stall_ns : kWaitLimitNs;
  a.stall = hk->debug_stall_ns ? 1 : 0;
  a.rn16 = rn16;
  const int G = decode_tc_grid(B, Hkv, T, hk->sm_count);
  if (int e = ensure_dyn_smem((const void*)decode_tc_kernel, kSmem)) return e;
  decode_tc_kernel<<<G, kThreads, kSmem, s>>>(a);
  if (cudaError_t e = cudaGetLastError()) return (int)e;
  return launch_decode_merge_records(partials, G, a.max_seg, a.nblk, a.total, B, Hq, Hkv, hv, out, partial_out,
                                     stream);
}

}  // namespace tqi
