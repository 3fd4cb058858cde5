// Register-fragment helpers shared by the mma.sync kernels over packed codes:
// byte-permute addressed table lookups (one table copy per lane, so the 32
// lookups of a warp never meet in a shared-memory bank) and the m16n8k16
// fp16 MMA with fp32 accumulation.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tqi {
namespace frag {

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) { return __byte_perm(a, b, s); }

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Table loads.  A kernel instantiated for the shared address at which its
// dynamic window starts (known on the host: see probe_dyn_smem_base) passes
// each table's absolute address as ADDR, and the address goes into the load's
// immediate offset; with ADDR = kDynRuntime the table address `tab` is added
// at run time (one integer add per lookup).
constexpr uint32_t kDynRuntime = 0xFFFFFFFFu;
// the dynamic window's start on sm_100 with the driver this library targets
// (the first 1 KB of a CTA's shared window is reserved); kernels also have an
// instance for kDynRuntime, taken when the probe reports another address
constexpr uint32_t kDynBaseSm100 = 1024u;

__host__ __device__ constexpr uint32_t tab_addr(uint32_t dyn_base, uint32_t offset) {
  return dyn_base == kDynRuntime ? kDynRuntime : dyn_base + offset;
}

template <uint32_t ADDR>
__device__ __forceinline__ uint32_t tab_ld32(uint32_t tab, uint32_t idx) {
  if constexpr (ADDR == kDynRuntime) {
    return lds32(tab + idx);
  } else {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(idx), "n"(ADDR));
    return v;
  }
}

template <uint32_t ADDR>
__device__ __forceinline__ uint2 tab_ld64(uint32_t tab, uint32_t idx) {
  if constexpr (ADDR == kDynRuntime) {
    return lds64(tab + idx);
  } else {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(idx), "n"(ADDR));
    return v;
  }
}

template <uint32_t ADDR>
__device__ __forceinline__ uint4 tab_ld128(uint32_t tab, uint32_t idx) {
  if constexpr (ADDR == kDynRuntime) {
    return lds128(tab + idx);
  } else {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4+%5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(idx), "n"(ADDR));
    return v;
  }
}

// the 4 bytes of a code word -> 4 fp16 pairs; `lane_off` holds this lane's
// column offset in byte 0, `tab` the table's shared-memory address (used when
// ADDR = kDynRuntime)
template <uint32_t ADDR>
__device__ __forceinline__ void lookup4(uint32_t w, uint32_t tab, uint32_t lane_off, uint32_t* out) {
  out[0] = tab_ld32<ADDR>(tab, prmt(w, lane_off, 0x5504));
  out[1] = tab_ld32<ADDR>(tab, prmt(w, lane_off, 0x5514));
  out[2] = tab_ld32<ADDR>(tab, prmt(w, lane_off, 0x5524));
  out[3] = tab_ld32<ADDR>(tab, prmt(w, lane_off, 0x5534));
}

// Position of a global token block gb = bh * nblk + blk, advanced one block at a
// time: the hot loops never divide 64-bit integers (a software routine of
// dozens of instructions per division).
struct BlockCursor {
  int64_t bh, blk;
  __device__ __forceinline__ void init(int64_t gb, int64_t nblk) {
    bh = gb / nblk;
    blk = gb - bh * nblk;
  }
  __device__ __forceinline__ void next(int64_t nblk) {
    if (++blk == nblk) blk = 0, ++bh;
  }
};

}  // namespace frag
}  // namespace tqi
