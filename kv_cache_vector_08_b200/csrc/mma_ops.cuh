// Register-level building blocks shared by the mma.sync kernels that read the packed
// cache (decode attention, standalone logits, search).
#pragma once

#include <cstdint>

#include "common.cuh"

namespace tq {
namespace mmaops {

constexpr float kFix = 32000.f;    // fixed-point range of queries and key centroids (< 2^15)

// D += A * B, int8 operands, int32 accumulators (16 x 8 x 32)
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// 0xFF in every byte whose msb is set, 0x00 elsewhere (prmt sign replication)
__device__ __forceinline__ uint32_t msb_bytes(uint32_t x) { return prmt(x, x, 0xBA98u); }

// Lookup tables, built on the host from the contexts' codebooks: key centroids by code as
// two int8 digits of round(c * kc_scale) (hi = floor((C+128)/256), lo = C - 256 hi), value
// magnitudes c[K/2 + m] as fp16 low / high bytes.  8 entries = 2 registers per table.
struct Luts {
  uint32_t kh[2], kl[2], vlo[2], vhi[2];
};

// Fills the tables of one (key context, value context) pair; returns 1 / key-centroid scale.
float host_luts(const tq_ctx* kc, const tq_ctx* vc, Luts* t);

}  // namespace mmaops
}  // namespace tq
