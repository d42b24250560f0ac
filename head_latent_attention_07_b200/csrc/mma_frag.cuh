// Warp-level bf16 tensor-core tiles (mma.sync m16n8k16, fp32 accumulate) for
// the small weight-streaming products of the decode step (W_DKV, W_UK, W_UV).
//
// Fragment convention used here: in a 32-wide slice of the reduction index k,
// the thread with (group g = lane / 4, quad q = lane % 4) owns the 8 consecutive
// k values [8q, 8q + 8).  Because k is summed over, any fixed assignment of k
// values to the instruction's fragment slots gives the same product as long as
// A and B use the same one; this one lets every thread load its A row and B
// column pieces as single 16-byte vectors.  A 32-wide slice is two
// m16n8k16 steps: step 0 takes k = 8q + {0,1,2,3}, step 1 k = 8q + {4,5,6,7}.
#pragma once

#include <stdint.h>

namespace mla {

// D (16x8 fp32) += A (16x16 bf16) * B (16x8 bf16)
__device__ __forceinline__ void mma_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 32-wide k slice: A rows g and g+8 (16 bytes each: ra, rb), B column g
// (16 bytes: cb) -> d (fragment of the 16x8 tile) += A B.
__device__ __forceinline__ void mma_k32(float* d, const uint4& ra, const uint4& rb, const uint4& cb) {
  mma_16816(d, ra.x, rb.x, ra.y, rb.y, cb.x, cb.y);
  mma_16816(d, ra.z, rb.z, ra.w, rb.w, cb.z, cb.w);
}

}  // namespace mla
