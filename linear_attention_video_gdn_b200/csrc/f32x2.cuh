// Packed fp32 pairs for the sm_100 paired FMA (fma.rn.f32x2): two fused
// multiply-adds in one instruction, each lane rounded as fmaf.
#pragma once

#include <stdint.h>

namespace gdn {

__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; }

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

}  // namespace gdn
