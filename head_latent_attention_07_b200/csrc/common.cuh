// Shared device helpers of the MLA decode kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

// ---------------------------------------------------------------- status word
// First error wins; later errors leave the word unchanged.
__device__ __forceinline__ void record_status(int32_t* dev_status, int32_t code) {
  if (dev_status != nullptr) atomicCAS(reinterpret_cast<int*>(dev_status), 0, code);
}

// ---------------------------------------------------------------- bf16 helpers
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
  __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&b);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return uint32_t(f32_to_bf16(lo)) | (uint32_t(f32_to_bf16(hi)) << 16);
}

// 8 bf16 values (one 16-byte vector) widened to fp32.
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// Global load of data read once (cache-streaming); the compiler may schedule
// it freely, so several can be in flight per thread.
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}

// ---------------------------------------------------------------- RoPE
// Rotation of a RoPE channel pair at position pos, inv_freq = theta^(-2i/d) of
// the pair: the angle pos * inv_freq is evaluated in double precision so that
// positions up to 2^31 keep their phase, then reduced modulo 2 pi in double
// precision; the cosine and sine of the remainder (|r| <= pi) are taken in fp32.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float* c, float* s) {
  const double ang = (double)pos * inv_freq;
  const double two_pi = 6.283185307179586476925286766559;
  const double k = rint(ang * (1.0 / two_pi));
  const float r = (float)fma(-k, two_pi, ang);
  sincosf(r, s, c);
}

// Programmatic dependent launch: the next kernel on the stream may start its
// prologue early; every kernel waits for its predecessor's completion (and the
// visibility of its writes) before it reads any input.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependent_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace mla
