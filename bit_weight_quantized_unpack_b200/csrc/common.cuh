// Shared device helpers of libwq (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libwq is written for sm_100a (B200) only"
#endif

namespace wq {

constexpr int kGroup = 128;             // weights per quantisation group along K
constexpr int kTernaryGroupBytes = 26;  // 128 trits, five per byte, last byte 3 + 2 pad

// 16-byte streaming load of data read exactly once: read-only path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 16-byte load of data reused by many warps (activations): read-only path, L1 cached.
__device__ __forceinline__ uint4 ld_reuse_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint16_t ld_u16(const uint16_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// acc + a * b with a, b binary16 and acc binary32. The product of two binary16 numbers
// has at most 22 significant bits, so it is exact in binary32; only the add rounds.
__device__ __forceinline__ float fma_f16f16_f32(uint16_t a, uint16_t b, float acc) {
  float d;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(acc));
  return d;
}

__device__ __forceinline__ uint16_t lo16(uint32_t v) { return (uint16_t)(v & 0xFFFFu); }
__device__ __forceinline__ uint16_t hi16(uint32_t v) { return (uint16_t)(v >> 16); }

// Packed binary16 subtract (two lanes), exact for the small integers used here.
__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// (v & mask) | orv as one three-input logic op (truth table 0xEA = (a & b) | c); written out
// because the plain C expression with two constant operands measured as two instructions.
__device__ __forceinline__ uint32_t lop_and_or(uint32_t v, uint32_t mask, uint32_t orv) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(v), "r"(mask), "r"(orv));
  return d;
}

}  // namespace wq

namespace wq {
__device__ __forceinline__ uint32_t prmt_u32(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t pack_h2(__half h) {
  const uint32_t b = __half_as_ushort(h);
  return b | (b << 16);
}
}  // namespace wq
