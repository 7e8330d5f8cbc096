// Quantisers: group-128 int4 / int3 / int2 asymmetric round-to-nearest, ternary absmean, and
// hierarchical int4 with group-32 indices against a per-row fp16 pair.
//
// Whetstone README, "What the weights can actually survive": round-to-nearest with group
// 128 and one fp16 scale plus one fp16 zero per group (format table rows "int4 g128",
// "int2 g128"), and a ternary g128 row; TKintegers K5, "What is K5?": five trits per byte.
// The arithmetic is float64 with correctly rounded division, rint (ties to even) and a
// direct float64 -> binary16 conversion, so that the codes and metadata are bit-identical
// to the float64 definition in wq.h. This file is compiled with --fmad=false: no
// expression may be contracted into a fused multiply-add.
//
// Data layout: one warp per (row, group). Lane l reads w[4l .. 4l+3] of the group (one
// coalesced 512-byte read per warp) and produces those four codes.
#include "common.cuh"

namespace wq {

__device__ __forceinline__ uint16_t f64_to_f16_bits(double v) {
  return __half_as_ushort(__double2half(v));  // cvt.rn.f16.f64: one rounding, ties to even
}
__device__ __forceinline__ double f16_bits_to_f64(uint16_t b) {
  return (double)__half2float(__ushort_as_half(b));  // exact widening
}

template <int BITS>
__global__ void __launch_bounds__(256) quantize_int_kernel(const float* __restrict__ W, int64_t N,
                                                           int64_t K, uint32_t* __restrict__ codes,
                                                           uint16_t* __restrict__ scale,
                                                           uint16_t* __restrict__ zero) {
  const int lane = threadIdx.x & 31;
  const int64_t G = K / kGroup;
  const int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (task >= N * G) return;
  const int64_t n = task / G, g = task - n * G;

  const float4 v = *reinterpret_cast<const float4*>(W + n * K + g * kGroup + 4 * lane);
  float lo = fminf(fminf(v.x, v.y), fminf(v.z, v.w));
  float hi = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  constexpr double Q = (double)((1 << BITS) - 1);
  const double dlo = (double)lo, dhi = (double)hi;
  uint16_t s_bits = f64_to_f16_bits((dhi - dlo) / Q);
  double s = f16_bits_to_f64(s_bits);
  if (s == 0.0) {
    s = 1.0;
    s_bits = 0x3C00;
  }
  const double z = fmin(fmax(rint(-dlo / s), 0.0), Q);

  const float wv[4] = {v.x, v.y, v.z, v.w};
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double q = fmin(fmax(rint((double)wv[i] / s) + z, 0.0), Q);
    packed |= (uint32_t)q << (BITS * i);
  }
  if (BITS == 3) {
    // lane l holds codes 4l..4l+3: bits 12l..12l+11 of the group's 384-bit stream (12
    // words); a lane whose 12 bits cross a word boundary contributes to two words
    const int off = (12 * lane) & 31, w0 = (12 * lane) >> 5;
    const uint32_t lo = packed << off, hi = off > 20 ? packed >> (32 - off) : 0u;
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < 12; ++j) {
      const uint32_t part = (w0 == j ? lo : 0u) | (w0 + 1 == j ? hi : 0u);
      const uint32_t word = __reduce_or_sync(0xffffffffu, part);
      if (lane == j) mine = word;
    }
    if (lane < 12) codes[n * (3 * K / 32) + g * 12 + lane] = mine;
  } else if (BITS == 4) {
    // lanes 2j and 2j+1 hold codes 8j..8j+3 and 8j+4..8j+7 of word j
    packed <<= 16 * (lane & 1);
    packed |= __shfl_xor_sync(0xffffffffu, packed, 1);
    if ((lane & 1) == 0) codes[n * (K / 8) + g * 16 + (lane >> 1)] = packed;
  } else {
    // lanes 4j..4j+3 hold codes 16j..16j+15 of word j, 4 codes (8 bits) each
    packed <<= 8 * (lane & 3);
    packed |= __shfl_xor_sync(0xffffffffu, packed, 1);
    packed |= __shfl_xor_sync(0xffffffffu, packed, 2);
    if ((lane & 3) == 0) codes[n * (K / 16) + g * 8 + (lane >> 2)] = packed;
  }
  if (lane == 0) {
    scale[task] = s_bits;
    zero[task] = f64_to_f16_bits(z) & 0x7FFFu;  // small integer: exact; no negative zero
  }
}

__global__ void __launch_bounds__(256) quantize_ternary_kernel(const float* __restrict__ W,
                                                               int64_t N, int64_t K,
                                                               uint8_t* __restrict__ packed,
                                                               uint16_t* __restrict__ scale) {
  __shared__ float s_abs[8][kGroup];
  __shared__ uint8_t s_dig[8][kTernaryGroupBytes * 5];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t G = K / kGroup;
  const int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + wid;
  if (task >= N * G) return;  // whole warps exit together: task is warp-uniform
  const int64_t n = task / G, g = task - n * G;

  const float4 v = *reinterpret_cast<const float4*>(W + n * K + g * kGroup + 4 * lane);
  const float wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) s_abs[wid][4 * lane + i] = fabsf(wv[i]);
  __syncwarp();
  // absmean: the float64 sum is taken strictly left to right (its rounding depends on
  // the order), so one lane does it; the group is 128 adds and this kernel is offline.
  double a = 0.0;
  if (lane == 0) {
    for (int k = 0; k < kGroup; ++k) a = __dadd_rn(a, (double)s_abs[wid][k]);
  }
  a = __shfl_sync(0xffffffffu, a, 0);
  uint16_t s_bits = f64_to_f16_bits(a / (double)kGroup);
  double s = f16_bits_to_f64(s_bits);
  if (s == 0.0) {
    s = 1.0;
    s_bits = 0x3C00;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double t = fmin(fmax(rint((double)wv[i] / s), -1.0), 1.0);
    s_dig[wid][4 * lane + i] = (uint8_t)(int)(t + 1.0);  // base-3 digit 0, 1, 2
  }
  if (lane < 2) s_dig[wid][kGroup + lane] = 1;  // two pad trits of value 0
  __syncwarp();
  if (lane < kTernaryGroupBytes) {
    const uint8_t* d = &s_dig[wid][5 * lane];
    const uint32_t byte = d[0] + 3u * d[1] + 9u * d[2] + 27u * d[3] + 81u * d[4];
    packed[n * (kTernaryGroupBytes * G) + g * kTernaryGroupBytes + lane] = (uint8_t)byte;
  }
  if (lane == 0) scale[task] = s_bits;
}

// Hierarchical int4, group 32 (Whetstone README, "What the weights can actually survive":
// two 4-bit indices per group of 32 against one fp16 pair per row; "New in 0.6.0": the row
// scale must not underflow to zero). The definition is per row (the pair depends on every
// group of the row), so one warp takes one row in two passes: the row maxima of s_g and m_g,
// then the indices and codes. Each pass reads 128 weights (four groups) per iteration;
// lanes 8j .. 8j+7 hold group j of the iteration, four weights each.

// rs(v) of the int4h definition: fp16(v / 15), 1 for v = 0, the smallest positive binary16
// where a positive v rounds to zero.
__device__ __forceinline__ uint16_t row_scale_bits(double v) {
  if (v == 0.0) return 0x3C00;
  const uint16_t b = f64_to_f16_bits(v / 15.0);
  return b == 0 ? (uint16_t)0x0001 : b;
}

// lo and hi of the 32 weights held by a lane's group of eight lanes (four each)
__device__ __forceinline__ void group32_minmax(const float4 v, float& lo, float& hi) {
  lo = fminf(fminf(v.x, v.y), fminf(v.z, v.w));
  hi = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
}

__global__ void __launch_bounds__(256) quantize_int4h_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                                             uint32_t* __restrict__ codes,
                                                             uint16_t* __restrict__ pair,
                                                             uint8_t* __restrict__ idx) {
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= N) return;  // warp-uniform
  const float* row = W + n * K;
  const int iters = (int)(K / 128);

  // pass 1: max_g s_g and max_g m_g (maxima are exact in any order)
  double smax = 0.0, mmax = 0.0;
  for (int it = 0; it < iters; ++it) {
    const float4 v = *reinterpret_cast<const float4*>(row + 128 * it + 4 * lane);
    float lo, hi;
    group32_minmax(v, lo, hi);
    const double m = fmax(0.0, -(double)lo);
    const double sg = ((double)hi + m) / 15.0;
    smax = fmax(smax, sg);
    mmax = fmax(mmax, m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    smax = fmax(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    mmax = fmax(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
  }
  const uint16_t d_bits = row_scale_bits(smax), dm_bits = row_scale_bits(mmax);
  const double d = f16_bits_to_f64(d_bits), dm = f16_bits_to_f64(dm_bits);

  // pass 2: indices and codes
  for (int it = 0; it < iters; ++it) {
    const float4 v = *reinterpret_cast<const float4*>(row + 128 * it + 4 * lane);
    float lo, hi;
    group32_minmax(v, lo, hi);
    const double m = fmax(0.0, -(double)lo);
    const double sg = ((double)hi + m) / 15.0;
    const double a = fmin(fmax(rint(sg / d), 0.0), 15.0);
    const double b = fmin(fmax(rint(m / dm), 0.0), 15.0);
    const double S = d * a, Z = dm * b;  // exact: a binary16 value times a 4-bit integer
    const float wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double q = S > 0.0 ? fmin(fmax(rint(((double)wv[i] + Z) / S), 0.0), 15.0) : 0.0;
      packed |= (uint32_t)q << (4 * i);
    }
    // lanes 2j and 2j+1 hold codes 8j..8j+3 and 8j+4..8j+7 of the iteration's word j
    packed <<= 16 * (lane & 1);
    packed |= __shfl_xor_sync(0xffffffffu, packed, 1);
    if ((lane & 1) == 0) codes[n * (K / 8) + 16 * it + (lane >> 1)] = packed;
    if ((lane & 7) == 0) idx[n * (K / 32) + 4 * it + (lane >> 3)] = (uint8_t)((uint32_t)a | (uint32_t)b << 4);
  }
  if (lane == 0) {
    pair[2 * n] = d_bits;
    pair[2 * n + 1] = dm_bits;
  }
}

cudaError_t launch_quantize(const float* W, int64_t N, int64_t K, int fmt, void* codes,
                            uint16_t* scale, uint16_t* zero, cudaStream_t stream) {
  if (fmt == 4) {  // int4h: one warp per row
    quantize_int4h_kernel<<<(unsigned)((N + 7) / 8), 256, 0, stream>>>(W, N, K, (uint32_t*)codes, scale,
                                                                      reinterpret_cast<uint8_t*>(zero));
    return cudaGetLastError();
  }
  const int64_t tasks = N * (K / kGroup);
  const int64_t blocks = (tasks + 7) / 8;
  if (fmt == 0)
    quantize_int_kernel<4><<<(unsigned)blocks, 256, 0, stream>>>(W, N, K, (uint32_t*)codes, scale,
                                                                 zero);
  else if (fmt == 1)
    quantize_int_kernel<2><<<(unsigned)blocks, 256, 0, stream>>>(W, N, K, (uint32_t*)codes, scale,
                                                                 zero);
  else if (fmt == 3)
    quantize_int_kernel<3><<<(unsigned)blocks, 256, 0, stream>>>(W, N, K, (uint32_t*)codes, scale,
                                                                 zero);
  else
    quantize_ternary_kernel<<<(unsigned)blocks, 256, 0, stream>>>(W, N, K, (uint8_t*)codes, scale);
  return cudaGetLastError();
}

}  // namespace wq
