// Products with int3 g128 weights (3-bit codes in each row's little-endian bit stream),
// Y[m, n] = sum_k X[m, k] * w_hat[n, k], for a set of matrices and any M.
//
// Whetstone README, format table row "int3 g128" (3.25 bits/weight): the same asymmetric
// round-to-nearest groups of 128 with an fp16 scale and integer zero point, three bits per
// code. A code no longer sits inside one 32-bit word, so the unit of work is three words:
// 96 bits = 32 codes, always inside one group (a group is four units, 12 words). Lane l of
// a warp takes units l, l + 32, ... of one row; code i of a unit sits at bit 3i of the
// unit's three words (codes 10 and 21 straddle two words), extracted with compile-time
// shifts. (q - z) x is exact in fp32; each unit's sum is scaled by s; a warp reduction
// gives the row's output. One warp per output row (an item); tokens in blocks of 8.
#include <climits>

#include "common.cuh"
#include "gemv.cuh"
#include "host_util.cuh"

namespace wq {

namespace {

constexpr int kInt3Threads = 256;
constexpr int kInt3TokBlock = 8;

template <int I>
__device__ __forceinline__ uint32_t code3(uint32_t w0, uint32_t w1, uint32_t w2) {
  constexpr int b = 3 * I;
  if constexpr (b + 3 <= 32) {
    return (w0 >> b) & 7u;
  } else if constexpr (b < 32) {
    return ((w0 >> b) | (w1 << (32 - b))) & 7u;
  } else if constexpr (b + 3 <= 64) {
    return (w1 >> (b - 32)) & 7u;
  } else if constexpr (b < 64) {
    return ((w1 >> (b - 32)) | (w2 << (64 - b))) & 7u;
  } else {
    return (w2 >> (b - 64)) & 7u;
  }
}

template <int I>
__device__ __forceinline__ void unit_dot(uint32_t w0, uint32_t w1, uint32_t w2, float z, const uint4 (&xv)[4],
                                         float& acc) {
  if constexpr (I < 32) {
    const uint4 c = xv[I / 8];
    const uint32_t xw = (I % 8) < 2 ? c.x : (I % 8) < 4 ? c.y : (I % 8) < 6 ? c.z : c.w;
    const uint16_t xh = (I % 2) ? hi16(xw) : lo16(xw);
    const float d = (float)code3<I>(w0, w1, w2) - z;  // an integer in [-7, 7]: exact
    acc = fmaf(d, __half2float(__ushort_as_half(xh)), acc);
    unit_dot<I + 1>(w0, w1, w2, z, xv, acc);
  }
}

template <int CAP>
__device__ __forceinline__ int mat_of_item(const SetParamsT<CAP>& P, int item) {
  int lo = 0, hi = P.count - 1;
  while (lo < hi) {  // last matrix whose item_begin <= item
    const int mid = (lo + hi + 1) >> 1;
    if (P.m[mid].item_begin <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace

template <int CAP>
__global__ void __launch_bounds__(kInt3Threads) gemv_int3_set_kernel(const __grid_constant__ SetParamsT<CAP> P) {
  const int lane = threadIdx.x & 31;
  const int wpb = kInt3Threads / 32;
  for (int item = blockIdx.x * wpb + (threadIdx.x >> 5); item < P.total_items; item += gridDim.x * wpb) {
    const SetMat& m = P.m[mat_of_item(P, item)];
    const int n = item - m.item_begin;
    const int K = m.K, G = K / kGroup, U = K / 32;
    const uint32_t* row = static_cast<const uint32_t*>(m.codes) + (size_t)n * (3 * (K / 32));
    const uint16_t* srow = m.scale + (size_t)n * G;
    const uint16_t* zrow = m.zero + (size_t)n * G;
    for (int m0 = 0; m0 < m.M; m0 += kInt3TokBlock) {
      float acc[kInt3TokBlock];
#pragma unroll
      for (int t = 0; t < kInt3TokBlock; ++t) acc[t] = 0.f;
      for (int u = lane; u < U; u += 32) {
        const uint32_t w0 = row[3 * u], w1 = row[3 * u + 1], w2 = row[3 * u + 2];
        const float s = __half2float(__ushort_as_half(srow[u >> 2]));
        const float z = __half2float(__ushort_as_half(zrow[u >> 2]));
#pragma unroll
        for (int t = 0; t < kInt3TokBlock; ++t) {
          if (m0 + t < m.M) {
            const uint4* xr = reinterpret_cast<const uint4*>(m.x + (size_t)(m0 + t) * m.ldx + 32 * u);
            const uint4 xv[4] = {xr[0], xr[1], xr[2], xr[3]};
            float part = 0.f;
            unit_dot<0>(w0, w1, w2, z, xv, part);
            acc[t] = fmaf(s, part, acc[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kInt3TokBlock; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
        if (lane == 0 && m0 + t < m.M) m.y[(size_t)(m0 + t) * m.ldy + n] = __half_as_ushort(__float2half_rn(acc[t]));
      }
    }
  }
}

cudaError_t launch_gemv_int3(const SetParams& p, cudaStream_t stream) {
  if (p.total_items < 1) return cudaErrorInvalidValue;
  const int sms = device_sm_count();
  if (sms == 0) return cudaErrorInvalidDevice;
  const int wpb = kInt3Threads / 32;
  const int64_t want = ((int64_t)p.total_items + wpb - 1) / wpb;
  const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  gemv_int3_set_kernel<kSetMax><<<grid, kInt3Threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace wq
