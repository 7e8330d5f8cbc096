// Matrix-vector (and skinny matrix-matrix) products against packed int4 / int2 weights.
//
// Whetstone README, "The one fact that shapes everything": at batch 1 every weight is
// read from memory once and used for one multiply-add, so the kernel is bound by the
// bytes it streams (tok/s ceiling = bandwidth / bytes per token). The packed codes are
// the only large traffic; they are streamed once with 16-byte read-only loads that do
// not allocate in L1, dequantised in registers, and never written back as fp16.
//
// Arithmetic per 32-bit word of codes (int4: 8 codes): two masks pick one nibble of each
// 16-bit half, OR-ed with the binary16 pattern of 1024 (0x6400), giving the binary16
// numbers 1024 + q or 1024 + 16 q (one LOP3 each). One packed binary16 subtract of
// 1024 + z (or 1024 + 16 z) leaves q - z (or 16 (q - z)) exactly. Each of those times
// an fp16 activation is exact in binary32 (at most 19 significant bits), and a mixed
// fma.rn.f32.f16 adds it to a binary32 accumulator; the 16x lanes go to a second
// accumulator that is scaled by 1/16 (exact) at the end of the chunk. So the only
// roundings are the binary32 adds, one multiply by the group scale, and the final fp16
// store; a group whose codes all equal its zero point contributes exactly 0.
//
// Work split. A "linear set" is up to WQ_LINEAR_SET_MAX independent matrices run in one
// persistent launch. Each matrix is cut into warp items of 32 / L rows, where L lanes
// share a row (L chosen per K so that every lane streams several 16-byte chunks). Items
// of all matrices are numbered consecutively and dealt round-robin to the warps of the
// grid, so consecutive warps of a CTA work on neighbouring rows of the same matrix.
#include "common.cuh"
#include "gemv.cuh"
#include "host_util.cuh"

namespace wq {

// ---- dequantise-and-multiply of one 16-byte chunk of codes ---------------------------

// int4: chunk = 4 words = 32 weights, all in one group.  x: the 32 activations (fp16).
template <int MT>
__device__ __forceinline__ void chunk_int4(const uint4 w, const uint16_t* const* xs, int k0,
                                           uint32_t c1, uint32_t c16, float s, float* acc) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  uint32_t d[4][4];  // [word][lane pair]: (q0-z,q4-z), 16(q1-z,q5-z), (q2-z,q6-z), 16(q3-z,q7-z)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = wv[i], v8 = v >> 8;
    d[i][0] = hsub2_u32(lop_and_or(v, 0x000F000Fu, 0x64006400u), c1);
    d[i][1] = hsub2_u32(lop_and_or(v, 0x00F000F0u, 0x64006400u), c16);
    d[i][2] = hsub2_u32(lop_and_or(v8, 0x000F000Fu, 0x64006400u), c1);
    d[i][3] = hsub2_u32(lop_and_or(v8, 0x00F000F0u, 0x64006400u), c16);
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const uint4* xp = reinterpret_cast<const uint4*>(xs[m] + k0);
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 x = ld_reuse_v4(xp + i);  // x[8i .. 8i+7] as (x0,x1) (x2,x3) (x4,x5) (x6,x7)
      a = fma_f16f16_f32(lo16(d[i][0]), lo16(x.x), a);
      a = fma_f16f16_f32(hi16(d[i][0]), lo16(x.z), a);
      a = fma_f16f16_f32(lo16(d[i][2]), lo16(x.y), a);
      a = fma_f16f16_f32(hi16(d[i][2]), lo16(x.w), a);
      b = fma_f16f16_f32(lo16(d[i][1]), hi16(x.x), b);
      b = fma_f16f16_f32(hi16(d[i][1]), hi16(x.z), b);
      b = fma_f16f16_f32(lo16(d[i][3]), hi16(x.y), b);
      b = fma_f16f16_f32(hi16(d[i][3]), hi16(x.w), b);
    }
    acc[m] = fmaf(s, fmaf(b, 0.0625f, a), acc[m]);
  }
}

// int2: chunk = 4 words = 64 weights (half a group). Per word, masks at bit offsets
// 0, 2, 4, 6 (values q, 4q, 16q, 64q) on v and on v >> 8 give codes (j, j + 8).
template <int MT>
__device__ __forceinline__ void chunk_int2(const uint4 w, const uint16_t* const* xs, int k0,
                                           const uint32_t* cz, float s, float* acc) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  constexpr uint32_t kMask[4] = {0x00030003u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
  uint32_t d[4][8];  // [word][j]: lanes (code j, code j+8) for j < 4 from v, j >= 4 from v>>8
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = wv[i], v8 = v >> 8;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      d[i][j] = hsub2_u32(lop_and_or(v, kMask[j], 0x64006400u), cz[j]);
      d[i][j + 4] = hsub2_u32(lop_and_or(v8, kMask[j], 0x64006400u), cz[j]);
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const uint4* xp = reinterpret_cast<const uint4*>(xs[m] + k0);
    float a[4] = {0.f, 0.f, 0.f, 0.f};  // accumulators of the 1x, 4x, 16x, 64x lanes
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 xa = ld_reuse_v4(xp + 2 * i);      // x[16i .. 16i+7]
      const uint4 xb = ld_reuse_v4(xp + 2 * i + 1);  // x[16i+8 .. 16i+15]
      const uint32_t xlo[4] = {xa.x, xa.y, xa.z, xa.w};
      const uint32_t xhi[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // code j (< 8) pairs with x[16i + j]; its partner code j + 8 with x[16i + j + 8]
        const uint16_t xj = (j & 1) ? hi16(xlo[j >> 1]) : lo16(xlo[j >> 1]);
        const uint16_t xj8 = (j & 1) ? hi16(xhi[j >> 1]) : lo16(xhi[j >> 1]);
        a[j & 3] = fma_f16f16_f32(lo16(d[i][j]), xj, a[j & 3]);
        a[j & 3] = fma_f16f16_f32(hi16(d[i][j]), xj8, a[j & 3]);
      }
    }
    const float t = fmaf(a[3], 0.015625f, fmaf(a[2], 0.0625f, fmaf(a[1], 0.25f, a[0])));
    acc[m] = fmaf(s, t, acc[m]);
  }
}

// ---- the persistent set kernel -------------------------------------------------------

// Resident CTAs per SM asked of the compiler for the batch-1 variants (register budget).
#ifndef WQ_GEMV_MIN_BLOCKS
#define WQ_GEMV_MIN_BLOCKS 2
#endif

template <int BITS, int MT, int CAP>
__global__ void __launch_bounds__(kGemvThreads, MT == 1 ? WQ_GEMV_MIN_BLOCKS : 1) gemv_int_set_kernel(const __grid_constant__ SetParamsT<CAP> P) {
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (kGemvThreads / 32);
  int mi = 0;
  for (int item = blockIdx.x * (kGemvThreads / 32) + (threadIdx.x >> 5); item < P.total_items;
       item += warps_total) {
    while (item >= P.m[mi].item_end) ++mi;
    const SetMat& M = P.m[mi];
    const int L2 = M.lanes_log2;
    const int L = 1 << L2;
    const int sub = lane & (L - 1);
    const int n = ((item - M.item_begin) << (5 - L2)) + (lane >> L2);
    const int K = M.K;
    const int cpr = K * BITS / 128;  // 16-byte chunks per row
    const int G = K / kGroup;
    const bool row_ok = n < M.N;

    for (int m0 = 0; m0 < M.M; m0 += MT) {
      float acc[MT];
      const uint16_t* xs[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        acc[m] = 0.f;
        xs[m] = M.x + (size_t)min(m0 + m, M.M - 1) * M.ldx;  // ragged tail reuses a row
      }
      if (row_ok) {
        const uint4* crow = reinterpret_cast<const uint4*>(M.codes) + (size_t)n * cpr;
        const uint16_t* srow = M.scale + (size_t)n * G;
        const uint16_t* zrow = M.zero + (size_t)n * G;
        // This lane's chunks are sub, sub + L, sub + 2L, ... (nc of them). Two register
        // batches of four chunks (codes + the group's scale and zero) alternate: the next
        // batch's loads are issued before the current batch is computed, so every warp
        // keeps four 16-byte loads in flight while it does arithmetic.
        const int nc = (cpr - sub + L - 1) >> L2;
        constexpr int CPG = kGroup * BITS / 128;  // 16-byte chunks per group
        uint4 w0[4], w1[4];
        uint16_t s0[4], s1[4], z0[4], z1[4];
        auto load4 = [&](uint4 (&w)[4], uint16_t (&sb)[4], uint16_t (&zb)[4], int j0) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (j0 + u < nc) {
              const int cc = sub + (j0 + u) * L;
              w[u] = ld_stream_v4(crow + cc);
              sb[u] = ld_u16(srow + cc / CPG);
              zb[u] = ld_u16(zrow + cc / CPG);
            }
          }
        };
        auto run4 = [&](const uint4 (&w)[4], const uint16_t (&sb)[4], const uint16_t (&zb)[4], int j0) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (j0 + u < nc) {
              const int cc = sub + (j0 + u) * L;
              const float sf = __half2float(__ushort_as_half(sb[u]));
              const __half z = __ushort_as_half(zb[u]);
              if (BITS == 4) {
                const uint32_t c1 = pack_h2(__hadd(z, __float2half(1024.f)));
                const uint32_t c16 = pack_h2(__hfma(z, __float2half(16.f), __float2half(1024.f)));
                chunk_int4<MT>(w[u], xs, cc * 32, c1, c16, sf, acc);
              } else {
                uint32_t cz[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  cz[j] = pack_h2(__hfma(z, __float2half((float)(1 << (2 * j))), __float2half(1024.f)));
                chunk_int2<MT>(w[u], xs, cc * 64, cz, sf, acc);
              }
            }
          }
        };
        load4(w0, s0, z0, 0);
        for (int j0 = 0; j0 < nc; j0 += 8) {
          load4(w1, s1, z1, j0 + 4);
          run4(w0, s0, z0, j0);
          load4(w0, s0, z0, j0 + 8);
          run4(w1, s1, z1, j0 + 4);
        }
      }
      // split-K reduction over the L lanes of a row (warp shuffles), then one fp16 store
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        for (int o = L >> 1; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
      }
      if (row_ok && sub == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m0 + m < M.M) M.y[(size_t)(m0 + m) * M.ldy + n] = __half_as_ushort(__float2half_rn(acc[m]));
      }
    }
  }
}

// ---- ternary (first version: per-byte base-3 digit extraction) ----------------------

template <int MT, int CAP>
__global__ void __launch_bounds__(kGemvThreads) gemv_ternary_set_kernel(const __grid_constant__ SetParamsT<CAP> P) {
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (kGemvThreads / 32);
  int mi = 0;
  for (int item = blockIdx.x * (kGemvThreads / 32) + (threadIdx.x >> 5); item < P.total_items;
       item += warps_total) {
    while (item >= P.m[mi].item_end) ++mi;
    const SetMat& M = P.m[mi];
    const int n = item - M.item_begin;  // one row per warp item
    const int K = M.K, G = K / kGroup;
    const int row_bytes = kTernaryGroupBytes * G;
    const uint8_t* prow = reinterpret_cast<const uint8_t*>(M.codes) + (size_t)n * row_bytes;
    for (int m0 = 0; m0 < M.M; m0 += MT) {
      float acc[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] = 0.f;
      for (int b = lane; b < row_bytes; b += 32) {
        uint32_t byte = prow[b];
        const int g = b / kTernaryGroupBytes, p = b - g * kTernaryGroupBytes;
        const float s = __half2float(__ushort_as_half(ld_u16(M.scale + (size_t)n * G + g)));
        float t[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          const uint32_t q3 = (byte * 171u) >> 9;  // byte / 3 for byte < 512
          t[i] = (float)(int)(byte - 3u * q3) - 1.f;
          byte = q3;
        }
        const int kb = g * kGroup + 5 * p;
        const int nt = min(5, kGroup - 5 * p);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint16_t* x = M.x + (size_t)min(m0 + m, M.M - 1) * M.ldx + kb;
          float part = 0.f;
          for (int i = 0; i < nt; ++i) part = fmaf(__half2float(__ushort_as_half(x[i])), t[i], part);
          acc[m] = fmaf(s, part, acc[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m0 + m < M.M) M.y[(size_t)(m0 + m) * M.ldy + n] = __half_as_ushort(__float2half_rn(acc[m]));
      }
    }
  }
}

// ---- host-side planning and launch ---------------------------------------------------

int gemv_lanes_log2(int fmt, int64_t K) {
  if (fmt == 2) return 5;  // ternary: one row per warp
  const int64_t cpr = K * (fmt == 0 ? 4 : 2) / 128;
  int l2 = 5;
  while (l2 > 0 && cpr < 4 * (1 << l2)) --l2;  // at least ~4 chunks per lane
  return l2;
}

static int grid_for(const void* kernel, int total_items) {
  const int sms = device_sm_count() > 0 ? device_sm_count() : 1;
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kGemvThreads, 0);
  if (per_sm < 1) per_sm = 1;
  const int need = (total_items + kGemvThreads / 32 - 1) / (kGemvThreads / 32);
  return need < sms * per_sm ? need : sms * per_sm;
}

template <int BITS, int MT, int CAP>
static cudaError_t launch_int(const SetParamsT<CAP>& p, cudaStream_t stream) {
  const void* k = (const void*)gemv_int_set_kernel<BITS, MT, CAP>;
  gemv_int_set_kernel<BITS, MT, CAP><<<grid_for(k, p.total_items), kGemvThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

template <int MT, int CAP>
static cudaError_t launch_ternary(const SetParamsT<CAP>& p, cudaStream_t stream) {
  const void* k = (const void*)gemv_ternary_set_kernel<MT, CAP>;
  gemv_ternary_set_kernel<MT, CAP><<<grid_for(k, p.total_items), kGemvThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

template <int CAP>
static cudaError_t launch_cap(const SetParamsT<CAP>& p, int fmt, int max_m, cudaStream_t stream) {
  const bool multi = max_m > 1;
  if (fmt == 0) return multi ? launch_int<4, 4, CAP>(p, stream) : launch_int<4, 1, CAP>(p, stream);
  if (fmt == 1) return multi ? launch_int<2, 4, CAP>(p, stream) : launch_int<2, 1, CAP>(p, stream);
  return multi ? launch_ternary<4, CAP>(p, stream) : launch_ternary<1, CAP>(p, stream);
}

cudaError_t launch_gemv_set(const SetParams& p, int fmt, int max_m, cudaStream_t stream) {
  if (p.count == 1) {  // a single matrix: a one-entry parameter block
    SetParamsT<1> p1;
    p1.count = 1;
    p1.total_items = p.total_items;
    p1.m[0] = p.m[0];
    return launch_cap<1>(p1, fmt, max_m, stream);
  }
  return launch_cap<kSetMax>(p, fmt, max_m, stream);
}

}  // namespace wq
