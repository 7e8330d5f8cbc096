// Matrix-vector product against packed int4 / int2 weights, one weight row per lane.
//
// Whetstone README, "The one fact that shapes everything": at batch 1 every weight is read
// once for one multiply-add, so the product is bound by the bytes streamed from HBM. This
// kernel spends as few instructions per weight as the CUDA cores allow:
//   - each lane owns one whole row and walks it group by group (128 weights), so the warp
//     never reduces across lanes and every lane loads its scale and zero once per group;
//   - a lane keeps the next groups of its row in flight with cp.async 16-byte copies into
//     its own slots of a shared-memory ring (no registers held while they land);
//   - the activation vector of the current matrix is staged once per CTA in shared
//     memory, one fp16 value per 32-bit word (low half), so that every mixed-precision
//     multiply-add reads both of its fp16 operands from the low half of a register;
// Work split: rows of all matrices of a set are laid end to end with their byte cost; CTA
// b processes the rows whose first byte falls in its 1/gridDim share (so every CTA
// streams the same number of bytes), matrix by matrix, its warps taking 32-row units.
//
// Arithmetic per 32-bit word of codes is the one of gemv.cu: binary16 magic numbers give
// q - z exactly, each product with an fp16 activation is exact in binary32, and only the
// binary32 adds, the multiply by the group scale and the final fp16 store round.
#include "common.cuh"
#include "gemv_rows.cuh"
#include "host_util.cuh"

namespace wq {

namespace {

constexpr int THREADS = kRowsThreads;


// x value k of the staged activation vector as an f16 operand (low half of a word).
template <int XM>
__device__ __forceinline__ uint16_t xval(const uint32_t* xs, int k) {
  if (XM == 0) return (uint16_t)xs[k];
  const uint32_t w = xs[k >> 1];
  return (k & 1) ? hi16(w) : lo16(w);
}

// One int4 group (128 weights = 16 words in two sectors) of a row against x[k0 .. k0+127].
// Four accumulators (even / odd words x plain / 16x lanes) keep four independent chains.
// XM selects the staged layout of x: 0 = one fp16 per 32-bit word; 1 = fp16 pairs in
// natural order; 2 = fp16 pairs (x_j, x_j+4) of each group of eight, matching the code
// pairs of one word of codes, so both operands of every multiply sit in the same half.
template <int XM>
__device__ __forceinline__ float group_int4(const uint32_t (&c)[16], const uint32_t* xs, int k0, uint16_t zbits) {
  const __half z = __ushort_as_half(zbits);
  const uint32_t c1 = pack_h2(__hadd(z, __float2half(1024.f)));
  const uint32_t c16 = pack_h2(__hfma(z, __float2half(16.f), __float2half(1024.f)));
  float a[2] = {0.f, 0.f}, b[2] = {0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t v = c[i], v8 = v >> 8;
    const uint32_t d0 = hsub2_u32(lop_and_or(v, 0x000F000Fu, 0x64006400u), c1);    // q0, q4
    const uint32_t d1 = hsub2_u32(lop_and_or(v, 0x00F000F0u, 0x64006400u), c16);   // 16 q1, 16 q5
    const uint32_t d2 = hsub2_u32(lop_and_or(v8, 0x000F000Fu, 0x64006400u), c1);   // q2, q6
    const uint32_t d3 = hsub2_u32(lop_and_or(v8, 0x00F000F0u, 0x64006400u), c16);  // 16 q3, 16 q7
    float& A = a[i & 1];
    float& B = b[i & 1];
    if (XM == 2) {  // one 16-byte load: (x0,x4) (x1,x5) (x2,x6) (x3,x7)
      const uint4 w = reinterpret_cast<const uint4*>(xs + k0 / 2)[i];
      A = fma_f16f16_f32(lo16(d0), lo16(w.x), A);
      A = fma_f16f16_f32(hi16(d0), hi16(w.x), A);
      A = fma_f16f16_f32(lo16(d2), lo16(w.z), A);
      A = fma_f16f16_f32(hi16(d2), hi16(w.z), A);
      B = fma_f16f16_f32(lo16(d1), lo16(w.y), B);
      B = fma_f16f16_f32(hi16(d1), hi16(w.y), B);
      B = fma_f16f16_f32(lo16(d3), lo16(w.w), B);
      B = fma_f16f16_f32(hi16(d3), hi16(w.w), B);
      continue;
    }
    uint16_t x[8];
    if (XM == 0) {  // two 16-byte shared loads: x[k .. k+3], x[k+4 .. k+7], one per 32-bit word
      const uint4 lo = reinterpret_cast<const uint4*>(xs + k0)[2 * i];
      const uint4 hi = reinterpret_cast<const uint4*>(xs + k0)[2 * i + 1];
      x[0] = lo16(lo.x); x[1] = lo16(lo.y); x[2] = lo16(lo.z); x[3] = lo16(lo.w);
      x[4] = lo16(hi.x); x[5] = lo16(hi.y); x[6] = lo16(hi.z); x[7] = lo16(hi.w);
    } else {        // one 16-byte shared load of four fp16x2 words
      const uint4 w = reinterpret_cast<const uint4*>(xs + k0 / 2)[i];
      x[0] = lo16(w.x); x[1] = hi16(w.x); x[2] = lo16(w.y); x[3] = hi16(w.y);
      x[4] = lo16(w.z); x[5] = hi16(w.z); x[6] = lo16(w.w); x[7] = hi16(w.w);
    }
    A = fma_f16f16_f32(lo16(d0), x[0], A);
    A = fma_f16f16_f32(hi16(d0), x[4], A);
    A = fma_f16f16_f32(lo16(d2), x[2], A);
    A = fma_f16f16_f32(hi16(d2), x[6], A);
    B = fma_f16f16_f32(lo16(d1), x[1], B);
    B = fma_f16f16_f32(hi16(d1), x[5], B);
    B = fma_f16f16_f32(lo16(d3), x[3], B);
    B = fma_f16f16_f32(hi16(d3), x[7], B);
  }
  return fmaf(b[0] + b[1], 0.0625f, a[0] + a[1]);
}

// One int2 group (128 weights = 8 words in one sector).
template <int XM>
__device__ __forceinline__ float group_int2(const uint32_t (&c)[8], const uint32_t* xs, int k0, uint16_t zbits) {
  const __half z = __ushort_as_half(zbits);
  constexpr uint32_t kMask[4] = {0x00030003u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
  uint32_t cz[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) cz[j] = pack_h2(__hfma(z, __float2half((float)(1 << (2 * j))), __float2half(1024.f)));
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t v = c[i], v8 = v >> 8;
    const int k = k0 + 16 * i;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // lanes of d: codes j and j + 8 of the word, scaled by 4^(j & 3)
      const uint32_t d = hsub2_u32(lop_and_or(j < 4 ? v : v8, kMask[j & 3], 0x64006400u), cz[j & 3]);
      a[j & 3] = fma_f16f16_f32(lo16(d), xval<XM>(xs, k + j), a[j & 3]);
      a[j & 3] = fma_f16f16_f32(hi16(d), xval<XM>(xs, k + j + 8), a[j & 3]);
    }
  }
  return fmaf(a[3], 0.015625f, fmaf(a[2], 0.0625f, fmaf(a[1], 0.25f, a[0])));
}

}  // namespace

// Shared memory of one CTA: the staged activations (K words, see xval) followed by the
// per-thread code ring: kRowsStages slots x (group bytes) for each of the 256 threads,
// laid out [slot][16-byte chunk][thread] so that a warp's 16-byte accesses are contiguous.
template <int BITS>
__device__ __forceinline__ uint4* ring_chunk(uint4* ring, int slot, int chunk) {
  constexpr int CH = kGroup * BITS / 8 / 16;  // 16-byte chunks per group: 4 (int4) / 2 (int2)
  return ring + ((size_t)(slot * CH + chunk) * THREADS + threadIdx.x);
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

#ifndef WQ_ROWS_XMODE
#define WQ_ROWS_XMODE 1
#endif
#ifndef WQ_ROWS_MIN_BLOCKS
#define WQ_ROWS_MIN_BLOCKS 3
#endif

template <int BITS, int XM, int CAP>
__global__ void __launch_bounds__(THREADS, WQ_ROWS_MIN_BLOCKS) gemv_rows_kernel(const __grid_constant__ RowParamsT<CAP> P) {
  extern __shared__ __align__(16) uint32_t smem[];
  const int64_t share = (P.total_cost + gridDim.x - 1) / gridDim.x;
  const int64_t lo = share * blockIdx.x, hi = lo + share;
  constexpr int GB = kGroup * BITS / 8;     // bytes of codes per group: 64 (int4) / 32 (int2)
  constexpr int CH = GB / 16;
  constexpr int S = kRowsStages;
  uint4* ring = reinterpret_cast<uint4*>(smem);
  uint32_t* xs = smem + S * CH * THREADS * 4;

  for (int mi = 0; mi < P.count; ++mi) {
    const RowMat& M = P.m[mi];
    // matrices are in cost order: skip those before this CTA's share, stop after it
    if (M.cost_begin + (int64_t)M.N * M.row_cost <= lo) continue;
    if (M.cost_begin >= hi) break;
    const int64_t rc = M.row_cost;
    // rows whose starting cost lies in [lo, hi)
    const int64_t r_lo = lo <= M.cost_begin ? 0 : (lo - M.cost_begin + rc - 1) / rc;
    const int64_t r_hi64 = hi <= M.cost_begin ? 0 : (hi - M.cost_begin + rc - 1) / rc;
    const int r_hi = (int)(r_hi64 < M.N ? r_hi64 : M.N);
    if (r_lo >= r_hi) continue;
    const int K = M.K, G = K / kGroup;

    // stage x of this matrix
    __syncthreads();
    for (int k8 = threadIdx.x; k8 < K / 8; k8 += THREADS) {
      const uint4 v = *reinterpret_cast<const uint4*>(M.x + 8 * k8);
      if (XM == 0) {
        reinterpret_cast<uint4*>(xs)[2 * k8] = make_uint4(v.x & 0xFFFFu, v.x >> 16, v.y & 0xFFFFu, v.y >> 16);
        reinterpret_cast<uint4*>(xs)[2 * k8 + 1] = make_uint4(v.z & 0xFFFFu, v.z >> 16, v.w & 0xFFFFu, v.w >> 16);
      } else if (XM == 2) {  // (x0,x4) (x1,x5) (x2,x6) (x3,x7)
        reinterpret_cast<uint4*>(xs)[k8] = make_uint4(prmt_u32(v.x, v.z, 0x5410), prmt_u32(v.x, v.z, 0x7632),
                                                      prmt_u32(v.y, v.w, 0x5410), prmt_u32(v.y, v.w, 0x7632));
      } else {
        reinterpret_cast<uint4*>(xs)[k8] = v;
      }
    }
    __syncthreads();

    // 32-row units dealt to the warps: a matrix boundary idles at most 31 lanes
    const int nunits = (int)((r_hi - r_lo + 31) >> 5);
    for (int u = threadIdx.x >> 5; u < nunits; u += THREADS / 32) {
      const int n = (int)r_lo + 32 * u + (threadIdx.x & 31);
      if (n >= r_hi) continue;
      const uint8_t* crow = reinterpret_cast<const uint8_t*>(M.codes) + (size_t)n * (K * BITS / 8);
      const uint16_t* srow = M.scale + (size_t)n * G;
      const uint16_t* zrow = M.zero + (size_t)n * G;
      // prologue: groups 0 .. S-2 in flight (one commit group each, empty ones past G)
#pragma unroll
      for (int g = 0; g < S - 1; ++g) {
        if (g < G) {
#pragma unroll
          for (int ch = 0; ch < CH; ++ch) cp_async16(ring_chunk<BITS>(ring, g, ch), crow + (size_t)g * GB + 16 * ch);
        }
        cp_async_commit();
      }
      // scale and zero of the next group, in separate registers until used (combining them
      // right after the loads would stall the lane for the load latency)
      uint16_t s_next = ld_u16(srow), z_next = ld_u16(zrow);
      float acc = 0.f;
      for (int g = 0; g < G; ++g) {
        // keep S-1 groups in flight: issue group g + S - 1, then wait for group g
        const int gi = g + S - 1;
        if (gi < G) {
#pragma unroll
          for (int ch = 0; ch < CH; ++ch)
            cp_async16(ring_chunk<BITS>(ring, gi % S, ch), crow + (size_t)gi * GB + 16 * ch);
        }
        cp_async_commit();
        const uint16_t sc = s_next, zc = z_next;
        if (g + 1 < G) {
          s_next = ld_u16(srow + g + 1);
          z_next = ld_u16(zrow + g + 1);
        }
        cp_async_wait<S - 1>();
        uint32_t c[GB / 4];
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
          const uint4 v = *ring_chunk<BITS>(ring, g % S, ch);
          c[4 * ch + 0] = v.x;
          c[4 * ch + 1] = v.y;
          c[4 * ch + 2] = v.z;
          c[4 * ch + 3] = v.w;
        }
        float part;
        if constexpr (BITS == 4) part = group_int4<XM>(c, xs, g * kGroup, zc);
        else part = group_int2<XM>(c, xs, g * kGroup, zc);
        acc = fmaf(__half2float(__ushort_as_half(sc)), part, acc);
      }
      cp_async_wait<0>();
      M.y[n] = __half_as_ushort(__float2half_rn(acc));
    }
  }
}

// ---- host side -----------------------------------------------------------------------

bool rows_plan(RowParams& p, int bits, int count, const RowMatDesc* d, int* max_k) {
  int64_t cost = 0;
  int mk = 0;
  for (int i = 0; i < count; ++i) {
    RowMat& m = p.m[i];
    m.codes = d[i].codes;
    m.scale = d[i].scale;
    m.zero = d[i].zero;
    m.x = d[i].x;
    m.y = d[i].y;
    m.N = (int)d[i].N;
    m.K = (int)d[i].K;
    m.row_cost = d[i].K * bits / 8 + 4 * (d[i].K / kGroup);
    m.cost_begin = cost;
    cost += (int64_t)m.N * m.row_cost;
    if (m.K > mk) mk = m.K;
  }
  p.count = count;
  p.total_cost = cost;
  *max_k = mk;
  return kRowsStages * (kGroup * bits / 8) * kRowsThreads + (int64_t)mk * 4 <= kRowsMaxSmem;
}

template <int BITS, int XM, int CAP>
static cudaError_t launch_cap(const RowParamsT<CAP>& p, int max_k, cudaStream_t stream) {
  const int smem = kRowsStages * (kGroup * BITS / 8) * THREADS + max_k * (XM == 0 ? 4 : 2);
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(gemv_rows_kernel<BITS, XM, CAP>, kRowsMaxSmem, configured);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  if (sms == 0) return cudaErrorInvalidDevice;
  gemv_rows_kernel<BITS, XM, CAP><<<WQ_ROWS_MIN_BLOCKS * sms, THREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int BITS, int XM>
static cudaError_t launch_t(const RowParams& p, int max_k, cudaStream_t stream) {
  if (p.count == 1) {
    RowParamsT<1> p1;
    p1.total_cost = p.total_cost;
    p1.count = 1;
    p1.m[0] = p.m[0];
    return launch_cap<BITS, XM, 1>(p1, max_k, stream);
  }
  return launch_cap<BITS, XM, kRowsMaxMats>(p, max_k, stream);
}

cudaError_t launch_gemv_rows(const RowParams& p, int bits, int max_k, cudaStream_t stream) {
  // x layout in shared memory: int4 pairs x with the code pairs of a word (mode 2); int2
  // codes pair (j, j + 8), so int2 uses the natural fp16-pair layout (mode 1)
  return bits == 4 ? launch_t<4, WQ_ROWS_XMODE>(p, max_k, stream) : launch_t<2, (WQ_ROWS_XMODE == 0 ? 0 : 1)>(p, max_k, stream);
}

}  // namespace wq
