// Matrix-vector product against packed int4 / int2 weights, staged through shared memory
// by the bulk-copy (TMA) engine.
//
// Whetstone README, "The one fact that shapes everything": at batch 1 every weight is
// read once for one multiply-add, so the product runs at the speed the packed codes
// stream in from HBM. Keeping ~5 MB in flight across 148 SMs takes deep queues: here one
// producer lane per CTA issues cp.async.bulk copies of whole contiguous row blocks of
// codes (up to 48 KB each, 4 in flight per SM) plus the block's scales and zeros, and
// 12 consumer warps dequantise from shared memory. Consumers never wait on DRAM directly.
//
// Work split. A matrix is cut into row blocks of R = 12 * (32 / L) rows, where L lanes
// share a row and each lane owns a contiguous range of 16-byte chunks of it (so a lane
// crosses group boundaries -- and reloads a scale/zero -- once per 128 weights). Rows
// longer than a stage are streamed as K segments; a lane keeps its partial sum across the
// segments of its row. Row blocks of all matrices of a set are numbered consecutively;
// CTA b takes the blocks whose starting byte offset falls in its 1/gridDim share of the
// total bytes, so every CTA streams nearly the same number of bytes.
//
// Arithmetic per 32-bit word of codes is the one of gemv.cu: binary16 magic numbers give
// q - z exactly, each product with an fp16 activation is exact in binary32, and only the
// binary32 adds, the multiply by the group scale and the final fp16 store round.
#include "common.cuh"
#include "gemv_bulk.cuh"
#include "tc_ptx.cuh"

namespace wq {

namespace {

constexpr int CW = kBulkConsumerWarps;
constexpr int THREADS = 32 * (1 + CW);
constexpr int OFF_META = kBulkStages * kBulkStageBytes;
constexpr int OFF_BAR = OFF_META + 2 * kBulkMetaBytes;
constexpr int SMEM_BYTES = OFF_BAR + 8 * (2 * kBulkStages + 4) + 16;

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Block range of CTA b: the blocks whose first byte lies in [b*C/G, (b+1)*C/G).
__device__ int first_block_at(const BulkParams& P, int64_t target) {
  for (int i = 0; i < P.count; ++i) {
    const BulkMat& m = P.m[i];
    const int64_t end = m.cost_begin + (int64_t)(m.block_end - m.block_begin) * m.block_bytes;
    if (target < end) {
      const int64_t off = target - m.cost_begin;
      const int64_t j = off <= 0 ? 0 : (off + m.block_bytes - 1) / m.block_bytes;
      return m.block_begin + (int)j;
    }
  }
  return P.total_blocks;
}


// int4 chunk (32 weights, one group): two accumulators, the 16x lanes scaled at the end.
__device__ __forceinline__ float dot_chunk_int4(const uint4 w, const uint4* xp, uint32_t c1, uint32_t c16) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = wv[i], v8 = v >> 8;
    const uint32_t d0 = hsub2_u32(lop_and_or(v, 0x000F000Fu, 0x64006400u), c1);
    const uint32_t d1 = hsub2_u32(lop_and_or(v, 0x00F000F0u, 0x64006400u), c16);
    const uint32_t d2 = hsub2_u32(lop_and_or(v8, 0x000F000Fu, 0x64006400u), c1);
    const uint32_t d3 = hsub2_u32(lop_and_or(v8, 0x00F000F0u, 0x64006400u), c16);
    const uint4 x = ld_reuse_v4(xp + i);
    a = fma_f16f16_f32(lo16(d0), lo16(x.x), a);
    a = fma_f16f16_f32(hi16(d0), lo16(x.z), a);
    a = fma_f16f16_f32(lo16(d2), lo16(x.y), a);
    a = fma_f16f16_f32(hi16(d2), lo16(x.w), a);
    b = fma_f16f16_f32(lo16(d1), hi16(x.x), b);
    b = fma_f16f16_f32(hi16(d1), hi16(x.z), b);
    b = fma_f16f16_f32(lo16(d3), hi16(x.y), b);
    b = fma_f16f16_f32(hi16(d3), hi16(x.w), b);
  }
  return fmaf(b, 0.0625f, a);
}

// int2 chunk (64 weights, half a group); cz[j] = 1024 + 4^j z.
__device__ __forceinline__ float dot_chunk_int2(const uint4 w, const uint4* xp, const uint32_t* cz) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  constexpr uint32_t kMask[4] = {0x00030003u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = wv[i], v8 = v >> 8;
    const uint4 xa = ld_reuse_v4(xp + 2 * i), xb = ld_reuse_v4(xp + 2 * i + 1);
    const uint32_t xlo[4] = {xa.x, xa.y, xa.z, xa.w};
    const uint32_t xhi[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t d = hsub2_u32(lop_and_or(j < 4 ? v : v8, kMask[j & 3], 0x64006400u), cz[j & 3]);
      const uint16_t xj = (j & 1) ? hi16(xlo[j >> 1]) : lo16(xlo[j >> 1]);
      const uint16_t xj8 = (j & 1) ? hi16(xhi[j >> 1]) : lo16(xhi[j >> 1]);
      a[j & 3] = fma_f16f16_f32(lo16(d), xj, a[j & 3]);
      a[j & 3] = fma_f16f16_f32(hi16(d), xj8, a[j & 3]);
    }
  }
  return fmaf(a[3], 0.015625f, fmaf(a[2], 0.0625f, fmaf(a[1], 0.25f, a[0])));
}

}  // namespace

template <int BITS>
__global__ void __launch_bounds__(THREADS, 1) gemv_bulk_kernel(const __grid_constant__ BulkParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = tc::smem_u32(smem);
  const uint32_t bar_full = sbase + OFF_BAR;
  const uint32_t bar_empty = bar_full + 8 * kBulkStages;
  const uint32_t bar_mfull = bar_empty + 8 * kBulkStages;  // [2]
  const uint32_t bar_mempty = bar_mfull + 16;               // [2]
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 8 * (2 * kBulkStages + 4));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kBulkStages; ++i) {
      tc::mbar_init(bar_full + 8 * i, 1);
      tc::mbar_init(bar_empty + 8 * i, CW);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(bar_mfull + 8 * i, 1);
      tc::mbar_init(bar_mempty + 8 * i, CW);
    }
    tc::fence_mbar_init();
    *abort_flag = 0;
  }
  __syncthreads();

  const int64_t share = (P.total_cost + gridDim.x - 1) / gridDim.x;
  const int blk_lo = first_block_at(P, share * blockIdx.x);
  const int blk_hi = first_block_at(P, share * (blockIdx.x + 1));
  bool timed_out = false;

  // Slab and meta-slot sequence numbers, identical on the producer and consumer sides.
  int it = 0, mseq = 0;
  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      int mi = 0;
      for (int blk = blk_lo; blk < blk_hi && !timed_out; ++blk) {
        while (blk >= P.m[mi].block_end) ++mi;
        const BulkMat& M = P.m[mi];
        const int row0 = (blk - M.block_begin) * M.rows_per_block;
        const int rows = min(M.rows_per_block, M.N - row0);
        const int G = M.K / kGroup;
        const int64_t row_bytes = (int64_t)M.K * BITS / 8;
        // scales and zeros of the block, when they can be bulk-copied (16-byte aligned)
        if (M.meta_bulk && (row0 * G) % 8 == 0 && (rows * G) % 8 == 0) {
          const int ms = mseq & 1;
          if (!tc::mbar_wait(bar_mempty + 8 * ms, ((mseq >> 1) & 1) ^ 1)) { timed_out = true; break; }
          const uint32_t mb = (uint32_t)(rows * G * 2);
          tc::mbar_arrive_expect_tx(bar_mfull + 8 * ms, 2 * mb);
          const uint32_t mdst = sbase + OFF_META + ms * kBulkMetaBytes;
          bulk_g2s(mdst, M.scale + (size_t)row0 * G, mb, bar_mfull + 8 * ms);
          bulk_g2s(mdst + mb, M.zero + (size_t)row0 * G, mb, bar_mfull + 8 * ms);
          ++mseq;
        }
        for (int seg = 0; seg < M.nseg; ++seg) {
          const int k0 = seg * M.kseg;
          const int kw = min(M.kseg, M.K - k0);
          const uint32_t seg_row_bytes = (uint32_t)(kw * BITS / 8);
          const int s = it % kBulkStages;
          if (!tc::mbar_wait(bar_empty + 8 * s, ((it / kBulkStages) & 1) ^ 1)) { timed_out = true; break; }
          tc::mbar_arrive_expect_tx(bar_full + 8 * s, seg_row_bytes * rows);
          const uint32_t dst = sbase + s * kBulkStageBytes;
          const uint8_t* src = reinterpret_cast<const uint8_t*>(M.codes) + (size_t)row0 * row_bytes + (size_t)k0 * BITS / 8;
          if (M.nseg == 1) {
            bulk_g2s(dst, src, seg_row_bytes * rows, bar_full + 8 * s);
          } else {
            for (int r = 0; r < rows; ++r)
              bulk_g2s(dst + r * seg_row_bytes, src + (size_t)r * row_bytes, seg_row_bytes, bar_full + 8 * s);
          }
          ++it;
        }
      }
    }
  } else {
    // ------------------------------ consumers ------------------------------
    const int cw = warp - 1;
    int mi = 0;
    for (int blk = blk_lo; blk < blk_hi && !timed_out; ++blk) {
      while (blk >= P.m[mi].block_end) ++mi;
      const BulkMat& M = P.m[mi];
      const int L2 = M.lanes_log2, L = 1 << L2;
      const int row0 = (blk - M.block_begin) * M.rows_per_block;
      const int rows = min(M.rows_per_block, M.N - row0);
      const int r = cw * (32 >> L2) + (lane >> L2);
      const int sub = lane & (L - 1);
      const bool valid = r < rows;
      const int G = M.K / kGroup;
      const bool meta_in_smem = M.meta_bulk && (row0 * G) % 8 == 0 && (rows * G) % 8 == 0;
      const int ms = mseq & 1;
      if (meta_in_smem && !tc::mbar_wait(bar_mfull + 8 * ms, (mseq >> 1) & 1)) { timed_out = true; break; }
      const uint16_t* s_meta = reinterpret_cast<const uint16_t*>(smem + OFF_META + ms * kBulkMetaBytes);
      const int row = row0 + r;
      float acc = 0.f;
      for (int seg = 0; seg < M.nseg; ++seg, ++it) {
        const int k0 = seg * M.kseg;
        const int kw = min(M.kseg, M.K - k0);
        const int s = it % kBulkStages;
        if (!tc::mbar_wait(bar_full + 8 * s, (it / kBulkStages) & 1)) { timed_out = true; break; }
        if (valid) {
          constexpr int WPC = (BITS == 4) ? 32 : 64;  // weights per 16-byte chunk
          const int SC = kw / WPC;
          const int c_lo = (sub * SC) >> L2, c_hi = ((sub + 1) * SC) >> L2;
          const uint4* sc = reinterpret_cast<const uint4*>(smem + s * kBulkStageBytes + (size_t)r * (kw * BITS / 8));
          int cur_g = -1;
          float sf = 0.f;
          uint32_t cz[4] = {0, 0, 0, 0};
          for (int c = c_lo; c < c_hi; ++c) {
            const int kg = k0 + c * WPC;
            const int g = kg / kGroup;
            if (g != cur_g) {
              cur_g = g;
              uint16_t sb, zb;
              if (meta_in_smem) {
                sb = s_meta[r * G + g];
                zb = s_meta[rows * G + r * G + g];
              } else {
                sb = ld_u16(M.scale + (size_t)row * G + g);
                zb = ld_u16(M.zero + (size_t)row * G + g);
              }
              sf = __half2float(__ushort_as_half(sb));
              const __half z = __ushort_as_half(zb);
#pragma unroll
              for (int j = 0; j < (BITS == 4 ? 2 : 4); ++j) {
                const float mul = (BITS == 4) ? (j == 0 ? 1.f : 16.f) : (float)(1 << (2 * j));
                cz[j] = pack_h2(__hfma(z, __float2half(mul), __float2half(1024.f)));
              }
            }
            const uint4 w = sc[c];
            const uint4* xp = reinterpret_cast<const uint4*>(M.x + kg);
            const float part = (BITS == 4) ? dot_chunk_int4(w, xp, cz[0], cz[1]) : dot_chunk_int2(w, xp, cz);
            acc = fmaf(sf, part, acc);
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar_empty + 8 * s);
      }
      if (meta_in_smem) {
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar_mempty + 8 * ms);
        ++mseq;
      }
      for (int o = L >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (valid && sub == 0 && !timed_out) M.y[row] = __half_as_ushort(__float2half_rn(acc));
    }
  }

  if (timed_out) {
    atomicOr(P.errors, tc::kErrTimeout);
    *abort_flag = 1;
  }
  __syncthreads();
  // On the error path the producer waits (bounded) for its own bulk copies that may still
  // be in flight -- the last kBulkStages slabs and the last two meta copies -- before the
  // shared memory they target is released.
  if (*abort_flag && warp == 0 && lane == 0) {
    for (int j = (it > kBulkStages ? it - kBulkStages : 0); j < it; ++j)
      tc::mbar_wait(bar_full + 8 * (j % kBulkStages), (j / kBulkStages) & 1);
    for (int j = (mseq > 2 ? mseq - 2 : 0); j < mseq; ++j)
      tc::mbar_wait(bar_mfull + 8 * (j & 1), (j >> 1) & 1);
  }
}

// ---- host side -----------------------------------------------------------------------

// Lanes per row, rows per block and K segment of one matrix; false if this kernel does
// not serve the shape (the caller then uses the register-streaming kernel).
bool bulk_plan_mat(BulkMat& m, int bits, const void* codes, const uint16_t* scale,
                   const uint16_t* zero, const uint16_t* x, uint16_t* y, int64_t N, int64_t K) {
  const int64_t cpr = K * bits / 128;  // 16-byte chunks per row
  const int l2 = cpr >= 128 ? 5 : cpr >= 64 ? 4 : cpr >= 32 ? 3 : 2;
  const int R = CW * (32 >> l2);
  const int64_t row_bytes = K * bits / 8;
  int64_t kseg = K;
  if (R * row_bytes > kBulkStageBytes) {
    // K segments of whole groups, each segment's rows fitting one stage
    kseg = (kBulkStageBytes / R) * 8 / bits;
    kseg -= kseg % kGroup;
    if (kseg < kGroup) return false;
  }
  m.codes = codes;
  m.scale = scale;
  m.zero = zero;
  m.x = x;
  m.y = y;
  m.N = (int)N;
  m.K = (int)K;
  m.lanes_log2 = l2;
  m.rows_per_block = R;
  m.kseg = (int)kseg;
  m.nseg = (int)((K + kseg - 1) / kseg);
  const int64_t G = K / kGroup;
  m.meta_bulk = (((uintptr_t)scale | (uintptr_t)zero) % 16 == 0) && (R * G * 2 * 2 <= kBulkMetaBytes);
  m.block_bytes = R * row_bytes;
  return true;
}

template <int BITS>
static cudaError_t launch_bits(const BulkParams& p, cudaStream_t stream) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemv_bulk_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int grid = p.total_blocks < sms ? p.total_blocks : sms;
  gemv_bulk_kernel<BITS><<<grid, THREADS, SMEM_BYTES, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemv_bulk(const BulkParams& p, int bits, cudaStream_t stream) {
  return bits == 4 ? launch_bits<4>(p, stream) : launch_bits<2>(p, stream);
}

}  // namespace wq
