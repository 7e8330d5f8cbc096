// Dequantising GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), int4 weights.
//
// TKintegers K5, "What is K5?": bounded weight tiles are expanded into fp16 tensor-core
// operands and multiplied with fp32 accumulation. Here the tile is dequantised in shared
// memory and the product runs on tcgen05.mma with the accumulator in tensor memory.
//
// Orientation ("swap AB"): the MMA's M side is 128 weight rows (output features) and its
// N side is BN <= 256 activation rows (tokens), so one CTA computes
//     D[n, m] = sum_k w_hat[n0 + n, k] * X[m0 + m, k]      (n < 128, m < BN)
// and every dequantised weight is reused by all BN tokens of the tile.
//
// Per 64-wide k-block (one stage of a 4-stage ring):
//   - warp 0 (one lane): TMA loads the X tile [BN x 64] fp16 (128-byte swizzle) and the
//     packed codes [128 rows x 32 bytes], both completing on full[s];
//   - warps 4-11 (256 threads, two per weight row): dequantise the codes into fp16
//     (q - z) * s and store them into A[s] in the 128-byte-swizzled K-major layout the
//     tensor core reads, fence the async proxy, arrive on a_ready[s];
//   - warp 1 (one lane): waits full[s] and a_ready[s], issues four m128 x nBN x k16 MMAs,
//     and commits them to empty[s], which frees the stage for the next TMA round.
// After the last k-block the MMA lane commits to tmem_full; warps 4-11 then read the
// accumulators (tcgen05.ld) and store fp16 Y[m, n] (one warp store covers 32 consecutive n).
//
// Every mbarrier wait is bounded; a wait that gives up sets kErrTimeout in the library's
// device error word, and the CTA drains its own TMA loads, frees its TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "tc_ptx.cuh"

namespace wq {

__device__ unsigned int g_device_errors;  // bit flags, read and cleared by wq_device_errors

namespace {

constexpr int BM = 128;       // weight rows per tile
constexpr int BK = 64;        // k per stage: one 128-byte swizzle row of fp16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = kTcMaxBN * BK * 2;      // 32 KB
constexpr int C_BYTES = BM * BK / 2;            // 4 KB of int4 codes
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
constexpr int OFF_BAR = OFF_C + STAGES * C_BYTES;
constexpr int NUM_BARS = 3 * STAGES + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_USED = OFF_MISC + 16;
constexpr int DEQ_THREADS = 256;
constexpr int THREADS = 384;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 8 int4 codes (natural order, code j at bits 4j) -> four fp16x2 words of (q - z) * s in
// natural order: (w0,w1) (w2,w3) (w4,w5) (w6,w7). (q - z) is exact; one rounding in * s.
__device__ __forceinline__ uint4 dequant8(uint32_t v, uint32_t c1024z, uint32_t s2) {
  const uint32_t d0 = hsub2_u32(lop_and_or(v, 0x000F000Fu, 0x64006400u), c1024z);        // (q0, q4)
  const uint32_t d1 = hsub2_u32(lop_and_or(v >> 4, 0x000F000Fu, 0x64006400u), c1024z);   // (q1, q5)
  const uint32_t d2 = hsub2_u32(lop_and_or(v >> 8, 0x000F000Fu, 0x64006400u), c1024z);   // (q2, q6)
  const uint32_t d3 = hsub2_u32(lop_and_or(v >> 12, 0x000F000Fu, 0x64006400u), c1024z);  // (q3, q7)
  const uint32_t e0 = hmul2_u32(d0, s2), e1 = hmul2_u32(d1, s2);
  const uint32_t e2 = hmul2_u32(d2, s2), e3 = hmul2_u32(d3, s2);
  uint4 r;
  r.x = prmt(e0, e1, 0x5410);  // (w0, w1)
  r.y = prmt(e2, e3, 0x5410);  // (w2, w3)
  r.z = prmt(e0, e1, 0x7632);  // (w4, w5)
  r.w = prmt(e2, e3, 0x7632);  // (w6, w7)
  return r;
}

}  // namespace

__global__ void __launch_bounds__(THREADS, 1) gemm_tc_int4_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment of the operand buffers is what the 128-byte swizzle assumes
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  const uint32_t bar_full = sbase + OFF_BAR;                 // [STAGES]
  const uint32_t bar_aready = bar_full + 8 * STAGES;         // [STAGES]
  const uint32_t bar_empty = bar_aready + 8 * STAGES;        // [STAGES]
  const uint32_t bar_tmem = bar_empty + 8 * STAGES;          // [1]
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);  // [0] tmem base, [1] abort

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which tile ----
  const int tile = blockIdx.x;
  int mi = 0;
  while (tile >= P.m[mi].tile_end) ++mi;
  const TcMat& M = P.m[mi];
  const int local = tile - M.tile_begin;
  const int n0 = (local / M.tiles_m) * BM;
  const int m0 = (local % M.tiles_m) * M.bn;
  const int BN = M.bn;
  const int nkb = M.K / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      tc::mbar_init(bar_full + 8 * i, 1);
      tc::mbar_init(bar_aready + 8 * i, DEQ_THREADS / 32);
      tc::mbar_init(bar_empty + 8 * i, 1);
    }
    tc::mbar_init(bar_tmem, 1);
    tc::fence_mbar_init();
    misc[1] = 0;
    tc::prefetch_tmap(&M.tmap_x);
    tc::prefetch_tmap(&M.tmap_codes);
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + OFF_MISC, kTcMaxBN);  // 256 fp32 columns x 128 lanes
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = misc[0];

  bool timed_out = false;
  int issued = 0;  // TMA stages issued by the producer (drained on the error path)

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      const uint32_t tx = (uint32_t)(BN * BK * 2 + C_BYTES);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!tc::mbar_wait(bar_empty + 8 * s, ph ^ 1)) { timed_out = true; break; }
        if (misc[1]) break;
        tc::mbar_arrive_expect_tx(bar_full + 8 * s, tx);
        tc::tma_load_2d(sbase + OFF_B + s * B_BYTES, &M.tmap_x, bar_full + 8 * s, kb * BK, m0);
        tc::tma_load_2d(sbase + OFF_C + s * C_BYTES, &M.tmap_codes, bar_full + 8 * s, kb * (BK / 2), n0);
        ++issued;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f16_f32(BM, BN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!tc::mbar_wait(bar_full + 8 * s, ph) || !tc::mbar_wait(bar_aready + 8 * s, ph)) {
          timed_out = true;
          break;
        }
        tc::tc_fence_after();
        const uint64_t ad = tc::sw128_kmajor_desc(sbase + OFF_A + s * A_BYTES);
        const uint64_t bd = tc::sw128_kmajor_desc(sbase + OFF_B + s * B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)  // +32 bytes along K inside the swizzled row
          tc::mma_f16_ss(tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
        tc::mma_commit(bar_empty + 8 * s);
      }
      tc::mma_commit(bar_tmem);  // fires when every MMA above has completed
    }
  } else if (warp >= 4) {
    // ---------------- dequantisers, then epilogue ----------------
    const int t = threadIdx.x - 128;     // 0..255
    const int r = t & (BM - 1);          // weight row within the tile
    const int h = t >> 7;                // which 32 of the k-block's 64
    const int n = min(n0 + r, M.N - 1);  // rows past N are computed but never stored
    const int G = M.K / kGroup;
    const uint16_t* srow = M.scale + (size_t)n * G;
    const uint16_t* zrow = M.zero + (size_t)n * G;
    uint32_t c1024z = 0, s2 = 0;
    for (int kb = 0; kb < nkb && !timed_out; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if ((kb & 1) == 0) {  // a 128-wide group spans two k-blocks
        const __half z = __ushort_as_half(ld_u16(zrow + kb / 2));
        const __half sc = __ushort_as_half(ld_u16(srow + kb / 2));
        c1024z = pack_h2(__hadd(z, __float2half(1024.f)));
        s2 = pack_h2(sc);
      }
      if (!tc::mbar_wait(bar_full + 8 * s, ph)) { timed_out = true; break; }
      const uint4 cw = *reinterpret_cast<const uint4*>(smem + OFF_C + s * C_BYTES + r * 32 + h * 16);
      const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
      uint8_t* arow = smem + OFF_A + s * A_BYTES + r * 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = 4 * h + i;  // logical 16-byte chunk (8 fp16) within the 128-byte row
        *reinterpret_cast<uint4*>(arow + ((j ^ (r & 7)) << 4)) = dequant8(words[i], c1024z, s2);
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_aready + 8 * s);
    }
    // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31, tokens [half*128, half*128+128)
    if (!timed_out) {
      if (!tc::mbar_wait(bar_tmem, 0)) timed_out = true;
    }
    if (!timed_out) {
      tc::tc_fence_after();
      const int q = warp & 3, half = (warp - 4) >> 2;
      const int row = n0 + 32 * q + lane;
      for (int c0 = half * 128; c0 < half * 128 + 128 && c0 < BN; c0 += 32) {
        uint32_t v[32];
        tc::tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
        tc::tmem_wait_ld();
        if (row < M.N) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int m = m0 + c0 + c;
            if (m < M.M)
              M.y[(size_t)m * M.ldy + row] = __half_as_ushort(__float2half_rn(__uint_as_float(v[c])));
          }
        }
      }
    }
  }

  if (timed_out) {
    atomicOr(&g_device_errors, tc::kErrTimeout);
    misc[1] = 1;
  }
  // The producer waits (bounded) for its own TMA loads still in flight before the shared
  // memory they target is released.
  if (warp == 0 && lane == 0 && misc[1]) {
    for (int kb = 0; kb < issued; ++kb) tc::mbar_wait(bar_full + 8 * (kb % STAGES), (kb / STAGES) & 1);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTcMaxBN);
  }
}

// ---- host side -----------------------------------------------------------------------

// cuTensorMapEncodeTiled, fetched through the runtime so libwq needs no -lcuda.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor maps of one matrix: X [M, K] fp16 (box 64 x bn, 128-byte swizzle) and the int4
// codes as bytes [N, K/2] (box 32 x 128, no swizzle). Returns false if encoding fails.
bool tc_plan_mat(TcMat& t, const uint16_t* X, int M, const void* codes, const uint16_t* scale,
                 const uint16_t* zero, uint16_t* Y, int N, int K, int bn) {
  auto enc = get_encode();
  if (!enc) return false;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)bn};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&t.tmap_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)K / 2};
    const cuuint32_t box[2] = {(cuuint32_t)(BK / 2), (cuuint32_t)BM};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&t.tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  t.scale = scale;
  t.zero = zero;
  t.y = Y;
  t.N = N;
  t.K = K;
  t.M = M;
  t.ldy = N;
  t.bn = bn;
  t.tiles_n = (N + BM - 1) / BM;
  t.tiles_m = (M + bn - 1) / bn;
  return true;
}

int tc_bn_for(int M) {
  const int bn = ((M + 15) / 16) * 16;
  return bn < kTcMaxBN ? bn : kTcMaxBN;
}

cudaError_t launch_gemm_tc(const TcParams& p, cudaStream_t stream) {
  static bool attr = false;
  const int smem = SMEM_USED + 1024;  // + alignment slack
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  gemm_tc_int4_kernel<<<p.total_tiles, THREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

unsigned int* device_error_word() {
  static unsigned int* addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_errors) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(p);
  }
  return addr[dev];
}

cudaError_t read_device_errors(unsigned int* flags, bool clear, cudaStream_t stream) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(flags, g_device_errors, sizeof(unsigned int), 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return e;
  if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return e;
  if (clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_device_errors, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  }
  return e;
}

}  // namespace wq
