// Skinny-batch int4 GEMM, Y[M, N] = X[M, K] * W_hat^T for M <= 32 tokens, on warp-level
// tensor-core MMAs (mma.sync m16n8k16, fp16 in, fp32 accumulate) fed from registers.
//
// Whetstone README, speculative decoding (the multi-token verify pass and its timing
// table): a pass over a few tokens still reads every weight once, so it stays bound by the
// weight stream, not by arithmetic, until M is in the tens. The tcgen05 GEMM (gemm_tc.cu)
// stages each dequantised tile in shared memory and hands it to the tensor core through
// mbarriers; at small M that hand-off, paid per 64-wide k-block, is what limits it. Here a
// warp dequantises straight into MMA operand registers: no shared-memory round trip for
// the weights and no cross-warp hand-off.
//
// Orientation: the MMA's M side is 16 weight rows (a warp's slab: rows g and g + 8 for lane
// group g = lane / 4), its N side is 8 tokens (TB blocks of 8), K is 16 per MMA. Lane
// (g, t = lane % 4) loads the 16 bytes at column 32 t of each 128-weight group of its two
// rows: four code words, word w holding the codes of k = 32 t + 8 w + 0..7. For each word
// the MMA's k slots are matched to codes as
//     slots 2t, 2t+1   <- codes 0, 1 (first MMA) or 4, 5 (second MMA)
//     slots 2t+8, 2t+9 <- codes 2, 3 (first MMA) or 6, 7 (second MMA)
// which is a permutation of the 16 k of each MMA that both operands follow, so the sum is
// unchanged. The activations' B-fragment registers of the two MMAs are then exactly the
// natural 16 bytes x[n][k .. k + 7]: the activations need no reordering.
//
// Dequantisation of a code byte (two codes, natural order) takes three instructions: PRMT
// copies the byte into both halves of a word; LOP3 keeps the low nibble in the low half and
// the high nibble (times 16) in the high half, over the binary16 bits of 1024, giving
// (1024 + q0, 1024 + 16 q1); one packed binary16 FMA with (1, 1/16) and -(1024 + z, 64 + z)
// gives (q0 - z, q1 - z). Every step is exact (integers below 2048 in binary16), so the MMA
// multiplies exact integer weights by the fp16 activations; the group scale is applied in
// fp32 to each group's MMA sum. Only fp32 adds and the final fp16 store round.
//
// Work: units of 128 weight rows x all of K (eight warps, one 16-row slab each), ordered by
// K (largest first) and dealt to CTAs round robin. The activations of a unit are staged in
// shared memory (cp.async) in chunks of up to kc groups, two buffers, the next chunk's copy
// in flight while the current one is used. Codes and metadata go straight from global
// memory into registers one group ahead, with a 256-byte L2 fetch size so that a row's next
// groups arrive with the current one.
#include <climits>

#include "common.cuh"
#include "gemm_skinny.cuh"

namespace wq {

namespace {

constexpr int kThreads = 32 * kSkWarps;

__device__ __forceinline__ uint4 ld_codes16(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// d += A * B (m16n8k16, A row-major 16 x 16 fp16, B column-major 16 x 8 fp16, fp32 d)
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Two codes of byte j of v, minus the zero point, as binary16 (q_{2j} - z, q_{2j+1} - z).
// nzc = -(1024 + z, 64 + z); one16 = (1, 1/16).
__device__ __forceinline__ uint32_t pair_minus_z(uint32_t v, uint32_t sel, uint32_t nzc) {
  const uint32_t one16 = 0x2C003C00u;
  return hfma2_u32(lop_and_or(prmt_u32(v, 0u, sel), 0x00F0000Fu, 0x64006400u), one16, nzc);
}

// -(1024 + z, 64 + z) from the binary16 bits of an integer zero point z (exact).
__device__ __forceinline__ uint32_t neg_zc(uint16_t zb) {
  const uint32_t zz = (uint32_t)zb | ((uint32_t)zb << 16);
  return hfma2_u32(zz, 0xBC00BC00u, 0xD400E400u);  // -z + (-1024, -64)
}

// Byte offset of 16-byte activation chunk c (c = k / 8 within the chunk) in a token's row:
// chunks 8..15 of each group swap pairs (c ^ 2), so that the eight lanes of a shared-memory
// phase (two tokens x four t, the same w) read eight different bank groups, given a row
// stride of 16 (mod 128) bytes.
__device__ __forceinline__ uint32_t xchunk_off(uint32_t c) { return (c ^ (((c >> 3) & 1u) << 1)) << 4; }

struct Item {
  int unit, ch, mi;
};

template <int CAP>
__device__ __forceinline__ int find_mat(const SkParamsT<CAP>& P, int unit) {
  int lo = 0, hi = P.count - 1;
  while (lo < hi) {  // last matrix whose unit_begin <= unit
    const int mid = (lo + hi + 1) >> 1;
    if (P.m[mid].unit_begin <= unit) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace

template <int TB, int CAP>
__global__ void __launch_bounds__(kThreads, kSkCtasPerSm) gemm_skinny_kernel(const __grid_constant__ SkParamsT<CAP> P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = P.M;
  constexpr int NT = 8 * TB;                       // staged token rows (zero past M)
  constexpr int TPT = kThreads / NT;               // staging threads per token row
  const int stage_n = threadIdx.x / TPT, stage_c0 = threadIdx.x % TPT;

  // stage the activations of item it into buffer b (cp.async; rows past M are zeroed)
  auto stage = [&](const Item& it, int b) {
    const SkMat& Mt = P.m[it.mi];
    const int G = Mt.K / kGroup;
    const int g0 = it.ch * Mt.kc, ng = min(Mt.kc, G - g0);
    const uint32_t ts = (uint32_t)Mt.kc * 256u + 16u;
    const uint32_t row = sbase + (uint32_t)b * (uint32_t)P.buf_bytes + (uint32_t)stage_n * ts;
    const int nc = 16 * ng;
    if (stage_n < M) {
      const uint16_t* src = Mt.x + (size_t)stage_n * Mt.K + (size_t)g0 * kGroup;
      for (int c = stage_c0; c < nc; c += TPT) cp_async16(row + xchunk_off((uint32_t)c), src + 8 * c);
    } else {
      for (int c = stage_c0; c < nc; c += TPT)
        asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(row + xchunk_off((uint32_t)c)), "r"(0u) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  auto next_item = [&](Item it) {
    if (it.ch + 1 < P.m[it.mi].nch) {
      ++it.ch;
    } else {
      it.unit += gridDim.x;
      it.ch = 0;
      if (it.unit < P.total_units) it.mi = find_mat(P, it.unit);
    }
    return it;
  };

  Item cur{(int)blockIdx.x, 0, 0};
  if (cur.unit >= P.total_units) return;
  cur.mi = find_mat(P, cur.unit);
  stage(cur, 0);

  float acc[TB][4];
#pragma unroll
  for (int b = 0; b < TB; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;

  for (int i = 0; cur.unit < P.total_units; ++i) {
    const SkMat& Mt = P.m[cur.mi];
    const int K = Mt.K, G = K / kGroup;
    const int g0 = cur.ch * Mt.kc, ng = min(Mt.kc, G - g0);
    const int n0 = (cur.unit - Mt.unit_begin) * kSkUnitRows + 16 * warp;
    const int r_lo = min(n0 + g, Mt.N - 1), r_hi = min(n0 + g + 8, Mt.N - 1);
    const uint8_t* c_lo = Mt.codes + (size_t)r_lo * (K / 2) + 16 * t;
    const uint8_t* c_hi = Mt.codes + (size_t)r_hi * (K / 2) + 16 * t;
    const uint16_t* s_lo = Mt.scale + (size_t)r_lo * G;
    const uint16_t* s_hi = Mt.scale + (size_t)r_hi * G;
    const uint16_t* z_lo = Mt.zero + (size_t)r_lo * G;
    const uint16_t* z_hi = Mt.zero + (size_t)r_hi * G;

    // first group of this item: its loads fly while the CTA waits for the activations
    uint4 nw_lo = ld_codes16(c_lo + (size_t)g0 * 64), nw_hi = ld_codes16(c_hi + (size_t)g0 * 64);
    uint16_t ns_lo = ld_u16(s_lo + g0), ns_hi = ld_u16(s_hi + g0);
    uint16_t nz_lo = ld_u16(z_lo + g0), nz_hi = ld_u16(z_hi + g0);

    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();  // item i's activations are visible; every warp is done with item i - 1
    const Item nxt = next_item(cur);
    if (nxt.unit < P.total_units) stage(nxt, (i + 1) & 1);

    const uint32_t ts = (uint32_t)Mt.kc * 256u + 16u;
    // this lane's activation row (token g of block 0) in the buffer of item i
    const uint8_t* xrow = smem + (size_t)(i & 1) * P.buf_bytes + (size_t)g * ts;
    for (int gl = 0; gl < ng; ++gl) {
      const uint4 w_lo = nw_lo, w_hi = nw_hi;
      const float sf_lo = __half2float(__ushort_as_half(ns_lo)), sf_hi = __half2float(__ushort_as_half(ns_hi));
      const uint32_t zc_lo = neg_zc(nz_lo), zc_hi = neg_zc(nz_hi);
      if (gl + 1 < ng) {
        const int gg = g0 + gl + 1;
        nw_lo = ld_codes16(c_lo + (size_t)gg * 64);
        nw_hi = ld_codes16(c_hi + (size_t)gg * 64);
        ns_lo = ld_u16(s_lo + gg);
        ns_hi = ld_u16(s_hi + gg);
        nz_lo = ld_u16(z_lo + gg);
        nz_hi = ld_u16(z_hi + gg);
      }
      float part[TB][4];
#pragma unroll
      for (int b = 0; b < TB; ++b) part[b][0] = part[b][1] = part[b][2] = part[b][3] = 0.f;
      const uint32_t wl[4] = {w_lo.x, w_lo.y, w_lo.z, w_lo.w};
      const uint32_t wh[4] = {w_hi.x, w_hi.y, w_hi.z, w_hi.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t a0 = pair_minus_z(wl[w], 0x0000u, zc_lo), a1 = pair_minus_z(wh[w], 0x0000u, zc_hi);
        const uint32_t a2 = pair_minus_z(wl[w], 0x1111u, zc_lo), a3 = pair_minus_z(wh[w], 0x1111u, zc_hi);
        const uint32_t e0 = pair_minus_z(wl[w], 0x2222u, zc_lo), e1 = pair_minus_z(wh[w], 0x2222u, zc_hi);
        const uint32_t e2 = pair_minus_z(wl[w], 0x3333u, zc_lo), e3 = pair_minus_z(wh[w], 0x3333u, zc_hi);
        const uint8_t* xo = xrow + (size_t)gl * 256 + xchunk_off((uint32_t)(4 * t + w));
#pragma unroll
        for (int b = 0; b < TB; ++b) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xo + (size_t)(8 * b) * ts);
          mma16816(part[b], a0, a1, a2, a3, xv.x, xv.y);
          mma16816(part[b], e0, e1, e2, e3, xv.z, xv.w);
        }
      }
#pragma unroll
      for (int b = 0; b < TB; ++b) {
        acc[b][0] = fmaf(sf_lo, part[b][0], acc[b][0]);
        acc[b][1] = fmaf(sf_lo, part[b][1], acc[b][1]);
        acc[b][2] = fmaf(sf_hi, part[b][2], acc[b][2]);
        acc[b][3] = fmaf(sf_hi, part[b][3], acc[b][3]);
      }
    }

    if (cur.ch + 1 == Mt.nch) {
      // C fragment: (row g, tokens 2t, 2t + 1) and (row g + 8, the same tokens)
      const int ra = n0 + g, rb = n0 + g + 8;
#pragma unroll
      for (int b = 0; b < TB; ++b) {
        const int m = 8 * b + 2 * t;
        if (m < M) {
          if (ra < Mt.N) Mt.y[(size_t)m * Mt.N + ra] = __half_as_ushort(__float2half_rn(acc[b][0]));
          if (rb < Mt.N) Mt.y[(size_t)m * Mt.N + rb] = __half_as_ushort(__float2half_rn(acc[b][2]));
        }
        if (m + 1 < M) {
          if (ra < Mt.N) Mt.y[(size_t)(m + 1) * Mt.N + ra] = __half_as_ushort(__float2half_rn(acc[b][1]));
          if (rb < Mt.N) Mt.y[(size_t)(m + 1) * Mt.N + rb] = __half_as_ushort(__float2half_rn(acc[b][3]));
        }
        acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;
      }
    }
    cur = nxt;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---- host side -----------------------------------------------------------------------

static int tb_for(int M) { return M <= 8 ? 1 : M <= 16 ? 2 : 4; }

int skinny_plan(SkParams& p, int count, const SkDesc* d, int M) {
  if (count < 1 || count > kSkMaxMats || M < 1 || M > kSkMaxM) return 0;
  const int tb = tb_for(M);
  // one buffer: 8 TB token rows of kc * 256 + 16 bytes; two buffers per CTA
  const int kc_max = ((kSkSmemPerCta / 2) / (8 * tb) - 16) / 256;
  if (kc_max < 1) return 0;
  static thread_local int order[kSkMaxMats];
  for (int i = 0; i < count; ++i) {
    if (((uintptr_t)d[i].codes & 15) || ((uintptr_t)d[i].x & 15) || ((uintptr_t)d[i].scale & 1) ||
        ((uintptr_t)d[i].zero & 1) || !d[i].zero)
      return 0;
    order[i] = i;
  }
  for (int i = 1; i < count; ++i) {  // stable insertion sort by K, descending
    const int v = order[i];
    int j = i;
    while (j > 0 && d[order[j - 1]].K < d[v].K) {
      order[j] = order[j - 1];
      --j;
    }
    order[j] = v;
  }
  int64_t units = 0;
  int kc_used = 1;
  for (int j = 0; j < count; ++j) {
    const SkDesc& s = d[order[j]];
    SkMat& m = p.m[j];
    m.codes = static_cast<const uint8_t*>(s.codes);
    m.scale = s.scale;
    m.zero = s.zero;
    m.x = s.x;
    m.y = s.y;
    m.N = (int)s.N;
    m.K = (int)s.K;
    const int G = (int)(s.K / kGroup);
    m.nch = (G + kc_max - 1) / kc_max;
    m.kc = (G + m.nch - 1) / m.nch;
    kc_used = m.kc > kc_used ? m.kc : kc_used;
    m.unit_begin = (int)units;
    units += (s.N + kSkUnitRows - 1) / kSkUnitRows;
    if (units > INT_MAX) return 0;
  }
  p.count = count;
  p.M = M;
  p.total_units = (int)units;
  p.buf_bytes = 8 * tb * (kc_used * 256 + 16);
  return 2 * p.buf_bytes;
}

template <int TB>
static cudaError_t launch_tb(const SkParams& p, int smem, cudaStream_t stream) {
  static int attr_done[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    e = cudaFuncSetAttribute(gemm_skinny_kernel<TB, kSkMaxMats>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSkSmemPerCta);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = p.total_units < kSkCtasPerSm * sms ? p.total_units : kSkCtasPerSm * sms;
  gemm_skinny_kernel<TB, kSkMaxMats><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_skinny(const SkParams& p, int smem, cudaStream_t stream) {
  if (smem <= 0 || smem > kSkSmemPerCta || p.total_units < 1) return cudaErrorInvalidValue;
  switch (tb_for(p.M)) {
    case 1: return launch_tb<1>(p, smem, stream);
    case 2: return launch_tb<2>(p, smem, stream);
    default: return launch_tb<4>(p, smem, stream);
  }
}

}  // namespace wq
