// Matrix-vector product against packed int4 / int2 / ternary / hierarchical-int4 weights,
// streamed as contiguous bytes.
//
// Whetstone README, "The one fact that shapes everything": at batch 1 every weight is read
// once for one multiply-add, so the product runs at the speed the packed codes stream from
// HBM. On B200 that speed needs long contiguous reads: rows are contiguous in memory, so
// each warp owns a contiguous range of whole rows and moves it into shared memory with
// cp.async.bulk copies (2 KB of codes plus their scales and zeros per copy, a ring of a few
// copies in flight per warp, completion on mbarriers).
//
// The staged bytes are a stream of cells, one cell = one row's 128-weight group (64 bytes
// of int4 codes, 32 of int2). Lane j takes cell j of each step of 32 cells. Its 16-byte
// chunks are read in an order permuted by the cell's group index, so that the eight lanes
// of a shared-memory phase hit eight different bank groups; the activation vector is staged
// with each group's chunks in that same order and 17 units of 16 bytes per group (one
// spare), so that activation reads are conflict-free too, and lanes holding the same group
// index read the same activations (a broadcast).
//
// Dequantisation is one AND per pair of codes: the masked bits of a binary16 lane are the
// subnormal number q * 2^-24 (16 q * 2^-24 for the high nibble of a byte, which stays below
// the subnormal limit of 1024 * 2^-24); one packed binary16 subtract of z * 2^-24 (the
// integer zero point as bits) gives (q - z) * 2^-24 exactly; each product with an fp16
// activation is exact in binary32 (mixed-precision FMA); the 2^24 returns, exactly, with
// the group scale. Only binary32 adds, the multiply by the scale and the final fp16 store
// round, and q = z gives an exact zero. The cells of one row sit in
// consecutive lanes (and steps): a segmented shuffle scan per step sums them, a carry
// holds the part of a row that continues into the next step, and the lane holding a row's
// last group writes y.
//
// Hierarchical int4 (Whetstone README, "What the weights can actually survive": groups of 32
// with two 4-bit indices against an f16 pair per row) uses the int4 cells unchanged: a cell
// of 128 weights is four groups of 32, one 16-byte chunk each, and its four index bytes form
// the per-cell metadata word; no zero point is subtracted (w_hat = d a q - dm b), the group
// sums of x are staged beside the activations, and the lane reads its row's (d, dm) itself.
//
// The activation vector of the matrix being processed is staged once per CTA; two buffers
// let the next matrix's vector load while the current one is in use.
#include <climits>
#include <cmath>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv_stream.cuh"
#include "host_util.cuh"
#include "tc_ptx.cuh"

namespace wq {

namespace {

constexpr int W = kStreamWarps;
constexpr int T = 32 * W;
constexpr int TERN = 1;  // format tag of ternary (5 trits per byte, 26 bytes per group)
constexpr int HIER = kStreamHier;  // hierarchical int4 (group-32 indices, per-row fp16 pair)

// Chunk permutation of group g (XOR mask on the chunk index), shared by the codes reads and
// the staged activation layout.
template <int BITS>
__host__ __device__ __forceinline__ int xrot(int g) {
  return (BITS == 4 || BITS == HIER) ? (g >> 1) & 3 : BITS == 2 ? (g >> 2) & 1 : 0;
}

// Per format (BITS = 4, 3, 2, TERN or HIER): bytes of codes per cell (128 weights of a row), ring
// slot layout (codes, then the per-cell metadata: scales and zeros of the g128 integer
// formats, scales of ternary, the four index bytes of HIER), staged activation units per group.
template <int BITS>
struct Fmt {
  static constexpr bool TRN = BITS == TERN;
  static constexpr bool HR = BITS == HIER;
  static constexpr int CB = TRN ? 26 : HR ? 64 : 128 * BITS / 8;  // codes bytes per cell: 64 / 48 / 32 / 26
  static constexpr int CH = TRN ? 1 : CB / 16;          // 16-byte chunks per cell: 4 / 2
  static constexpr int UPC = 16 / CH;                   // activation units per chunk: 4 / 8
  static constexpr int SPS = TRN ? 4 : kStreamSlotCodes / (32 * CB);  // steps of 32 cells per slot
  static constexpr int SC = 32 * SPS * CB;              // codes bytes per slot: 4096 / 4096 / 3328
  static constexpr int GPSL = 32 * SPS;                 // groups per ring slot: 64 / 128 / 128
  static constexpr int MB0 = HR ? 4 : 2;                // bytes per cell of metadata array 0 (scale / index)
  static constexpr int MB1 = (TRN || HR) ? 0 : 2;       // bytes per cell of metadata array 1 (zero)
  static constexpr int META0 = MB0 * GPSL;              // bytes of metadata array 0 per slot
  static constexpr int META1 = MB1 * GPSL;
  static constexpr int SLOT = SC + META0 + META1;
  static constexpr int XU = TRN ? 27 : 17;              // staged activation units per group
  static constexpr int LUT = TRN ? 256 * 4 : 0;         // byte -> five base-3 digits (shared memory)
};

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint16_t lds16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}

// Dot products of one 16-byte chunk of codes with the activations of MT rows of X (row m
// at shared-memory address xa + m * xs), accumulated in binary32 with the factor 2^-24
// described above. Each pair of codes is dequantised once for all MT rows.
// int4: 32 codes; z1 / z16 hold z and 16 z as binary16 bit patterns in both lanes; the a
// accumulators take codes at bits 0-3 of a byte, the b ones (16x) bits 4-7. SUBZ = false
// (no zero point to subtract, the hierarchical format) leaves the masked codes as they are.
template <int MT, bool SUBZ = true>
__device__ __forceinline__ void chunk_int4(const uint4 c, uint32_t xa, uint32_t xs, uint32_t z1, uint32_t z16,
                                           float (&a)[MT][2], float (&b)[MT][2]) {
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = cw[i], v8 = v >> 8;
    const uint32_t d0 = SUBZ ? hsub2_u32(v & 0x000F000Fu, z1) : v & 0x000F000Fu;     // q0, q4
    const uint32_t d1 = SUBZ ? hsub2_u32(v & 0x00F000F0u, z16) : v & 0x00F000F0u;   // 16 q1, 16 q5
    const uint32_t d2 = SUBZ ? hsub2_u32(v8 & 0x000F000Fu, z1) : v8 & 0x000F000Fu;   // q2, q6
    const uint32_t d3 = SUBZ ? hsub2_u32(v8 & 0x00F000F0u, z16) : v8 & 0x00F000F0u;  // 16 q3, 16 q7
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const uint4 xw = lds128(xa + m * xs + 16 * i);  // (x0, x1) (x2, x3) (x4, x5) (x6, x7)
      float& A = a[m][i & 1];
      float& B = b[m][i & 1];
      A = fma_f16f16_f32(lo16(d0), lo16(xw.x), A);
      A = fma_f16f16_f32(hi16(d0), lo16(xw.z), A);
      A = fma_f16f16_f32(lo16(d2), lo16(xw.y), A);
      A = fma_f16f16_f32(hi16(d2), lo16(xw.w), A);
      B = fma_f16f16_f32(lo16(d1), hi16(xw.x), B);
      B = fma_f16f16_f32(hi16(d1), hi16(xw.z), B);
      B = fma_f16f16_f32(lo16(d3), hi16(xw.y), B);
      B = fma_f16f16_f32(hi16(d3), hi16(xw.w), B);
    }
  }
}

// int2: 64 codes (four words of 16); zm[k] holds 4^k z as binary16 bits in both lanes; the
// lanes of d_j are codes j and j + 8 of a word, scaled by 4^(j mod 4), accumulated in
// a[m][j mod 4].
template <int MT>
__device__ __forceinline__ void chunk_int2(const uint4 c, uint32_t xa, uint32_t xs, const uint32_t (&zm)[4],
                                           float (&a)[MT][4]) {
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = cw[i], v8 = v >> 8;
    uint32_t d[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) d[j] = hsub2_u32((j < 4 ? v : v8) & (0x00030003u << (2 * (j & 3))), zm[j & 3]);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const uint4 xl = lds128(xa + m * xs + 32 * i), xh = lds128(xa + m * xs + 32 * i + 16);  // x0..x7, x8..x15
      const uint32_t xlw[4] = {xl.x, xl.y, xl.z, xl.w}, xhw[4] = {xh.x, xh.y, xh.z, xh.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint16_t xj = (j & 1) ? hi16(xlw[j >> 1]) : lo16(xlw[j >> 1]);
        const uint16_t xj8 = (j & 1) ? hi16(xhw[j >> 1]) : lo16(xhw[j >> 1]);
        a[m][j & 3] = fma_f16f16_f32(lo16(d[j]), xj, a[m][j & 3]);
        a[m][j & 3] = fma_f16f16_f32(hi16(d[j]), xj8, a[m][j & 3]);
      }
    }
  }
}

// out[m] = 2^-24 * sum_k x_mk (q_k - z) over one cell at shared address `cell`, for the MT
// rows of X; xg: shared address of the group's activation units in row 0, xs: bytes between
// rows; oc[c] / ox[c]: offsets of the cell's c-th chunk in this lane's permuted order and of
// that chunk's first activation unit.
template <int BITS, int MT>
__device__ __forceinline__ void cell_dot(uint32_t cell, uint32_t xg, uint32_t xs, const int (&oc)[Fmt<BITS>::CH],
                                         const int (&ox)[Fmt<BITS>::CH], uint16_t zbits, float (&out)[MT]) {
  using F = Fmt<BITS>;
  const uint32_t zi = (uint32_t)__half2int_rn(__ushort_as_half(zbits));  // integer zero point
  if constexpr (BITS == 4) {
    const uint32_t z1 = zi * 0x00010001u, z16 = zi * 0x00100010u;
    float a[MT][2], b[MT][2];
#pragma unroll
    for (int m = 0; m < MT; ++m) a[m][0] = a[m][1] = b[m][0] = b[m][1] = 0.f;
#pragma unroll
    for (int c = 0; c < F::CH; ++c) chunk_int4<MT>(lds128(cell + oc[c]), xg + ox[c], xs, z1, z16, a, b);
#pragma unroll
    for (int m = 0; m < MT; ++m) out[m] = fmaf(b[m][0] + b[m][1], 0.0625f, a[m][0] + a[m][1]);
  } else {
    uint32_t zm[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) zm[k] = (zi << (2 * k)) * 0x00010001u;
    float a[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m) a[m][0] = a[m][1] = a[m][2] = a[m][3] = 0.f;
#pragma unroll
    for (int c = 0; c < F::CH; ++c) chunk_int2<MT>(lds128(cell + oc[c]), xg + ox[c], xs, zm, a);
#pragma unroll
    for (int m = 0; m < MT; ++m) out[m] = fmaf(a[m][3], 0.015625f, fmaf(a[m][2], 0.0625f, fmaf(a[m][1], 0.25f, a[m][0])));
  }
}

// int3: out[m] = 2^-24 * sum_k x_mk (q_k - z) over one cell of 48 bytes (12 words, code k at
// bit 3k; codes 10, 21, 42, ... straddle two words). Codes are taken in pairs (2p, 2p + 1): a
// funnel shift brings bit 6p to bit 0, a byte permute copies byte 0 to bytes 0 and 2, and one
// AND leaves code 2p in bits 0-2 (the binary16 subnormal q 2^-24) and code 2p + 1 in bits
// 19-21 (8 q 2^-24); one packed subtract of (z, 8 z) 2^-24 gives the differences exactly, and
// the activations pair with them in natural order. The cells of a step sit 48 bytes apart, 12
// words: the 8 lanes of a shared-memory phase read 8 different bank groups without a permutation.
template <int MT>
__device__ __forceinline__ void cell_dot_int3(uint32_t cell, uint32_t xg, uint32_t xs, uint16_t zbits,
                                              float (&out)[MT]) {
  uint32_t wd[13];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const uint4 v = lds128(cell + 16 * c);
    wd[4 * c] = v.x;
    wd[4 * c + 1] = v.y;
    wd[4 * c + 2] = v.z;
    wd[4 * c + 3] = v.w;
  }
  wd[12] = 0u;
  const uint32_t zi = (uint32_t)__half2int_rn(__ushort_as_half(zbits));
  const uint32_t zp = zi | (zi << 19);  // (z, 8 z) as binary16 subnormal bits
  float a[MT][2], b[MT][2];
#pragma unroll
  for (int m = 0; m < MT; ++m) a[m][0] = a[m][1] = b[m][0] = b[m][1] = 0.f;
#pragma unroll
  for (int u = 0; u < 16; ++u) {  // 16 units of 8 activations
    uint4 xw[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) xw[m] = lds128(xg + m * xs + 16 * u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int bit = 6 * (4 * u + q);
      const uint32_t w = __funnelshift_r(wd[bit >> 5], wd[(bit >> 5) + 1], bit & 31);
      const uint32_t d = hsub2_u32(prmt_u32(w, 0u, 0x4040u) & 0x00380007u, zp);  // (q0 - z, 8 (q1 - z))
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint32_t xr = q == 0 ? xw[m].x : q == 1 ? xw[m].y : q == 2 ? xw[m].z : xw[m].w;
        a[m][q & 1] = fma_f16f16_f32(lo16(d), lo16(xr), a[m][q & 1]);
        b[m][q & 1] = fma_f16f16_f32(hi16(d), hi16(xr), b[m][q & 1]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) out[m] = fmaf(b[m][0] + b[m][1], 0.125f, a[m][0] + a[m][1]);
}

// Ternary: out[m] = 2^-24 * sum_k x_mk t_k over one cell (26 bytes at the 2-byte aligned
// shared address `cell`). lut: shared table of 256 words, word b = the base-3 digits
// d_i = t_i + 1 of byte b at bits 0, 16 (d0, d1), 2, 18 (d2, d3) and 4 (d4) (digits 1,
// i.e. zero trits, for the invalid bytes 243..255). Masking two digits gives the binary16
// subnormals d 2^-24; one packed subtract of 2^-24 gives (d - 1) 2^-24 = t 2^-24 exactly.
// xg: the group's 26 staged activation units of row 0 (unit j = x[5j .. 5j + 4]), rows xs
// bytes apart. Each product is exact in binary32.
template <int MT>
__device__ __forceinline__ void cell_dot_ternary(uint32_t cell, uint32_t xg, uint32_t xs, uint32_t lut,
                                                 float (&out)[MT]) {
  float a[MT][2];
#pragma unroll
  for (int m = 0; m < MT; ++m) a[m][0] = a[m][1] = 0.f;
#pragma unroll
  for (int h = 0; h < 13; ++h) {
    const uint32_t two = lds16(cell + 2 * h);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = 2 * h + e;
      uint32_t w;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(lut + 4 * ((two >> (8 * e)) & 0xFFu)));
      const uint32_t t01 = hsub2_u32(w & 0x00030003u, 0x00010001u);         // t0, t1
      const uint32_t t23 = hsub2_u32((w >> 2) & 0x00030003u, 0x00010001u);  // t2, t3
      const uint32_t t4 = hsub2_u32((w >> 4) & 0x00000003u, 0x00010001u);   // t4 (low half)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4 xw = lds128(xg + m * xs + 16 * j);
        float& A = a[m][e];
        A = fma_f16f16_f32(lo16(t01), lo16(xw.x), A);
        A = fma_f16f16_f32(hi16(t01), hi16(xw.x), A);
        A = fma_f16f16_f32(lo16(t23), lo16(xw.y), A);
        A = fma_f16f16_f32(hi16(t23), hi16(xw.y), A);
        A = fma_f16f16_f32(lo16(t4), lo16(xw.z), A);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) out[m] = a[m][0] + a[m][1];
}

// Hierarchical int4 (one cell = 128 weights of a row = four groups of 32, one 16-byte chunk
// each): P[m] = 2^-24 sum_j a_j sum_{k in group j} x_mk q_k and Q[m] = sum_j b_j sum_{k in
// group j} x_mk, so that the cell's share of y is d 2^24 P - dm Q (w_hat = d a_j q - dm b_j).
// ib: the cell's four index bytes (a_j | b_j << 4, group j in byte j); rot: the cell's chunk
// permutation (chunk c of the read order is group c ^ rot); the group sums of x are staged as
// four binary32 values (group order) in the spare unit 16 of the cell's activation units.
// The masked codes are the binary16 subnormals q 2^-24 (16 q 2^-24 for bits 4-7), so each
// product with x is exact in binary32, as for int4.
__device__ __forceinline__ float small_int_f32(uint32_t v) {  // exact float of 0 <= v < 2^23
  return __uint_as_float(0x4B000000u | v) - 8388608.0f;
}

template <int MT>
__device__ __forceinline__ void cell_dot_hier(uint32_t cell, uint32_t xg, uint32_t xs, const int (&oc)[4],
                                              const int (&ox)[4], int rot, uint32_t ib, float (&P)[MT],
                                              float (&Q)[MT]) {
#pragma unroll
  for (int m = 0; m < MT; ++m) P[m] = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float aj = small_int_f32((ib >> (8 * (c ^ rot))) & 15u);
    float a[MT][2], b[MT][2];
#pragma unroll
    for (int m = 0; m < MT; ++m) a[m][0] = a[m][1] = b[m][0] = b[m][1] = 0.f;
    chunk_int4<MT, false>(lds128(cell + oc[c]), xg + ox[c], xs, 0u, 0u, a, b);
#pragma unroll
    for (int m = 0; m < MT; ++m) P[m] = fmaf(aj, fmaf(b[m][0] + b[m][1], 0.0625f, a[m][0] + a[m][1]), P[m]);
  }
  const float b0 = small_int_f32((ib >> 4) & 15u), b1 = small_int_f32((ib >> 12) & 15u);
  const float b2 = small_int_f32((ib >> 20) & 15u), b3 = small_int_f32(ib >> 28);
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const uint4 sx = lds128(xg + m * xs + 16 * 16);
    Q[m] = fmaf(b3, __uint_as_float(sx.w),
                fmaf(b2, __uint_as_float(sx.z), fmaf(b1, __uint_as_float(sx.y), b0 * __uint_as_float(sx.x))));
  }
}

// Wait for an mbarrier phase, giving up after max_polls polls (false).
__device__ __forceinline__ bool mbar_wait_n(uint32_t bar, uint32_t parity, uint32_t max_polls) {
  for (uint32_t i = 0; i < max_polls; ++i)
    if (tc::mbar_try_wait(bar, parity)) return true;
  return false;
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ceil(num / M.unit_cost) for 0 <= num < 2^52: a double-precision estimate through the
// stored reciprocal, then an exact integer correction (the estimate is off by at most 1).
__device__ __forceinline__ int64_t units_ceil(int64_t num, const StreamMat& M) {
  const int64_t bc = M.unit_cost;
  int64_t q = (int64_t)((double)num * M.inv_unit_cost);
  if (q * bc > num) --q;
  if ((q + 1) * bc <= num) ++q;
  return q * bc < num ? q + 1 : q;
}

// Units (RA rows each) of M whose first byte of cost lies in [lo, hi): [b0, b1).
__device__ __forceinline__ void cta_units(const StreamMat& M, int64_t lo, int64_t hi, int& b0, int& b1) {
  const int64_t a = lo <= M.cost_begin ? 0 : units_ceil(lo - M.cost_begin, M);
  const int64_t b = hi <= M.cost_begin ? 0 : units_ceil(hi - M.cost_begin, M);
  b0 = (int)(a < M.nunit ? a : M.nunit);
  b1 = (int)(b < M.nunit ? b : M.nunit);
}

// One warp's share of a matrix: whole units [wb0, wb1) of the CTA's range, as rows.
// m0 / m1: the segment's per-cell metadata arrays (scales and zeros; HIER: index bytes, none).
struct Seg {
  const uint8_t* codes;
  const uint8_t* m0;
  const uint8_t* m1;
  int rows;
  int row0;
  int bytes;   // codes bytes
  int groups;  // rows * K / 128
};

template <int BITS>
__device__ __forceinline__ Seg warp_seg(const StreamMat& M, int b0, int b1, int w) {
  const int wb0 = b0 + (int)((int64_t)(b1 - b0) * w / W);
  const int wb1 = b0 + (int)((int64_t)(b1 - b0) * (w + 1) / W);
  const int64_t r0 = (int64_t)wb0 * M.RA;
  const int64_t r1 = (int64_t)wb1 * M.RA < M.N ? (int64_t)wb1 * M.RA : M.N;
  const int G = M.K / kGroup;
  const int64_t rb = (int64_t)G * Fmt<BITS>::CB;
  Seg s;
  s.rows = r1 > r0 ? (int)(r1 - r0) : 0;
  s.row0 = (int)r0;
  s.codes = reinterpret_cast<const uint8_t*>(M.codes) + r0 * rb;
  // HIER: the index bytes (passed as `zero`) are the per-cell metadata; the row pairs (passed
  // as `scale`) are read by the consumer lanes
  s.m0 = reinterpret_cast<const uint8_t*>(Fmt<BITS>::HR ? M.zero : M.scale) + r0 * G * Fmt<BITS>::MB0;
  s.m1 = reinterpret_cast<const uint8_t*>(M.zero) + r0 * G * Fmt<BITS>::MB1;
  s.bytes = (int)(s.rows * rb);
  s.groups = s.rows * G;
  return s;
}

// Copy state of one warp's producer, kept identically by all its lanes: what remains of the
// segment being issued.
struct Prod {
  const uint8_t* c;
  const uint8_t* m0;
  const uint8_t* m1;
  int cleft;  // codes bytes not yet issued
  int gleft;  // groups not yet issued
  int pm;     // matrix of the segment
};

// Consume one warp segment from the ring: cells in order, lane j taking cell j of each step
// of 32 cells, SPS steps per ring slot. `issue(slot)` refills a consumed slot (whole warp).
// AM: also keep this lane's best (fp16 value, row) among the rows it completes, for the fused
// argmax (ties to the lowest row).
template <int BITS, int MT, bool AM, class Issue>
__device__ __forceinline__ void consume(const Seg& seg, const StreamMat& M, uint32_t xb, uint32_t lut, uint32_t ring,
                                        uint32_t bars, int slots, int& cslot, uint32_t& cphase, int& consumed,
                                        bool& dead, int& dead_at, uint32_t max_polls, Issue& issue, int lane,
                                        float& bv, int& bi) {
  using F = Fmt<BITS>;
  const int G = M.K / kGroup;
  const int ncells = seg.groups;
  const int nsteps = (ncells + 31) / 32;
  const int nslots = (nsteps + F::SPS - 1) / F::SPS;
  uint16_t* y = M.y + seg.row0;
  // the matrix's last partial 16-byte unit of each metadata array, if this segment ends there:
  // loaded now, stored into its ring slot before that slot is read (a unit holds 16 / MB0
  // cells of array 0: 8, or 4 for HIER; array 1, where present, has MB1 = MB0 = 2)
  const int rem = ncells & (16 / F::MB0 - 1);
  // ternary rows are 26 K / 128 bytes: a segment at the end of a matrix may end inside a
  // 16-byte unit; those last bytes are loaded here too
  const int crem = F::TRN ? (int)(seg.bytes & 15) : 0;
  uint32_t cr = 0;
  if (F::TRN && crem && lane >= 16 && lane < 16 + crem)
    cr = __ldg(seg.codes + (seg.bytes & ~(int64_t)15) + (lane - 16));
  uint32_t rs = 0;
  uint16_t rz = 0;
  if (rem) {
    const int gb = ncells - rem;
    if (lane < rem) {
      if constexpr (F::MB0 == 4) rs = __ldg(reinterpret_cast<const uint32_t*>(seg.m0) + gb + lane);
      else rs = ld_u16(reinterpret_cast<const uint16_t*>(seg.m0) + gb + lane);
    }
    if (F::MB1 && lane >= 8 && lane < 8 + rem) rz = ld_u16(reinterpret_cast<const uint16_t*>(seg.m1) + gb + lane - 8);
  }
  // group gp of row `row` of the segment: this lane's cell
  const uint32_t gmul = ((1u << 20) + G - 1) / G;  // floor(n / G) = (n * gmul) >> 20 for n < G + 32, G < 32
  int row = G >= 32 ? 0 : (int)(((uint32_t)lane * gmul) >> 20);
  int gp = lane - row * G;
  const uint32_t xs = (uint32_t)(G * F::XU * 16);  // bytes between the staged rows of X
  float carry[MT];  // per row of X: part of the row of W that continues from the previous step
#pragma unroll
  for (int m = 0; m < MT; ++m) carry[m] = 0.f;
  for (int k = 0; k < nslots; ++k) {
    const uint32_t slot = ring + cslot * F::SLOT;
    if (!dead) {
      const bool ok = mbar_wait_n(bars + 8 * cslot, cphase, max_polls);
      if (!__all_sync(0xffffffffu, ok)) {
        dead = true;
        dead_at = consumed;  // the copy this wait was for never completed
      }
    }
    if (F::TRN && crem && k == nslots - 1) {
      const int cl = (int)(seg.bytes & ~(int64_t)15) - k * F::SC;  // slot offset of the tail
      if (lane >= 16 && lane < 16 + crem)
        asm volatile("st.shared.u8 [%0], %1;" ::"r"(slot + cl + lane - 16), "r"(cr));
      tc::fence_proxy_async_smem();
      __syncwarp();
    }
    if (rem && k == nslots - 1) {
      const int gl = ncells - rem - k * F::GPSL;
      if (lane < rem) {
        if constexpr (F::MB0 == 4)
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(slot + F::SC + 4 * (gl + lane)), "r"(rs));
        else
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(slot + F::SC + 2 * (gl + lane)), "h"((uint16_t)rs));
      }
      if (F::MB1 && lane >= 8 && lane < 8 + rem)
        asm volatile("st.shared.u16 [%0], %1;" ::"r"(slot + F::SC + F::META0 + 2 * (gl + lane - 8)), "h"(rz));
      tc::fence_proxy_async_smem();  // the slot is refilled by bulk copies later
      __syncwarp();
    }
    const uint32_t cell0 = slot + lane * F::CB, meta0 = slot + F::SC + F::MB0 * lane;
#pragma unroll
    for (int ss = 0; ss < F::SPS; ++ss) {
      const int st = k * F::SPS + ss;
      if (F::SPS > 1 && st >= nsteps) break;
      const bool valid = st * 32 + lane < ncells;
      float v[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) v[m] = 0.f;
      if constexpr (F::HR) {
        if (valid && !dead) {
          // the row's pair (d, dm): read here, used after the cell's products
          const uint32_t pr = __ldg(reinterpret_cast<const uint32_t*>(M.scale) + seg.row0 + row);
          uint32_t ib;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(ib) : "r"(meta0 + 32 * F::MB0 * ss));
          const int rot = xrot<BITS>(gp);
          int oc[4], ox[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            oc[c] = 16 * (c ^ rot);
            ox[c] = 16 * F::UPC * c;
          }
          float Pv[MT], Qv[MT];
          cell_dot_hier<MT>(cell0 + 32 * F::CB * ss, xb + 16 * F::XU * gp, xs, oc, ox, rot, ib, Pv, Qv);
          const float d24 = __half2float(__ushort_as_half(lo16(pr))) * 16777216.f;  // 2^24 back, exactly
          const float dm = __half2float(__ushort_as_half(hi16(pr)));
#pragma unroll
          for (int m = 0; m < MT; ++m) v[m] = fmaf(Pv[m], d24, -(Qv[m] * dm));
        }
      } else if (valid && !dead) {
        const uint16_t sb = lds16(meta0 + 64 * ss);
        if constexpr (F::TRN) {
          cell_dot_ternary<MT>(cell0 + 32 * F::CB * ss, xb + 16 * F::XU * gp, xs, lut, v);
          const float sf = __half2float(__ushort_as_half(sb)) * 16777216.f;  // 2^24 back, exactly
#pragma unroll
          for (int m = 0; m < MT; ++m) v[m] *= sf;
        } else {
        const uint16_t zb = lds16(meta0 + 64 * ss + F::META0);
        if constexpr (BITS == 3) {
          cell_dot_int3<MT>(cell0 + 32 * F::CB * ss, xb + 16 * F::XU * gp, xs, zb, v);
          const float s24 = __half2float(__ushort_as_half(sb)) * 16777216.f;
#pragma unroll
          for (int m = 0; m < MT; ++m) v[m] *= s24;
        } else {
        // chunks in an order permuted by the group index, so that the lanes of one
        // shared-memory phase (consecutive cells) hit different bank groups; the staged
        // activations of each group are stored in that same order (see stage_x), so the
        // x chunk read at step c is always the c-th stored one, and lanes that hold the same
        // group index (of different rows) read the same activations, which is a broadcast
        const int rot = xrot<BITS>(gp);
        int oc[F::CH], ox[F::CH];
#pragma unroll
        for (int c = 0; c < F::CH; ++c) {
          oc[c] = 16 * (c ^ rot);
          ox[c] = 16 * F::UPC * c;
        }
        // the cell's sum carries a factor 2^-24; the scale times 2^24 takes it back (exactly)
        cell_dot<BITS, MT>(cell0 + 32 * F::CB * ss, xb + 16 * F::XU * gp, xs, oc, ox, zb, v);
        const float s24 = __half2float(__ushort_as_half(sb)) * 16777216.f;
#pragma unroll
        for (int m = 0; m < MT; ++m) v[m] *= s24;
        }
        }
      }
      // segmented inclusive scan over the lanes of each row within this step
      const int lim = gp < lane ? gp : lane;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float u = __shfl_up_sync(0xffffffffu, v[m], off);
          if (off <= lim) v[m] += u;
        }
      }
      const int gp31 = __shfl_sync(0xffffffffu, gp, 31);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float total = gp > lane ? v[m] + carry[m] : v[m];  // rows begun earlier add the carry
        if (valid && gp == G - 1 && !dead) {
          const __half h = __float2half_rn(total);
          if (M.y) y[(size_t)m * M.N + row] = __half_as_ushort(h);
          if (AM) {
            const float hv = __half2float(h);
            const int r = seg.row0 + row;
            if (hv > bv || (hv == bv && r < bi)) {
              bv = hv;
              bi = r;
            }
          }
        }
        const float t31 = __shfl_sync(0xffffffffu, total, 31);
        carry[m] = gp31 == G - 1 ? 0.f : t31;
      }
      // advance to the cell 32 further on
      gp += 32;
      if (G >= 32) {
        if (gp >= G) {
          gp -= G;
          ++row;
        }
      } else {
        const int wr = (int)(((uint32_t)gp * gmul) >> 20);
        gp -= wr * G;
        row += wr;
      }
    }
    __syncwarp();  // every lane is done reading the slot: refill it
    ++consumed;
    if (!dead) issue(cslot);
    if (++cslot == slots) {
      cslot = 0;
      cphase ^= 1u;
    }
  }
}

// Better of two (value, row) candidates of the fused argmax: larger value, then lower row.
__device__ __forceinline__ void am_take(float& bv, int& bi, float v, int i) {
  if (v > bv || (v == bv && i < bi)) {
    bv = v;
    bi = i;
  }
}

template <int BITS, int MT, int CAP, bool AM>
__global__ void __launch_bounds__(T, kStreamMaxCtasPerSm) gemv_stream_kernel(const __grid_constant__ StreamParamsT<CAP> P) {
  using F = Fmt<BITS>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slots = P.slots;
  const uint32_t sbase = tc::smem_u32(smem);
  const uint32_t ring = sbase + w * slots * F::SLOT;
  const uint32_t bars = sbase + W * slots * F::SLOT + 8 * w * slots;
  const uint32_t xbase = sbase + W * slots * (F::SLOT + 8);
  const uint32_t lut = xbase + P.xbufs * P.xbuf_bytes;  // ternary byte -> trits table
  if constexpr (F::TRN) {
    for (int e = threadIdx.x; e < 256; e += T) {
      uint32_t d[5] = {1, 1, 1, 1, 1};  // digit 1 = trit 0 (also for the invalid bytes)
      if (e < 243) {
        int b = e;
        for (int i = 0; i < 5; ++i, b /= 3) d[i] = (uint32_t)(b % 3);
      }
      const uint32_t word = d[0] | d[1] << 16 | d[2] << 2 | d[3] << 18 | d[4] << 4;
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(lut + 4 * e), "r"(word) : "memory");
    }
  }

  const int64_t share = (P.total_cost + gridDim.x - 1) / gridDim.x;
  const int64_t lo = share * blockIdx.x, hi = lo + share;

  // first matrix that ends after lo (matrices are in cost order)
  int mfirst = 0;
  for (int a = 0, b = P.count; a < b;) {
    const int c = (a + b) >> 1;
    if (P.m[c].cost_end <= lo) a = mfirst = c + 1;
    else b = c;
  }

  // ---- producer: the warp's segments, in matrix order, as ring slots (state kept by every
  // lane alike; lane 0 issues the codes and metadata copies of a slot)
  Prod pd;
  pd.cleft = 0;
  pd.pm = mfirst - 1;
  int issued = 0, consumed = 0, dead_at = -1;
  bool dead = false;  // a bounded wait gave up: stop computing, drain, report
  // failure-detection test hook: CTA 0's warp 0 never fills its first ring slot
  const bool skip_first = P.skip_first_copy && blockIdx.x == 0 && w == 0;
  auto issue = [&](int slot) {
    while (pd.cleft == 0) {  // next non-empty segment of this warp
      if (++pd.pm >= P.count) return;
      const StreamMat& M = P.m[pd.pm];
      if (M.cost_begin >= hi) {
        pd.pm = P.count;
        return;
      }
      int b0, b1;
      cta_units(M, lo, hi, b0, b1);
      const Seg sg = warp_seg<BITS>(M, b0, b1, w);
      pd.c = sg.codes;
      pd.m0 = sg.m0;
      pd.m1 = sg.m1;
      pd.cleft = sg.bytes;
      pd.gleft = sg.groups;
    }
    const uint32_t bar = bars + 8 * slot, dst = ring + slot * F::SLOT;
    int cb = F::SC, gc = F::GPSL;
    if (pd.cleft < F::SC) {
      cb = pd.cleft;
      gc = pd.gleft;
    }
    // whole 16-byte units of the metadata arrays (and, for ternary, of codes); the rest, at
    // the end of a matrix, is loaded by the consumer lanes
    const uint32_t units = (uint32_t)(gc & ~(16 / F::MB0 - 1));  // cells in whole units
    const uint32_t mb0 = F::MB0 * units, mb1 = F::MB1 * units;
    const uint32_t cbb = (uint32_t)cb & ~15u;
    // one lane issues the slot's copies: their operands live in uniform registers, so copies
    // with different operands from several lanes would be issued one lane at a time anyway
    if (lane == 0 && !(skip_first && issued == 0)) {
      tc::mbar_arrive_expect_tx(bar, cbb + mb0 + mb1);
      bulk_g2s(dst, pd.c, cbb, bar);
      if (mb0) bulk_g2s(dst + F::SC, pd.m0, mb0, bar);
      if (F::MB1 && mb1) bulk_g2s(dst + F::SC + F::META0, pd.m1, mb1, bar);
    }
    pd.c += cb;
    pd.m0 += F::MB0 * gc;
    pd.m1 += F::MB1 * gc;
    pd.cleft -= cb;
    pd.gleft -= gc;
    ++issued;
  };
  if (lane == 0) {
    for (int s = 0; s < slots; ++s) tc::mbar_init(bars + 8 * s, 1);
    tc::fence_mbar_init();
  }
  __syncwarp();
  for (int s = 0; s < slots; ++s) issue(s);

  // ---- consumer
  int cslot = 0;
  uint32_t cphase = 0;
  auto cta_next = [&](int from) -> int {
    for (int mi = from; mi < P.count; ++mi) {
      const StreamMat& M = P.m[mi];
      if (M.cost_begin >= hi) return P.count;
      if (M.cost_end <= lo) continue;
      int b0, b1;
      cta_units(M, lo, hi, b0, b1);
      if (b0 < b1) return mi;
    }
    return P.count;
  };
  // activations, row by row of X: the 16 units (8 fp16 each) of group g at units
  // 17 g .. 17 g + 15 of the row, its chunks (UPC units each) in the order of the group's
  // chunk permutation
  auto stage_x = [&](const StreamMat& M, uint32_t xb) {
    if constexpr (F::TRN) {
      // ternary: unit j of group g holds x[128 g + 5 j .. + 4] (three values in unit 25);
      // 10-byte pieces, so plain loads and stores (made visible by the caller's barrier)
      const int G = M.K / kGroup, per = G * 26;
      for (int t = threadIdx.x; t < MT * per; t += T) {
        const int m = t / per, r = t - m * per, g = r / 26, j = r - g * 26;
        const uint16_t* src = M.x + (size_t)m * M.K + kGroup * g + 5 * j;
        uint32_t h[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) h[i] = (5 * j + i < kGroup) ? (uint32_t)__ldg(src + i) : 0u;
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(xb + 16 * (m * G * F::XU + F::XU * g + j)),
                     "r"(h[0] | h[1] << 16), "r"(h[2] | h[3] << 16), "r"(h[4]), "r"(0u)
                     : "memory");
      }
      return;
    }
    const int units = M.K / 8, rowu = (M.K / kGroup) * F::XU;
    for (int t = threadIdx.x; t < MT * units; t += T) {
      const int m = t / units, u = t - m * units;
      const int g = u >> 4, lc = (u & 15) / F::UPC, i = u & (F::UPC - 1);
      // int3: natural order (its cells need no chunk permutation)
      const int pu = BITS == 3 ? m * rowu + F::XU * g + (u & 15) : m * rowu + F::XU * g + F::UPC * (lc ^ xrot<BITS>(g)) + i;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(xb + 16 * pu), "l"(M.x + (size_t)8 * t)
                   : "memory");
    }
    cp_async_commit();
    if constexpr (F::HR) {
      // the sums of x over each group of 32, as binary32, in the spare unit 16 of the
      // group's 17 (four per 128-weight cell, in group order)
      const int ng = M.K / 32;
      for (int t = threadIdx.x; t < MT * ng; t += T) {
        const int m = t / ng, j = t - m * ng;
        const uint4* src = reinterpret_cast<const uint4*>(M.x + (size_t)m * M.K + 32 * j);
        float sum = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint4 q = __ldg(src + u);
          const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            sum += __half2float(__ushort_as_half(lo16(qw[e]))) + __half2float(__ushort_as_half(hi16(qw[e])));
        }
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(xb + 16 * (m * rowu + F::XU * (j >> 2) + 16) + 4 * (j & 3)),
                     "f"(sum)
                     : "memory");
      }
    }
  };

  float am_v = -INFINITY;  // fused argmax: this lane's best fp16 value and its row
  int am_i = INT_MAX;
  int mi = cta_next(mfirst);
  if (P.xbufs == 2 && mi < P.count) stage_x(P.m[mi], xbase);
  for (int xi = 0; mi < P.count; mi = cta_next(mi + 1), ++xi) {
    const StreamMat& M = P.m[mi];
    const uint32_t xb = xbase + (P.xbufs == 2 ? (xi & 1) : 0) * P.xbuf_bytes;
    if (P.xbufs == 1) {
      __syncthreads();  // everyone is done with the previous vector
      stage_x(M, xb);
    }
    cp_async_wait_all();
    __syncthreads();  // this matrix's vector is staged; the other buffer is free
    {
      const int nx = cta_next(mi + 1);
      if (nx < P.count) {
        if (P.xbufs == 2) {
          stage_x(P.m[nx], xbase + ((xi + 1) & 1) * P.xbuf_bytes);
        } else {  // one buffer: have the next vector waiting in L2 when it is staged
          const int lines = MT * P.m[nx].K / 64;
          for (int l = threadIdx.x; l < lines; l += T)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(P.m[nx].x + 64 * l));
        }
      }
    }
    int b0, b1;
    cta_units(M, lo, hi, b0, b1);
    const Seg seg = warp_seg<BITS>(M, b0, b1, w);
    if (seg.rows > 0)
      consume<BITS, MT, AM>(seg, M, xb, lut, ring, bars, slots, cslot, cphase, consumed, dead, dead_at, P.max_polls,
                            issue, lane, am_v,
                            am_i);
  }

  // ---- fused argmax: warp, CTA, then the last CTA to finish combines every CTA's partial
  // (each CTA publishes its partial, fences, takes a ticket; the holder of the last ticket
  // reads them all and resets the ticket counter for the next call)
  if (AM) {
    __shared__ float s_v[W];
    __shared__ int s_i[W];
    __shared__ int s_last;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      am_take(am_v, am_i, __shfl_xor_sync(0xffffffffu, am_v, off), __shfl_xor_sync(0xffffffffu, am_i, off));
    if (lane == 0) {
      s_v[w] = am_v;
      s_i[w] = am_i;
    }
    __syncthreads();
    float* part = reinterpret_cast<float*>(P.am_ws + 4);
    if (threadIdx.x == 0) {
      float v = s_v[0];
      int i = s_i[0];
      for (int k = 1; k < W; ++k) am_take(v, i, s_v[k], s_i[k]);
      part[2 * blockIdx.x] = v;
      reinterpret_cast<int*>(part)[2 * blockIdx.x + 1] = i;
      __threadfence();
      s_last = atomicAdd(P.am_ws, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      float v = -INFINITY;
      int i = INT_MAX;
      for (int b = threadIdx.x; b < (int)gridDim.x; b += T)
        am_take(v, i, __ldcg(part + 2 * b), __ldcg(reinterpret_cast<const int*>(part) + 2 * b + 1));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        am_take(v, i, __shfl_xor_sync(0xffffffffu, v, off), __shfl_xor_sync(0xffffffffu, i, off));
      __syncthreads();  // s_v / s_i are reused
      if (lane == 0) {
        s_v[w] = v;
        s_i[w] = i;
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        for (int k = 1; k < W; ++k) am_take(s_v[0], s_i[0], s_v[k], s_i[k]);
        *P.am_out = s_i[0];
        *P.am_ws = 0u;  // ticket counter back to zero for the next call
      }
    }
  }

  // ---- error path: report, then wait (bounded) for copies still landing in this CTA
  // (dead is warp-uniform); every copy issued after the wait that gave up is waited for, with
  // the same bound, so that none is still landing in this CTA's shared memory when it exits
  if (dead) {
    if (lane == 0) {
      atomicOr(P.errors, tc::kErrTimeout);
      for (int j = dead_at + 1; j < issued; ++j)
        mbar_wait_n(bars + 8 * (j % slots), (uint32_t)((j / slots) & 1), P.max_polls);
    }
    __syncwarp();
  }
}

int gcd_int(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

template <int BITS>
int plan_t(StreamParams& p, int count, const StreamDesc* d, int mt) {
  using F = Fmt<BITS>;
  int64_t cost = 0;
  int max_k = 0;
  for (int i = 0; i < count; ++i) {
    // bulk-copied arrays 16-byte aligned; HIER row pairs are read as 4-byte words
    const uintptr_t bulk = (uintptr_t)d[i].codes | (uintptr_t)d[i].zero | (uintptr_t)d[i].x |
                           (F::HR ? 0 : (uintptr_t)d[i].scale);
    if ((bulk & 15) != 0 || (F::HR && ((uintptr_t)d[i].scale & 3) != 0)) return 0;
    const int K = (int)d[i].K, N = (int)d[i].N;
    const int G = K / kGroup;
    // rows per unit: segments start at multiples of RA rows, so that their metadata starts
    // on a 16-byte boundary (a unit of 16 / MB0 cells)
    const int RA = (16 / F::MB0) / gcd_int(G, 16 / F::MB0);
    const int64_t row_cost = (int64_t)G * (F::CB + F::MB0 + F::MB1) + (F::HR ? 4 : 0);
    StreamMat& m = p.m[i];
    m.codes = d[i].codes;
    m.scale = d[i].scale;
    m.zero = d[i].zero;
    m.x = d[i].x;
    m.y = d[i].y;
    m.N = N;
    m.K = K;
    m.RA = RA;
    m.nunit = (N + RA - 1) / RA;
    m.unit_cost = RA * row_cost;
    m.inv_unit_cost = 1.0 / (double)m.unit_cost;
    m.cost_begin = cost;
    cost += (int64_t)N * row_cost;
    m.cost_end = cost;
    if (K > max_k) max_k = K;
  }
  p.count = count;
  p.total_cost = cost;
  p.am_ws = nullptr;
  p.am_out = nullptr;
  p.xbuf_bytes = (mt * (max_k / kGroup) * F::XU * 16 + 127) & ~127;
  p.errors = device_error_word();
  if (!p.errors) return 0;
  p.max_polls = tc::kMaxPolls;
  p.skip_first_copy = 0;
  // kStreamSlots ring slots per warp; two activation buffers when four CTAs still fit on an
  // SM (measured best on the 0.5B decode set), else one; then as many CTAs as fit
  const int ring = W * kStreamSlots * (F::SLOT + 8) + F::LUT;
  const int two = ring + 2 * p.xbuf_bytes, one = ring + p.xbuf_bytes;
  const int bytes = (kStreamSmPool / (two + 1024) >= kStreamMaxCtasPerSm) ? two : one;
  if (bytes > kStreamMaxSmem) return 0;
  p.slots = kStreamSlots;
  p.xbufs = bytes == two ? 2 : 1;
  const int fit = kStreamSmPool / (bytes + 1024);
  p.ctas_per_sm = fit < kStreamMaxCtasPerSm ? fit : kStreamMaxCtasPerSm;
  return bytes;
}

template <int BITS, int MT, int CAP, bool AM = false>
cudaError_t launch_cap(const StreamParamsT<CAP>& p, int smem, cudaStream_t stream) {
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(gemv_stream_kernel<BITS, MT, CAP, AM>, kStreamMaxSmem, configured);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  if (sms == 0) return cudaErrorInvalidDevice;
  gemv_stream_kernel<BITS, MT, CAP, AM><<<p.ctas_per_sm * sms, T, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int BITS, int MT, int CAP, bool AM = false>
cudaError_t launch_copy(const StreamParams& p, int smem, cudaStream_t stream) {
  static thread_local StreamParamsT<CAP> q;
  q.am_ws = p.am_ws;
  q.am_out = p.am_out;
  q.errors = p.errors;
  q.total_cost = p.total_cost;
  q.count = p.count;
  q.slots = p.slots;
  q.xbufs = p.xbufs;
  q.ctas_per_sm = p.ctas_per_sm;
  q.xbuf_bytes = p.xbuf_bytes;
  q.max_polls = p.max_polls;
  q.skip_first_copy = p.skip_first_copy;
  for (int i = 0; i < p.count; ++i) q.m[i] = p.m[i];
  return launch_cap<BITS, MT, CAP, AM>(q, smem, stream);
}

template <int BITS, int MT>
cudaError_t launch_t(const StreamParams& p, int smem, cudaStream_t stream) {
  // size the parameter block to the set: a launch copies its whole parameter block
  if (p.count <= 1) return launch_copy<BITS, MT, 1>(p, smem, stream);
  if (MT == 1 && p.count <= 64) return launch_copy<BITS, MT, 64>(p, smem, stream);
  return launch_cap<BITS, MT, kStreamMaxMats>(p, smem, stream);
}

template <int BITS>
cudaError_t launch_b(const StreamParams& p, int mt, int smem, cudaStream_t stream) {
  switch (mt) {
    case 1: return launch_t<BITS, 1>(p, smem, stream);
    case 2: return launch_t<BITS, 2>(p, smem, stream);
    case 3: return launch_t<BITS, 3>(p, smem, stream);
    default: return launch_t<BITS, 4>(p, smem, stream);
  }
}

}  // namespace

int stream_plan(StreamParams& p, int bits, int count, const StreamDesc* d, int mt) {
  if (count < 1 || count > kStreamMaxMats || mt < 1 || mt > kStreamMaxRows) return 0;
  switch (bits) {
    case 4: return plan_t<4>(p, count, d, mt);
    case 3: return plan_t<3>(p, count, d, mt);
    case 2: return plan_t<2>(p, count, d, mt);
    case HIER: return plan_t<HIER>(p, count, d, mt);
    default: return plan_t<TERN>(p, count, d, mt);
  }
}

cudaError_t launch_gemv_stream(const StreamParams& p, int bits, int mt, int smem, cudaStream_t stream) {
  switch (bits) {
    case 4: return launch_b<4>(p, mt, smem, stream);
    case 3: return launch_b<3>(p, mt, smem, stream);
    case 2: return launch_b<2>(p, mt, smem, stream);
    case HIER: return launch_b<HIER>(p, mt, smem, stream);
    default: return launch_b<TERN>(p, mt, smem, stream);
  }
}

cudaError_t launch_gemv_stream_argmax(const StreamParams& p, int bits, int smem, cudaStream_t stream) {
  switch (bits) {
    case 4: return launch_copy<4, 1, 1, true>(p, smem, stream);
    case HIER: return launch_copy<HIER, 1, 1, true>(p, smem, stream);
    default: return launch_copy<2, 1, 1, true>(p, smem, stream);
  }
}

int stream_grid(const StreamParams& p) { return p.ctas_per_sm * device_sm_count(); }

}  // namespace wq
