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
// Work: one CTA of 16 warps per SM. CTA b takes the contiguous range of slabs (16 rows x all
// of K) whose cost (128-weight groups) falls in its 1/gridDim share of the set, walked in
// windows: warp w takes slabs w, w + 16, ... of a window (up to 8 each when the matrix's
// activations fit one chunk; one when they need several, whose sums stay in registers
// across the chunks). The activations of a window are staged in shared memory with cp.async
// in chunks of up to kc groups (two buffers), restaged only when the matrix or the chunk
// changes. Codes travel through a per-thread cp.async ring in shared memory, several groups
// deep, with a 256-byte L2 fetch size so that a row's next groups come with the current one;
// the thread's copies form one commit group per compute step, and a restaged chunk's copies
// ride in the group of the item's first step, so the per-step waits cover them too. Each
// lane loads one of its lane group's four scale / zero values one step ahead; shuffles share
// them.
#include <climits>

#include "common.cuh"
#include "gemm_skinny.cuh"
#include "host_util.cuh"

namespace wq {

namespace {



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

// Per-step ring traffic: these statements are volatile, so they keep their order among
// themselves (copy, commit, wait, read back); they carry no memory clobber, so that the
// compiler may schedule the step's other work across them. (The activation buffer a step
// reads is never the one being written; restaging is ordered by barriers.)
__device__ __forceinline__ void cp_async16_l2(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(dst), "l"(src));
}

__device__ __forceinline__ void cp_async_commit_step() { asm volatile("cp.async.commit_group;"); }

template <int RING>
__device__ __forceinline__ void cp_async_wait_step() { asm volatile("cp.async.wait_group %0;" ::"n"(RING - 1)); }

__device__ __forceinline__ uint4 lds_ring(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// wait until at most n (0 <= n < 6) of this thread's newest copy groups are pending
__device__ __forceinline__ void cp_async_wait_upto(int n) {
  if (n <= 0) cp_async_wait<0>();
  else if (n == 1) cp_async_wait<1>();
  else if (n == 2) cp_async_wait<2>();
  else if (n == 3) cp_async_wait<3>();
  else if (n == 4) cp_async_wait<4>();
  else cp_async_wait<5>();
}

// d = A * B with a zero accumulator (first MMA of a group)
__device__ __forceinline__ void mma16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// A position in a CTA's work: item = window [ws, we) of slabs of matrix mi (warp w takes
// slabs ws + w, ws + w + 16, ...) and activation chunk ch (groups g0 .. g0 + ng - 1).
struct Walk {
  int ws, we, mi, ch, g0, ng, gl;
};

template <int CAP>
__device__ __forceinline__ void item_fill(const SkParamsT<CAP>& P, Walk& w, int hi) {
  const SkMat& m = P.m[w.mi];
  w.we = min(min(w.ws + m.span, m.slab_end), hi);
  w.g0 = w.ch * m.kc;
  w.ng = min(m.kc, m.G - w.g0);
}

// the next item (ch + 1, or the next window); false past the CTA's last slab
template <int CAP>
__device__ __forceinline__ bool item_next(const SkParamsT<CAP>& P, Walk& w, int hi) {
  if (w.ch + 1 < P.m[w.mi].nch) {
    ++w.ch;
  } else {
    w.ws = w.we;
    if (w.ws >= hi) return false;
    while (w.ws >= P.m[w.mi].slab_end) ++w.mi;
    w.ch = 0;
  }
  item_fill(P, w, hi);
  return true;
}

// first slab whose cost position is >= c (slab j of matrix i sits at cost_begin_i + j G_i)
template <int CAP>
__device__ __forceinline__ int slab_at(const SkParamsT<CAP>& P, int64_t c) {
  if (c >= P.total_cost) return P.total_slabs;
  int lo = 0, hi = P.count - 1;
  while (lo < hi) {  // last matrix with cost_begin <= c
    const int mid = (lo + hi + 1) >> 1;
    if (P.m[mid].cost_begin <= c) lo = mid; else hi = mid - 1;
  }
  const SkMat& m = P.m[lo];
  return m.slab_begin + (int)((c - m.cost_begin + m.G - 1) / m.G);
}

template <int CAP>
__device__ __forceinline__ int mat_of_slab(const SkParamsT<CAP>& P, int s) {
  int lo = 0, hi = P.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.m[mid].slab_begin <= s) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace

template <int TB, int CAP>
__global__ void __launch_bounds__(kSkThreads, 1) gemm_skinny_kernel(const __grid_constant__ SkParamsT<CAP> P) {
  constexpr int kRing = sk_ring(TB);
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = P.M;
  constexpr int NT = 8 * TB;                  // staged token rows (rows past M are never read
  constexpr int TPT = kSkThreads / NT;        // into a stored output)
  const int stage_n = tid / TPT, stage_c0 = tid % TPT;
  constexpr uint32_t kSlot = 2u * kSkThreads * 16u;   // ring slot: [row g | row g + 8][thread][16 B]
  const uint32_t ring_me = sbase + 2u * (uint32_t)P.buf_bytes + 16u * (uint32_t)tid;

  // this CTA's slabs: a contiguous range of about equal cost
  const int64_t C = P.total_cost;
  const int lo = slab_at(P, C * blockIdx.x / gridDim.x);
  const int hi = slab_at(P, C * (blockIdx.x + 1) / gridDim.x);
  if (lo >= hi) return;

  auto stage_x = [&](const Walk& it, int b) {
    if (stage_n < M) {
      const SkMat& m = P.m[it.mi];
      const uint32_t row = sbase + (uint32_t)b * (uint32_t)P.buf_bytes + (uint32_t)stage_n * ((uint32_t)m.kc * 256u + 16u);
      const uint16_t* src = m.x + (size_t)stage_n * m.K + (size_t)it.g0 * kGroup;
      for (int c = stage_c0; c < 16 * it.ng; c += TPT) cp_async16(row + xchunk_off((uint32_t)c), src + 8 * c);
    }
  };

  Walk it;
  it.ws = lo;
  it.mi = mat_of_slab(P, lo);
  it.ch = 0;
  it.gl = 0;
  item_fill(P, it, hi);
  stage_x(it, 0);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // Fetch cursor (kRing - 1 steps ahead of the compute) and metadata cursor (one step
  // ahead) over this warp's steps: items in order, in each the warp's slabs in order, in each
  // slab the chunk's groups. Each keeps the source of its next step in registers and the
  // steps left in its slab; the slab and item bookkeeping runs only when that count runs out.
  Walk f = it;
  bool fv = true;
  while (warp >= f.we - f.ws)
    if (!item_next(P, f, hi)) { fv = false; break; }
  Walk sc = f;
  bool sv = fv;
  int fs = f.ws + warp, ss = fs;  // the cursors' current slabs
  const uint8_t* fp_lo = nullptr;
  const uint8_t* fp_hi = nullptr;
  int f_left = 0;  // steps left in the fetch cursor's slab (0: no more steps)
  auto fetch_slab = [&]() {
    const SkMat& m = P.m[f.mi];
    const int r0 = (fs - m.slab_begin) * 16 + g;
    fp_lo = m.codes + (size_t)min(r0, m.N - 1) * (m.K / 2) + (size_t)f.g0 * 64 + 16 * t;
    fp_hi = m.codes + (size_t)min(r0 + 8, m.N - 1) * (m.K / 2) + (size_t)f.g0 * 64 + 16 * t;
    f_left = f.ng;
  };
  if (fv) fetch_slab();
  const uint32_t ring_first = ring_me, ring_last = ring_me + (uint32_t)(kRing - 1) * kSlot;
  uint32_t fslot = ring_first, cslot = ring_first;
  auto fetch = [&]() {
    if (f_left > 0) {
      cp_async16_l2(fslot, fp_lo);
      cp_async16_l2(fslot + kSlot / 2, fp_hi);
      fp_lo += 64;
      fp_hi += 64;
      if (--f_left == 0) {
        fs += kSkWarps;
        if (fs >= f.we) {
          f.gl = 0;
          do {
            if (!item_next(P, f, hi)) { fv = false; break; }
          } while (warp >= f.we - f.ws);
          fs = f.ws + warp;
        }
        if (fv) fetch_slab();
      }
    }
    cp_async_commit_step();
    fslot = fslot == ring_last ? ring_first : fslot + kSlot;
  };
#pragma unroll 1
  for (int d = 0; d < kRing - 1; ++d) fetch();

  // Metadata: lane (g, t) loads one value per step (t = 0, 1: scale of row g, g + 8;
  // t = 2, 3: zero of row g, g + 8), one step ahead; shuffles within the lane group hand
  // each lane all four.
  const uint16_t* mp = nullptr;
  int m_left = 0;
  auto meta_slab = [&]() {
    const SkMat& m = P.m[sc.mi];
    const int r = min((ss - m.slab_begin) * 16 + g + ((t & 1) ? 8 : 0), m.N - 1);
    mp = ((t & 2) ? m.zero : m.scale) + (size_t)r * m.G + sc.g0;
    m_left = sc.ng;
  };
  uint32_t nmeta = 0;
  auto load_meta = [&]() {
    if (m_left > 0) {
      nmeta = ld_u16(mp);
      ++mp;
      if (--m_left == 0) {
        ss += kSkWarps;
        if (ss >= sc.we) {
          do {
            if (!item_next(P, sc, hi)) { sv = false; break; }
          } while (warp >= sc.we - sc.ws);
          ss = sc.ws + warp;
        }
        if (sv) meta_slab();
      }
    }
  };
  if (sv) meta_slab();
  load_meta();

  uint32_t xoff[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) xoff[w] = xchunk_off((uint32_t)(4 * t + w));

  float acc[TB][4];
#pragma unroll
  for (int b = 0; b < TB; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;
  int buf = 0;

  for (;;) {
    const SkMat& m = P.m[it.mi];
    const int nmine = warp < it.we - it.ws ? (it.we - it.ws - warp + kSkWarps - 1) / kSkWarps : 0;
    Walk nx = it;
    const bool has_next = item_next(P, nx, hi);
    const bool restage = has_next && (nx.mi != it.mi || nx.ch != it.ch);
    if (restage) stage_x(nx, buf ^ 1);  // these copies join this thread's next commit

    if (nmine > 0) {
      const uint32_t ts = (uint32_t)m.kc * 256u + 16u;
      const uint8_t* xrow = smem + (size_t)buf * P.buf_bytes + (size_t)g * ts;
#pragma unroll 1
      for (int k = 0; k < nmine; ++k) {
#pragma unroll 1
        for (int gl = 0; gl < it.ng; ++gl) {
          fetch();
          cp_async_wait_step<kRing>();  // this step's codes have landed
          const uint4 w_lo = lds_ring(cslot), w_hi = lds_ring(cslot + kSlot / 2);
          cslot = cslot == ring_last ? ring_first : cslot + kSlot;
          const uint32_t meta = nmeta;
          load_meta();
          const int q = lane & ~3;
          const uint16_t s_lo = (uint16_t)__shfl_sync(0xFFFFFFFFu, meta, q);
          const uint16_t s_hi = (uint16_t)__shfl_sync(0xFFFFFFFFu, meta, q + 1);
          const uint16_t z_lo = (uint16_t)__shfl_sync(0xFFFFFFFFu, meta, q + 2);
          const uint16_t z_hi = (uint16_t)__shfl_sync(0xFFFFFFFFu, meta, q + 3);
          const float sf_lo = __half2float(__ushort_as_half(s_lo)), sf_hi = __half2float(__ushort_as_half(s_hi));
          const uint32_t zc_lo = neg_zc(z_lo), zc_hi = neg_zc(z_hi);
          float part[TB][4];
          const uint32_t wl[4] = {w_lo.x, w_lo.y, w_lo.z, w_lo.w};
          const uint32_t wh[4] = {w_hi.x, w_hi.y, w_hi.z, w_hi.w};
          const uint8_t* xg = xrow + (size_t)gl * 256;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint32_t a0 = pair_minus_z(wl[w], 0x0000u, zc_lo), a1 = pair_minus_z(wh[w], 0x0000u, zc_hi);
            const uint32_t a2 = pair_minus_z(wl[w], 0x1111u, zc_lo), a3 = pair_minus_z(wh[w], 0x1111u, zc_hi);
            const uint32_t e0 = pair_minus_z(wl[w], 0x2222u, zc_lo), e1 = pair_minus_z(wh[w], 0x2222u, zc_hi);
            const uint32_t e2 = pair_minus_z(wl[w], 0x3333u, zc_lo), e3 = pair_minus_z(wh[w], 0x3333u, zc_hi);
#pragma unroll
            for (int b = 0; b < TB; ++b) {
              const uint4 xv = *reinterpret_cast<const uint4*>(xg + xoff[w] + (size_t)(8 * b) * ts);
              if (w == 0) mma16816_z(part[b], a0, a1, a2, a3, xv.x, xv.y);
              else mma16816(part[b], a0, a1, a2, a3, xv.x, xv.y);
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
        if (it.ch + 1 == m.nch) {
          // C fragment: (row g, tokens 2t, 2t + 1) and (row g + 8, the same tokens)
          const int ra = (it.ws + warp + kSkWarps * k - m.slab_begin) * 16 + g, rb = ra + 8;
#pragma unroll
          for (int b = 0; b < TB; ++b) {
            const int mt = 8 * b + 2 * t;
            if (mt < M) {
              if (ra < m.N) m.y[(size_t)mt * m.N + ra] = __half_as_ushort(__float2half_rn(acc[b][0]));
              if (rb < m.N) m.y[(size_t)mt * m.N + rb] = __half_as_ushort(__float2half_rn(acc[b][2]));
            }
            if (mt + 1 < M) {
              if (ra < m.N) m.y[(size_t)(mt + 1) * m.N + ra] = __half_as_ushort(__float2half_rn(acc[b][1]));
              if (rb < m.N) m.y[(size_t)(mt + 1) * m.N + rb] = __half_as_ushort(__float2half_rn(acc[b][3]));
            }
            acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;
          }
        }
      }
    } else if (restage) {
      cp_async_commit();  // the staging copies alone
    }
    if (!has_next) break;
    if (restage) {
      // This thread's staging copies rode in the group committed at its first step of the
      // item, which the per-step waits have covered once the item had as many of its steps as the ring has slots;
      // otherwise wait for it here. Then every thread's copies are visible after the
      // barrier, and no warp still reads the buffer the next restage will overwrite.
      const int steps = nmine * it.ng;
      if (steps == 0) cp_async_wait<0>();
      else if (steps < kRing) cp_async_wait_upto(steps - 1);
      __syncthreads();
      buf ^= 1;
    }
    it = nx;
  }
  cp_async_wait<0>();
}

// ---- host side -----------------------------------------------------------------------

static int tb_for(int M) { return M <= 8 ? 1 : M <= 16 ? 2 : 4; }

int skinny_plan(SkParams& p, int count, const SkDesc* d, int M) {
  if (count < 1 || count > kSkMaxMats || M < 1 || M > kSkMaxM) return 0;
  const int nt = 8 * tb_for(M);
  // two activation buffers of nt token rows, kc * 256 + 16 bytes each, beside the codes ring
  const int kc_max = (((kSkSmemMax - sk_ring_bytes(tb_for(M))) / 2) / nt - 16) / 256;
  if (kc_max < 1) return 0;
  int64_t slabs = 0, cost = 0;
  int kc_used = 1;
  for (int i = 0; i < count; ++i) {
    const SkDesc& s = d[i];
    if (((uintptr_t)s.codes & 15) || ((uintptr_t)s.x & 15) || ((uintptr_t)s.scale & 1) || !s.zero ||
        ((uintptr_t)s.zero & 1))
      return 0;
    SkMat& m = p.m[i];
    m.codes = static_cast<const uint8_t*>(s.codes);
    m.scale = s.scale;
    m.zero = s.zero;
    m.x = s.x;
    m.y = s.y;
    m.N = (int)s.N;
    m.K = (int)s.K;
    m.G = (int)(s.K / kGroup);
    m.nch = (m.G + kc_max - 1) / kc_max;
    m.kc = (m.G + m.nch - 1) / m.nch;
    m.span = kSkWarps * (m.nch == 1 ? kSkSpanOne : 1);
    kc_used = m.kc > kc_used ? m.kc : kc_used;
    const int64_t ns = (s.N + 15) / 16;
    m.slab_begin = (int)slabs;
    m.cost_begin = cost;
    slabs += ns;
    cost += ns * m.G;
    if (slabs > INT_MAX) return 0;
    m.slab_end = (int)slabs;
  }
  p.count = count;
  p.M = M;
  p.total_slabs = (int)slabs;
  p.total_cost = cost;
  p.buf_bytes = nt * (kc_used * 256 + 16);
  return 2 * p.buf_bytes + sk_ring_bytes(tb_for(M));
}

template <int TB>
static cudaError_t launch_tb(const SkParams& p, int smem, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_limit(gemm_skinny_kernel<TB, kSkMaxMats>, kSkSmemMax, attr_done);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  if (sms == 0) return cudaErrorInvalidDevice;
  const int grid = p.total_slabs < sms ? p.total_slabs : sms;  // one CTA per SM
  gemm_skinny_kernel<TB, kSkMaxMats><<<grid, kSkThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_skinny(const SkParams& p, int smem, cudaStream_t stream) {
  if (smem <= 0 || smem > kSkSmemMax || p.total_slabs < 1) return cudaErrorInvalidValue;
  switch (tb_for(p.M)) {
    case 1: return launch_tb<1>(p, smem, stream);
    case 2: return launch_tb<2>(p, smem, stream);
    default: return launch_tb<4>(p, smem, stream);
  }
}

}  // namespace wq
