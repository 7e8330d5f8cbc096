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
// Warp roles (one persistent CTA of 16 warps per SM; tiles dealt to CTAs as tile_deal.cuh
// describes), per 64-wide k-block:
//   - warp 4 (one lane): TMA loads the activation tile [bn x 64] fp16 (128-byte swizzle) into
//     an XSTAGES-deep ring, completing on xfull[s]; it waits xempty[s] before reusing a stage;
//   - warps 8-15 (two teams of four warps, one weight row per thread, the teams taking
//     alternate k-blocks): copy their rows' packed codes with per-thread cp.async into a
//     CRING-deep ring, dequantise them into fp16 (q - z) * s, store them into the A stage
//     in the 128-byte-swizzled K-major layout the tensor core reads, fence the async proxy
//     and arrive on aready[a] (ASTAGES-deep ring, freed through aempty[a]);
//   - warp 5 (one lane): allocates the tensor memory; per k-block waits xfull[s] and
//     aready[a], issues four m128 x n(bn) x k16 tcgen05 MMAs into the tile's accumulator (two
//     accumulators of 256 columns, alternating tiles) and commits them to xempty[s] and
//     aempty[a]; after a tile's last k-block it commits to tfull[b];
//   - warps 0-3 (epilogue, 32 weight rows each): wait tfull[b], read the accumulator with
//     tcgen05.ld, and store fp16 Y[m, n], through a TMA tensor store of 32 x 32 blocks staged
//     in shared memory when Y's layout allows, else with plain stores; then arrive on
//     tempty[b] so that the MMA lane can reuse that accumulator.
// Every mbarrier wait is bounded; a wait that gives up sets kErrTimeout in the library's
// device error word, and the CTA drains its own TMA loads, frees its TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "host_util.cuh"
#include "tc_ptx.cuh"

namespace wq {

__device__ unsigned int g_device_errors;  // bit flags, read and cleared by wq_device_errors

namespace {

constexpr int BM = 128;       // weight rows per tile
constexpr int BK = 64;        // k per stage: one 128-byte swizzle row of fp16
#ifndef WQ_TC_XSTAGES
#define WQ_TC_XSTAGES 3
#endif
#ifndef WQ_TC_ASTAGES
#define WQ_TC_ASTAGES 4
#endif
#ifndef WQ_TC_CRING
#define WQ_TC_CRING 6
#endif
constexpr int XSTAGES = WQ_TC_XSTAGES;  // activation tiles [bn x 64] (read from L2)
constexpr int CRING = WQ_TC_CRING;      // codes ring slots: CRING - 1 of a team's k-blocks in flight
constexpr int ASTAGES = WQ_TC_ASTAGES;  // dequantised weight tiles (written by CUDA cores, read by MMA)
constexpr int A_BYTES = BM * BK * 2;            // 16 KB of dequantised fp16 weights
#ifndef WQ_TC_XBN
#define WQ_TC_XBN kTcMaxBN
#endif
constexpr int XBN = WQ_TC_XBN;                  // tokens one activation stage holds
constexpr int B_BYTES = XBN * BK * 2;           // activations of one stage
constexpr int CSLOT_BYTES = 2 * BM * BK / 2;   // one ring slot: 32 B of codes for each of 256 threads
constexpr int OFF_A = 0;
constexpr int OFF_X = OFF_A + ASTAGES * A_BYTES;
constexpr int OFF_C = OFF_X + XSTAGES * B_BYTES;
constexpr int EPI_BYTES = 32 * 32 * 2;          // one warp's 32 x 32 fp16 output block
constexpr int OFF_E = OFF_C + CRING * CSLOT_BYTES;  // [4 warps][2 buffers] staged output blocks
constexpr int OFF_BAR = OFF_E + 4 * 2 * EPI_BYTES;
constexpr int NUM_BARS = 2 * XSTAGES + 2 * ASTAGES + 4;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_USED = OFF_MISC + 16;
constexpr int THREADS = 512;                    // 16 warps
constexpr int XPROD_WARP = 4, MMA_WARP = 5, DEQ_WARP0 = 8, DEQ_WARPS = 8, TEAM_WARPS = 4;
constexpr int TMEM_COLS = 2 * kTcMaxBN;         // two accumulator buffers
static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzled operands need 1 KB alignment");
static_assert(SMEM_USED + 1024 <= 232448, "shared memory per block");
static_assert(DEQ_WARPS == 2 * TEAM_WARPS && TEAM_WARPS * 32 == BM, "two teams, one row per thread");

__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_ring() {
  asm volatile("cp.async.wait_group %0;" ::"n"(CRING - 1) : "memory");
}

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

struct SzPair {
  uint16_t s, z;  // fp16 bits of one group's scale and zero
};

struct TileInfo {
  int mi, n0, m0, bn, nkb;
};

template <int CAP>
__device__ __forceinline__ TileInfo tile_info(const TcParamsT<CAP>& P, int tile, int& mi) {
  while (tile >= P.m[mi].tile_end) ++mi;
  const TcMat& M = P.m[mi];
  const int local = tile - M.tile_begin;
  TileInfo t;
  t.mi = mi;
  t.n0 = (local / M.tiles_m) * BM;
  t.m0 = (local % M.tiles_m) * M.bn;
  t.bn = M.bn;
  t.nkb = M.K / BK;
  return t;
}

}  // namespace

// Persistent: CTA b runs its dealt tiles (tile_deal.cuh) in increasing order. Warp roles: 0-3 epilogue (TMEM lanes 32w..32w+31 = weight rows), 4 TMA producer,
// 5 MMA issuer (and TMEM owner), 8-15 dequantisers (two threads per weight row, 32 k each
// per stage); 6-7 idle. The two 256-column TMEM accumulators let the epilogue of one tile
// overlap the main loop of the next.
template <int CAP>
__global__ void __launch_bounds__(THREADS, 1) gemm_tc_int4_kernel(const __grid_constant__ TcParamsT<CAP> P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment of the operand buffers is what the 128-byte swizzle assumes
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  const uint32_t bar_xfull = sbase + OFF_BAR;                 // [XSTAGES] activation tile landed
  const uint32_t bar_xempty = bar_xfull + 8 * XSTAGES;        // [XSTAGES] MMAs reading it done
  const uint32_t bar_aready = bar_xempty + 8 * XSTAGES;       // [ASTAGES] dequantised A written
  const uint32_t bar_aempty = bar_aready + 8 * ASTAGES;       // [ASTAGES] MMAs reading A done
  const uint32_t bar_tfull = bar_aempty + 8 * ASTAGES;        // [2] accumulator complete
  const uint32_t bar_tempty = bar_tfull + 16;                 // [2] accumulator drained
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);  // [0] tmem base, [1] abort

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < XSTAGES; ++i) {
      tc::mbar_init(bar_xfull + 8 * i, 1);
      tc::mbar_init(bar_xempty + 8 * i, 1);
    }
    for (int i = 0; i < ASTAGES; ++i) {
      tc::mbar_init(bar_aready + 8 * i, TEAM_WARPS);
      tc::mbar_init(bar_aempty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(bar_tfull + 8 * i, 1);
      tc::mbar_init(bar_tempty + 8 * i, 4);
    }
    tc::fence_mbar_init();
    misc[1] = 0;
  }
  if (warp == MMA_WARP) {
    tc::tmem_alloc(sbase + OFF_MISC, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = misc[0];

  // this CTA's j-th tile (-1 past its last); the host orders each launch's matrices by tile
  // cost, largest first, and chooses the dealing that evens out the CTAs' total cost
  const TileDeal deal = P.deal;
  const int ctas = gridDim.x, total = P.total_tiles, cta = blockIdx.x;
  auto tile_of = [&](int j) { return dealt_tile(cta, j, ctas, total, deal); };

  bool timed_out = false;
  int it = 0;    // k-block sequence number over this CTA's tiles
  int mi = 0;

  if (warp == XPROD_WARP) {
    // activation tiles, one per k-block
    if (lane == 0) {
      for (int j = 0, tile; (tile = tile_of(j)) >= 0 && !timed_out; ++j) {
        const TileInfo ti = tile_info(P, tile, mi);
        const TcMat& M = P.m[ti.mi];
        const uint32_t tx = (uint32_t)(ti.bn * BK * 2);
        for (int kb = 0; kb < ti.nkb; ++kb, ++it) {
          const int s = it % XSTAGES;
          if (!tc::mbar_wait(bar_xempty + 8 * s, ((it / XSTAGES) & 1) ^ 1)) { timed_out = true; break; }
          if (misc[1]) { timed_out = true; break; }
          tc::mbar_arrive_expect_tx(bar_xfull + 8 * s, tx);
          tc::tma_load_2d(sbase + OFF_X + s * B_BYTES, &M.tmap_x, bar_xfull + 8 * s, kb * BK, ti.m0);
        }
      }
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      int lt = 0;
      for (int j = 0, tile; (tile = tile_of(j)) >= 0 && !timed_out; ++j, ++lt) {
        const TileInfo ti = tile_info(P, tile, mi);
        const int b = lt & 1;
        if (!tc::mbar_wait(bar_tempty + 8 * b, ((lt >> 1) & 1) ^ 1)) { timed_out = true; break; }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * kTcMaxBN);
        const uint32_t idesc = tc::idesc_f16_f32(BM, ti.bn);
        for (int kb = 0; kb < ti.nkb; ++kb, ++it) {
          const int s = it % XSTAGES, a = it % ASTAGES;
          if (!tc::mbar_wait(bar_xfull + 8 * s, (it / XSTAGES) & 1) ||
              !tc::mbar_wait(bar_aready + 8 * a, (it / ASTAGES) & 1)) {
            timed_out = true;
            break;
          }
          tc::tc_fence_after();
          const uint64_t ad = tc::sw128_kmajor_desc(sbase + OFF_A + a * A_BYTES);
          const uint64_t bd = tc::sw128_kmajor_desc(sbase + OFF_X + s * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // +32 bytes along K inside the swizzled row
            tc::mma_f16_ss(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
          tc::mma_commit(bar_xempty + 8 * s);  // frees the activation stage ...
          tc::mma_commit(bar_aempty + 8 * a);  // ... and the dequantised tile
        }
        tc::mma_commit(bar_tfull + 8 * b);  // fires when every MMA of the tile has completed
      }
    }
  } else if (warp >= DEQ_WARP0) {
    // Two teams of four warps; team e dequantises the k-blocks with it % 2 == e, so each
    // warp has two k-block periods for one k-block's work and its fixed costs (waits,
    // fence, arrive) are paid once per 64 k of a row. Thread r of a team owns weight row r.
    const int t = threadIdx.x - 32 * DEQ_WARP0;   // 0 .. 255 (slot of the codes ring)
    const int team = t >> 7, r = t & 127;
    // scale and zero of the team's next two k-blocks (one k-block per 128-k group and team),
    // in separate registers until used: combining them at load time would stall the warp
    // for the whole load latency.
    auto load_sz = [&](const TcMat& M, int n, int g) -> SzPair {
      const int G = M.K / kGroup;
      return {ld_u16(M.scale + (size_t)n * G + g), ld_u16(M.zero + (size_t)n * G + g)};
    };
    // A cursor over this CTA's (tile, k-block) sequence restricted to one team's k-blocks.
    struct Cursor {
      int j, tile, kb, mi;  // tile = this CTA's j-th tile, -1 past the last
      TileInfo ti;
    };
    auto cursor_start = [&](Cursor& c) {
      c.j = 0;
      c.tile = tile_of(0);
      c.kb = team;
      c.mi = 0;
      if (c.tile >= 0) c.ti = tile_info(P, c.tile, c.mi);
    };
    auto cursor_next = [&](Cursor& c) {
      c.kb += 2;
      if (c.kb >= c.ti.nkb) {
        c.kb = team;
        c.tile = tile_of(++c.j);
        if (c.tile >= 0) c.ti = tile_info(P, c.tile, c.mi);
      }
    };
    // Codes are not copied by TMA: a slow DRAM copy would hold up the activation copies
    // queued behind it. Each thread streams the 32 bytes of its row in each of the team's
    // k-blocks with two cp.async copies into its slot of a CRING-deep ring
    // ([slot][16-byte half][thread]), CRING - 1 of the team's k-blocks ahead, across tiles.
    Cursor fc;
    cursor_start(fc);
    int fseq = 0;
    auto fetch_next = [&]() {
      if (fc.tile >= 0) {
        const TcMat& Mf = P.m[fc.ti.mi];
        const int nf = min(fc.ti.n0 + r, Mf.N - 1);
        const uint8_t* src = reinterpret_cast<const uint8_t*>(Mf.codes) + (size_t)nf * (Mf.K / 2) + fc.kb * (BK / 2);
        const uint32_t dst = sbase + OFF_C + (uint32_t)(fseq % CRING) * CSLOT_BYTES + 16u * (uint32_t)t;
        cp_async16(dst, src);
        cp_async16(dst + CSLOT_BYTES / 2, src + 16);
        cursor_next(fc);
      }
      cp_async_commit();
      ++fseq;
    };
    for (int i = 0; i < CRING - 1; ++i) fetch_next();
    // scale / zero prefetch cursor, two of the team's k-blocks ahead
    Cursor sc;
    cursor_start(sc);
    SzPair sz0{0, 0}, sz1{0, 0};
    auto sz_fetch = [&]() -> SzPair {
      SzPair v{0, 0};
      if (sc.tile >= 0) {
        const TcMat& Ms = P.m[sc.ti.mi];
        v = load_sz(Ms, min(sc.ti.n0 + r, Ms.N - 1), sc.kb >> 1);
        cursor_next(sc);
      }
      return v;
    };
    sz0 = sz_fetch();
    sz1 = sz_fetch();
    int cseq = 0;
    for (int j = 0, tile; (tile = tile_of(j)) >= 0 && !timed_out; ++j) {
      const TileInfo ti = tile_info(P, tile, mi);
      for (int kb = team; kb < ti.nkb; kb += 2) {
        const int itk = it + kb;               // sequence number of this k-block
        const int a = itk % ASTAGES;
        const __half z = __ushort_as_half(sz0.z);
        const uint32_t c1024z = pack_h2(__hadd(z, __float2half(1024.f)));
        const uint32_t s2 = (uint32_t)sz0.s | ((uint32_t)sz0.s << 16);
        sz0 = sz1;
        sz1 = sz_fetch();
        fetch_next();
        cp_async_wait_ring();  // this k-block's codes (issued CRING - 1 fetches ago) have landed
        if (!tc::mbar_wait(bar_aempty + 8 * a, ((itk / ASTAGES) & 1) ^ 1)) { timed_out = true; break; }
        const uint8_t* cslot = smem + OFF_C + (cseq % CRING) * CSLOT_BYTES + 16 * t;
        const uint4 c0 = *reinterpret_cast<const uint4*>(cslot);
        const uint4 c1 = *reinterpret_cast<const uint4*>(cslot + CSLOT_BYTES / 2);
        ++cseq;
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint8_t* arow = smem + OFF_A + a * A_BYTES + r * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)  // logical 16-byte chunk (8 fp16) j of the 128-byte row
          *reinterpret_cast<uint4*>(arow + ((j ^ (r & 7)) << 4)) = dequant8(words[j], c1024z, s2);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar_aready + 8 * a);
      }
      it += ti.nkb;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp < 4) {
    // epilogue: this warp's 32 weight rows, all bn tokens of the tile. Each 32-token block
    // is transposed through shared memory into Y's [token][row] order and written by one
    // TMA tensor store; per-thread 2-byte global stores would flood the SM's memory path
    // and delay the TMA loads queued behind them.
    int lt = 0, nst = 0;
    const uint32_t ebuf = sbase + OFF_E + (uint32_t)(warp * 2 * EPI_BYTES);
    uint16_t* ebuf_g = reinterpret_cast<uint16_t*>(smem + OFF_E + warp * 2 * EPI_BYTES);
    for (int j = 0, tile; (tile = tile_of(j)) >= 0 && !timed_out; ++j, ++lt) {
      const TileInfo ti = tile_info(P, tile, mi);
      const TcMat& M = P.m[ti.mi];
      const int b = lt & 1;
      if (!tc::mbar_wait(bar_tfull + 8 * b, (lt >> 1) & 1)) { timed_out = true; break; }
      tc::tc_fence_after();
      const int row = ti.n0 + 32 * warp + lane;
      const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(b * kTcMaxBN);
      for (int c0 = 0; c0 < ti.bn; c0 += 32, ++nst) {
        uint32_t v[32];
        tc::tmem_ld_32x32b_x32(taddr + (uint32_t)c0, v);
        tc::tmem_wait_ld();
        if (M.y_tma) {
          // staging buffer nst & 1: the store issued from it two blocks ago has read it
          if (lane == 0) tc::bulk_wait_read<1>();
          __syncwarp();
          uint16_t* eb = ebuf_g + (nst & 1) * (EPI_BYTES / 2);
#pragma unroll
          for (int c = 0; c < 32; ++c) eb[c * 32 + lane] = __half_as_ushort(__float2half_rn(__uint_as_float(v[c])));
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tc::tma_store_2d(&M.tmap_y, ebuf + (uint32_t)((nst & 1) * EPI_BYTES), ti.n0 + 32 * warp, ti.m0 + c0);
            tc::bulk_commit();
          }
        } else if (row < M.N) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int m = ti.m0 + c0 + c;
            if (m < M.M)
              M.y[(size_t)m * M.ldy + row] = __half_as_ushort(__float2half_rn(__uint_as_float(v[c])));
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_tempty + 8 * b);
    }
    if (lane == 0) tc::bulk_wait_all();  // stores complete before the kernel exits
  }

  if (timed_out) {
    atomicOr(&g_device_errors, tc::kErrTimeout);
    misc[1] = 1;
  }
  __syncthreads();
  // On the error path each producer waits (bounded) for its own TMA loads that may still be
  // in flight before the shared memory they target is released.
  if (misc[1] && lane == 0) {
    if (warp == XPROD_WARP)
      for (int j = (it > XSTAGES ? it - XSTAGES : 0); j < it; ++j)
        tc::mbar_wait(bar_xfull + 8 * (j % XSTAGES), (j / XSTAGES) & 1);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
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
  // Y [M, N] fp16 as a tensor for the epilogue's TMA stores (box 32 rows x 32 tokens);
  // needs N * 2 bytes a multiple of 16 and a 16-byte aligned base, else plain stores
  t.y_tma = 0;
  if (N % 8 == 0 && ((uintptr_t)Y & 15) == 0) {
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)N * 2};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&t.tmap_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, Y, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
      t.y_tma = 1;
  }
  t.codes = codes;
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
  t.tile_cost = K / BK + 4;  // k-blocks of the main loop + an allowance for the epilogue
  return true;
}

int tc_bn_for(int M) {
  const int bn = ((M + 15) / 16) * 16;
  return bn < XBN ? bn : XBN;
}

// The dealing of p's tiles to `grid` CTAs: the leading matrices whose tiles have the largest
// cost against the cost of the next matrix's tiles (matrices come in non-increasing cost).
template <int CAP>
static TileDeal deal_for(const TcParamsT<CAP>& p, int grid) {
  const int c1 = p.m[0].tile_cost;
  int n1 = 0, c2 = 0;
  for (int i = 0; i < p.count; ++i) {
    if (p.m[i].tile_cost != c1) {
      c2 = p.m[i].tile_cost;
      break;
    }
    n1 += p.m[i].tile_end - p.m[i].tile_begin;
  }
  if (c2 > c1) return TileDeal{0, 0, 0};  // not in cost order: plain round robin
  return plan_deal(grid, n1, c1, c2);
}

template <int CAP>
static cudaError_t launch_cap(TcParamsT<CAP>& p, cudaStream_t stream) {
  static std::atomic<uint64_t> attr{0};
  const int smem = SMEM_USED + 1024;  // + alignment slack
  cudaError_t e = ensure_smem_limit(gemm_tc_int4_kernel<CAP>, smem, attr);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  if (sms == 0) return cudaErrorInvalidDevice;
  const int grid = p.total_tiles < sms ? p.total_tiles : sms;
  p.deal = deal_for(p, grid);
  gemm_tc_int4_kernel<CAP><<<grid, THREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(TcParams& p, cudaStream_t stream) {
  if (p.count == 1) {
    TcParamsT<1> p1;
    p1.m[0] = p.m[0];
    p1.total_cost = p.total_cost;
    p1.count = 1;
    p1.total_tiles = p.total_tiles;
    return launch_cap<1>(p1, stream);
  }
  return launch_cap<kTcMaxMats>(p, stream);
}

unsigned int* device_error_word() {
  static std::atomic<unsigned int*> addr[kMaxDevices];  // threads racing on a first call store the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned int* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_errors) != cudaSuccess) return nullptr;
    a = static_cast<unsigned int*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
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
