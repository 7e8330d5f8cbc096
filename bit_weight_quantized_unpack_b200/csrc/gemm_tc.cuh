// Parameters of the tensor-core dequantising GEMM (gemm_tc.cu) and its host entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tile_deal.cuh"

namespace wq {

constexpr int kTcMaxBN = 256;   // tokens per tile (MMA N), also the TMEM columns allocated
constexpr int kTcMaxMats = 80;  // matrices per launch: 80 x 384 B of tensor maps and fields fit
                                // the 32 KB kernel parameter block
constexpr int kTcMinM = 5;      // int4 products from this M up that the skinny-batch kernel
                                // does not take (M > 32, or its alignment needs unmet) run
                                // here; token rows past M in a 16-row tile are zero-filled by TMA

// One matrix: tiles [tile_begin, tile_end) of the launch, tiles_m token tiles per
// 128-row weight tile. Tensor maps first: CUtensorMap needs 64-byte alignment.
struct TcMat {
  CUtensorMap tmap_x;      // X [M, K] fp16, box 64 x bn, 128-byte swizzle
  CUtensorMap tmap_y;      // Y [M, N] fp16, box 32 x 32 (valid when y_tma)
  const void* codes;       // int4 codes uint32 [N, K/8] (streamed with cp.async, not TMA)
  const uint16_t* scale;
  const uint16_t* zero;
  uint16_t* y;             // fp16 [M, ldy]
  int64_t cost_begin;      // cost of all tiles of the launch before this matrix's first
  int N, K, M, ldy, bn, tiles_n, tiles_m, tile_begin, tile_end, tile_cost;
  int y_tma;               // the epilogue stores Y through tmap_y
};

// Passed by value as the kernel parameter; CAP is chosen per call (1 for a single matrix).
template <int CAP>
struct TcParamsT {
  TcMat m[CAP];
  int64_t total_cost;
  int count;
  int total_tiles;
  TileDeal deal;  // how the tiles are dealt to the CTAs (filled by launch_gemm_tc)
};
using TcParams = TcParamsT<kTcMaxMats>;
static_assert(sizeof(TcParams) <= 32764, "kernel parameter block");

bool tc_plan_mat(TcMat& t, const uint16_t* X, int M, const void* codes, const uint16_t* scale,
                 const uint16_t* zero, uint16_t* Y, int N, int K, int bn);
int tc_bn_for(int M);
// Fills p.deal for the grid it launches; p's matrices must be in non-increasing tile cost.
cudaError_t launch_gemm_tc(TcParams& p, cudaStream_t stream);
cudaError_t read_device_errors(unsigned int* flags, bool clear, cudaStream_t stream);
// Device address of the error word on the current device (looked up once per device).
unsigned int* device_error_word();

}  // namespace wq
