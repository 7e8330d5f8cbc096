// Parameters of the persistent matrix-vector kernels (shared by gemv.cu and wq_api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

constexpr int kGemvThreads = 256;
constexpr int kSetMax = 256;  // WQ_LINEAR_SET_MAX

// One matrix of a set. Rows [n0, n0 + 32/L) of warp item i (item_begin <= i < item_end)
// have n0 = (i - item_begin) * (32 >> lanes_log2).
struct SetMat {
  const void* codes;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint16_t* x;  // fp16 [M, ldx]
  uint16_t* y;        // fp16 [M, ldy]
  int N, K, M, ldx, ldy;
  int lanes_log2;     // L = 2^lanes_log2 lanes share one row
  int item_begin, item_end;
};

// Passed by value as a __grid_constant__ kernel parameter (about 15 KB): the set needs
// no device-side table and the library allocates nothing.
template <int CAP>
struct SetParamsT {
  int count;
  int total_items;
  SetMat m[CAP];
};
using SetParams = SetParamsT<kSetMax>;

int gemv_lanes_log2(int fmt, int64_t K);
cudaError_t launch_gemv_set(const SetParams& p, int fmt, int max_m, cudaStream_t stream);
// int3 products of a set (one warp per output row, items = rows): gemv_int3.cu
cudaError_t launch_gemv_int3(const SetParams& p, cudaStream_t stream);
cudaError_t launch_quantize(const float* W, int64_t N, int64_t K, int fmt, void* codes,
                            uint16_t* scale, uint16_t* zero, cudaStream_t stream);

}  // namespace wq
