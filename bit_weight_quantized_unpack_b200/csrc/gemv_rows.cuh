// Parameters of the row-per-lane matrix-vector kernel (gemv_rows.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

constexpr int kRowsThreads = 256;
constexpr int kRowsMaxMats = 256;
constexpr int kRowsStages = 3;           // per-thread ring of code groups (2 in flight)
constexpr int kRowsMaxSmem = 200 * 1024;  // ring + staged activations (K * 4 bytes)

// One matrix: its rows start at byte cost cost_begin of the whole set, row_cost bytes of
// codes + metadata each.
struct RowMat {
  const void* codes;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint16_t* x;
  uint16_t* y;
  int64_t cost_begin;
  int64_t row_cost;
  int N, K;
};

// Passed by value as the kernel parameter; CAP is chosen per call (1 for a single matrix)
// so that a launch copies no more parameter bytes than it uses.
template <int CAP>
struct RowParamsT {
  int64_t total_cost;
  int count;
  RowMat m[CAP];
};
using RowParams = RowParamsT<kRowsMaxMats>;

struct RowMatDesc {
  const void* codes;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint16_t* x;
  uint16_t* y;
  int64_t N, K;
};

// Fills p; false if the set needs more shared memory than this kernel stages.
bool rows_plan(RowParams& p, int bits, int count, const RowMatDesc* d, int* max_k);
cudaError_t launch_gemv_rows(const RowParams& p, int bits, int max_k, cudaStream_t stream);

}  // namespace wq
