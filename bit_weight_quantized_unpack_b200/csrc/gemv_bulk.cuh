// Parameters of the bulk-copy-staged matrix-vector kernel (gemv_bulk.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

constexpr int kBulkStages = 4;
constexpr int kBulkStageBytes = 48 * 1024;  // codes of one row block (or K segment)
constexpr int kBulkMetaBytes = 8 * 1024;    // scales + zeros of one row block
constexpr int kBulkConsumerWarps = 12;
constexpr int kBulkMaxMats = 256;

// One matrix: row blocks [block_begin, block_end) of the launch, rows_per_block rows each
// (the last one may be short), every block block_bytes of codes, the first of them at
// byte offset cost_begin of the whole set.
struct BulkMat {
  const void* codes;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint16_t* x;
  uint16_t* y;
  int64_t cost_begin;
  int N, K;
  int lanes_log2, rows_per_block, kseg, nseg;
  int block_begin, block_end, block_bytes;
  int meta_bulk;  // scales / zeros are 16-byte aligned and a block's fit one meta slot
};

struct BulkParams {
  unsigned int* errors;  // the library's device error word (see device_error_word)
  int64_t total_cost;
  int count;
  int total_blocks;
  BulkMat m[kBulkMaxMats];
};

bool bulk_plan_mat(BulkMat& m, int bits, const void* codes, const uint16_t* scale,
                   const uint16_t* zero, const uint16_t* x, uint16_t* y, int64_t N, int64_t K);
cudaError_t launch_gemv_bulk(const BulkParams& p, int bits, cudaStream_t stream);

}  // namespace wq
