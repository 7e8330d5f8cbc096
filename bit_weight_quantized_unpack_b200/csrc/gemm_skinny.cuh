// Parameters of the skinny-batch int4 GEMM (gemm_skinny.cu): Y[M, N] = X[M, K] * W_hat^T for
// a few tokens (M <= kSkMaxM), weights read once and multiplied from registers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

constexpr int kSkWarps = 8;           // warps per CTA, one 16-row weight slab each
constexpr int kSkUnitRows = 16 * kSkWarps;  // weight rows per unit of work (128)
#ifndef WQ_SK_MIN_M
#define WQ_SK_MIN_M 5
#endif
constexpr int kSkMinM = WQ_SK_MIN_M;  // wq_gemm / wq_linear_set use this kernel for int4 from
                                      // this M (below it the streaming kernel is faster) ...
constexpr int kSkMaxM = 32;           // ... up to this M (tokens per product)
constexpr int kSkMaxMats = 256;
constexpr int kSkCtasPerSm = 2;       // register budget of the launch bounds
constexpr int kSkSmemPerCta = 112 * 1024;  // two activation buffers

// One matrix; its units are [unit_begin, unit_begin + ceil(N / 128)). The activations of a
// unit are staged in chunks of kc groups (nch chunks, the last one possibly shorter).
struct SkMat {
  const uint8_t* codes;    // int4 codes, bytes [N, K/2]
  const uint16_t* scale;   // fp16 [N, K/128]
  const uint16_t* zero;    // fp16 [N, K/128]
  const uint16_t* x;       // fp16 [M, K], 16-byte aligned
  uint16_t* y;             // fp16 [M, N]
  int N, K;
  int unit_begin;
  int nch, kc;
};

template <int CAP>
struct SkParamsT {
  int count;
  int M;
  int total_units;
  int buf_bytes;           // bytes of one activation buffer
  SkMat m[CAP];
};
using SkParams = SkParamsT<kSkMaxMats>;

struct SkDesc {
  const void* codes;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint16_t* x;
  uint16_t* y;
  int64_t N, K;
};

// Fills p for `count` int4 matrices multiplied by M tokens (1 <= M <= kSkMaxM), ordered by
// K, largest first, and returns the dynamic shared memory of a CTA, or 0 if the kernel
// cannot serve the set (alignment, or more than kSkMaxMats matrices).
int skinny_plan(SkParams& p, int count, const SkDesc* d, int M);
cudaError_t launch_gemm_skinny(const SkParams& p, int smem, cudaStream_t stream);

}  // namespace wq
