// Parameters of the skinny-batch int4 GEMM (gemm_skinny.cu): Y[M, N] = X[M, K] * W_hat^T for
// a few tokens (M <= kSkMaxM), weights read once and multiplied from registers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

constexpr int kSkWarps = 16;          // warps per CTA (one CTA per SM), one 16-row slab each
constexpr int kSkThreads = 32 * kSkWarps;
#ifndef WQ_SK_MIN_M
#define WQ_SK_MIN_M 2
#endif
constexpr int kSkMinM = WQ_SK_MIN_M;  // wq_gemm / wq_linear_set use this kernel for int4 from
                                      // this M (at M = 1 the streaming GEMV is faster) ...
constexpr int kSkMaxM = 32;           // ... up to this M (tokens per product)
constexpr int kSkMaxMats = 256;
// code groups in flight per thread (cp.async ring of 16 KB slots): six for up to 16 tokens;
// four for more, whose activation chunks need the room
__host__ __device__ constexpr int sk_ring(int tb) { return tb >= 4 ? 4 : 6; }
__host__ __device__ constexpr int sk_ring_bytes(int tb) { return sk_ring(tb) * 2 * kSkThreads * 16; }
constexpr int kSkSpanOne = 8;         // slabs per warp and window when the activations of a
                                      // matrix fit one chunk
constexpr int kSkSmemMax = 232448;    // dynamic shared memory of one CTA (227 KB)

// One matrix: slabs [slab_begin, slab_end) of the launch (16 weight rows each, the last one
// possibly short), at cost positions cost_begin + j * G (cost = 128-weight groups). Its
// slabs are taken in windows of up to `span` slabs (warp w: slabs w, w + 16, ...), and the
// activations of a window are staged in chunks of kc groups (nch chunks, the last one
// possibly shorter); with more than one chunk a window holds one slab per warp, whose sums
// stay in registers across the chunks.
struct SkMat {
  const uint8_t* codes;    // int4 codes, bytes [N, K/2]
  const uint16_t* scale;   // fp16 [N, K/128]
  const uint16_t* zero;    // fp16 [N, K/128]
  const uint16_t* x;       // fp16 [M, K], 16-byte aligned
  uint16_t* y;             // fp16 [M, N]
  int64_t cost_begin;
  int N, K, G;
  int slab_begin, slab_end;
  int nch, kc, span;
};

template <int CAP>
struct SkParamsT {
  int count;
  int M;
  int total_slabs;
  int buf_bytes;           // bytes of one activation buffer
  int64_t total_cost;
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

// Fills p for `count` int4 matrices multiplied by M tokens (1 <= M <= kSkMaxM) and returns
// the dynamic shared memory of a CTA, or 0 if the kernel cannot serve the set (alignment, or
// more than kSkMaxMats matrices).
int skinny_plan(SkParams& p, int count, const SkDesc* d, int M);
cudaError_t launch_gemm_skinny(const SkParams& p, int smem, cudaStream_t stream);

}  // namespace wq
