// Head rescoring: the quantised lm_head's logits pick candidates, an fp16 copy of the head
// recomputes them, and the token is the best recomputed candidate.
//
// Whetstone README, feature list (--head-rescore): an fp16 copy of the output projection is
// kept and only the logits that decide the token are recomputed from it, so the token comes
// close to an fp16 head's while the bytes read per token stay those of the quantised head.
// The candidates are the k largest quantised logits (equal values: the lower row); the
// token is the candidate with the largest recomputed logit (equal values: the lower row).
//
// Pass 1 (one CTA per 2048 logits): each logit becomes a 64-bit key that orders by value,
// then by lower row; k rounds of a block-wide maximum (shuffles, then one shared-memory step
// across warps), each removing the winner from its owner's registers, leave the chunk's k
// largest keys in the caller's work space. Pass 2 (one CTA): the same rounds over all
// chunks' candidates; each of the k winners is recomputed by one warp (x . w16[row], fp32
// accumulation over exact fp16 x fp16 products, a fixed-order shuffle reduction); thread 0
// picks the token.
#include <climits>

#include "common.cuh"
#include "gemv_stream.cuh"
#include "wq.h"

namespace wq {
namespace {

constexpr int kChunk = 2048;          // logits per CTA of pass 1
constexpr int kTopThreads = 256;
constexpr int kMergeThreads = 1024;
constexpr int kMaxTopk = WQ_RESCORE_MAX_TOPK;
constexpr int kMaxChunks = 256;       // pass 2 sorts up to kMaxChunks * kMaxTopk keys
constexpr int64_t kMaxRows = (int64_t)kChunk * kMaxChunks;

// Larger value -> larger key; equal values -> the lower row has the larger key. -0 and +0
// are one value. (binary16 bits: positive values order as unsigned; negative values in
// reverse, below all positive ones.)
__device__ __forceinline__ uint64_t key_of(uint16_t hbits, uint32_t row) {
  uint32_t b = hbits;
  if ((b & 0x7FFFu) == 0) b = 0;
  const uint32_t o = (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
  return ((uint64_t)o << 32) | (uint64_t)(0xFFFFFFFFu - row);
}

__device__ __forceinline__ uint32_t row_of(uint64_t key) { return 0xFFFFFFFFu - (uint32_t)key; }

// k rounds of "largest key of the block, then remove it": out[r] = the r-th largest of all
// threads' keys (PER per thread, in registers; keys are unique, 0 = none). All threads call
// it; out is written by thread 0. red: shared scratch of one key per warp plus one.
template <int PER>
__device__ void block_topk(uint64_t (&key)[PER], int k, uint64_t* out, uint64_t* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  uint64_t mine = 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) mine = key[q] > mine ? key[q] : mine;
  for (int r = 0; r < k; ++r) {
    uint64_t m = mine;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t v = __shfl_xor_sync(0xFFFFFFFFu, m, o);
      m = v > m ? v : m;
    }
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
      uint64_t b = lane < nw ? red[lane] : 0ull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint64_t v = __shfl_xor_sync(0xFFFFFFFFu, b, o);
        b = v > b ? v : b;
      }
      if (lane == 0) {
        red[32] = b;
        out[r] = b;
      }
    }
    __syncthreads();
    const uint64_t best = red[32];
    if (best != 0ull && mine == best) {  // this thread holds it: drop it, find the next
      uint64_t nm = 0;
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        if (key[q] == best) key[q] = 0ull;
        nm = key[q] > nm ? key[q] : nm;
      }
      mine = nm;
    }
  }
}

constexpr int kPerChunk = kChunk / kTopThreads;                       // 8 keys per thread
constexpr int kPerMerge = kMaxChunks * kMaxTopk / kMergeThreads;     // 16 keys per thread

__global__ void __launch_bounds__(kTopThreads) topk_chunk_kernel(const uint16_t* __restrict__ y, int N, int topk,
                                                                  uint64_t* __restrict__ ws) {
  __shared__ uint64_t red[33];
  __shared__ uint64_t out[kMaxTopk];
  uint64_t key[kPerChunk];
  const int base = blockIdx.x * kChunk;
#pragma unroll
  for (int q = 0; q < kPerChunk; ++q) {
    const int r = base + q * kTopThreads + threadIdx.x;
    key[q] = r < N ? key_of(y[r], (uint32_t)r) : 0ull;  // key 0: below every real logit
  }
  block_topk(key, topk, out, red);
  __syncthreads();
  for (int i = threadIdx.x; i < topk; i += kTopThreads) ws[(size_t)blockIdx.x * topk + i] = out[i];
}

__global__ void __launch_bounds__(kMergeThreads) merge_rescore_kernel(const uint64_t* __restrict__ ws, int nkeys,
                                                                       int N, int topk,
                                                                       const uint16_t* __restrict__ x,
                                                                       const uint16_t* __restrict__ w16, int K,
                                                                       int32_t* __restrict__ cand,
                                                                       float* __restrict__ cand_logits,
                                                                       int32_t* __restrict__ token) {
  __shared__ uint64_t red[33];
  __shared__ uint64_t top[kMaxTopk];
  __shared__ float lg[kMaxTopk];
  __shared__ int rw[kMaxTopk];
  uint64_t key[kPerMerge];
#pragma unroll
  for (int q = 0; q < kPerMerge; ++q) {
    const int i = q * kMergeThreads + threadIdx.x;
    key[q] = i < nkeys ? ws[i] : 0ull;
  }
  const int k = topk < N ? topk : N;  // fewer rows than candidates asked for
  block_topk(key, k, top, red);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int c = warp; c < k; c += kMergeThreads / 32) {
    const uint32_t row = row_of(top[c]);
    const uint4* xr = reinterpret_cast<const uint4*>(x);
    const uint4* wr = reinterpret_cast<const uint4*>(w16 + (size_t)row * K);
    float acc = 0.f;
    for (int j = lane; j < K / 8; j += 32) {
      const uint4 xv = xr[j], wv = wr[j];
      const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, wsv[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc = fma_f16f16_f32(lo16(xs[q]), lo16(wsv[q]), acc);
        acc = fma_f16f16_f32(hi16(xs[q]), hi16(wsv[q]), acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) {
      lg[c] = acc;
      rw[c] = (int)row;
      cand[c] = (int32_t)row;
      cand_logits[c] = acc;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int best = 0;
    for (int c = 1; c < k; ++c)
      if (lg[c] > lg[best] || (lg[c] == lg[best] && rw[c] < rw[best])) best = c;
    token[0] = rw[best];
  }
}

int chunks_for(int64_t N) { return (int)((N + kChunk - 1) / kChunk); }

}  // namespace
}  // namespace wq

extern "C" {

size_t wq_rescore_workspace_bytes(int64_t N, int topk) {
  if (N < 1 || N > wq::kMaxRows || topk < 1 || topk > wq::kMaxTopk) return 0;
  return (size_t)wq::chunks_for(N) * (size_t)topk * sizeof(uint64_t);
}

int wq_gemv_rescore(const uint16_t* x, const void* codes, const uint16_t* scale, const uint16_t* zero, int fmt,
                    const uint16_t* w16, int64_t N, int64_t K, int topk, uint16_t* y, int32_t* cand,
                    float* cand_logits, int32_t* token, void* workspace, size_t workspace_bytes, void* stream) {
  if (!w16 || !cand || !cand_logits || !token || !workspace || !x || !y) return WQ_ERR_ARG;
  if (topk < 1 || topk > wq::kMaxTopk) return WQ_ERR_ARG;
  if (N < 1 || N > wq::kMaxRows || K < 128 || K % 128 != 0 || K > INT_MAX) return WQ_ERR_SHAPE;
  const size_t need = wq_rescore_workspace_bytes(N, topk);
  if (workspace_bytes < need) return WQ_ERR_ARG;
  if (((uintptr_t)w16 & 15) || ((uintptr_t)x & 15) || ((uintptr_t)workspace & 7) || ((uintptr_t)cand & 3) ||
      ((uintptr_t)cand_logits & 3) || ((uintptr_t)token & 3))
    return WQ_ERR_ALIGN;
  // the quantised head's logits (all of wq_gemv's checks run before its launch)
  int st = wq_gemv(x, codes, scale, zero, fmt, N, K, y, stream);
  if (st != WQ_OK) return st;
  const cudaStream_t s = (cudaStream_t)stream;
  const int nchunks = wq::chunks_for(N);
  wq::topk_chunk_kernel<<<nchunks, wq::kTopThreads, 0, s>>>(y, (int)N, topk, static_cast<uint64_t*>(workspace));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return wq::note_cuda_error(e);
  const int nkeys = nchunks * topk;
  wq::merge_rescore_kernel<<<1, wq::kMergeThreads, 0, s>>>(static_cast<const uint64_t*>(workspace), nkeys, (int)N,
                                                            topk, x, w16, (int)K, cand, cand_logits, token);
  e = cudaGetLastError();
  return e == cudaSuccess ? WQ_OK : wq::note_cuda_error(e);
}

}  // extern "C"
