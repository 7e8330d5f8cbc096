// Parameters of the streaming matrix-vector kernel (gemv_stream.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

constexpr int kStreamWarps = 4;              // warps per CTA (up to four CTAs per SM)
constexpr int kStreamMaxCtasPerSm = 4;       // register budget of the launch bounds
constexpr int kStreamMaxMats = 256;
constexpr int kStreamMaxRows = 4;            // rows of X per product (M = 1 .. 4)
constexpr int kStreamSmPool = 233472;        // shared memory of one SM (228 KB)
constexpr int kStreamMaxSmem = 232448 - 1024; // dynamic, per CTA (227 KB less room for static)
#ifndef WQ_STREAM_SLOT_CODES
#define WQ_STREAM_SLOT_CODES 4096
#endif
#ifndef WQ_STREAM_SLOTS
#define WQ_STREAM_SLOTS 2
#endif
constexpr int kStreamSlotCodes = WQ_STREAM_SLOT_CODES;  // bytes of codes per ring slot (one bulk copy)
constexpr int kStreamSlots = WQ_STREAM_SLOTS;           // ring slots per warp

// One matrix. Rows are dealt to warps in units of RA rows, RA chosen so that every unit's
// scales and zeros start on a 16-byte boundary; cost counts bytes of codes + scales + zeros.
struct StreamMat {
  const void* codes;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint16_t* x;
  uint16_t* y;
  int64_t cost_begin;  // cost of the set's matrices before this one
  int64_t cost_end;    // cost_begin + cost of this matrix
  int64_t unit_cost;   // cost of one full unit
  double inv_unit_cost;  // 1 / unit_cost
  int N, K;
  int RA;              // rows per unit
  int nunit;           // ceil(N / RA)
};

template <int CAP>
struct StreamParamsT {
  unsigned int* errors;  // device error word (bounded waits that gave up)
  int64_t total_cost;
  int count;
  int slots;             // ring slots per warp
  int xbufs;             // staged activation buffers per CTA (1 or 2)
  int ctas_per_sm;       // CTAs that fit on one SM with this set's shared memory
  int xbuf_bytes;        // bytes of one activation buffer
  uint32_t max_polls;    // bound on the polls of one mbarrier wait
  int skip_first_copy;   // failure-detection test: CTA 0's warp 0 never fills its first ring slot
  // fused argmax over the rows of a single matrix (null when not wanted): work space of
  // 16 + 8 * gridDim.x bytes whose first word is a CTA ticket counter (zero between calls),
  // followed by one (fp32 value, int32 row) partial per CTA; the result row goes to am_out
  unsigned int* am_ws;
  int* am_out;
  StreamMat m[CAP];
};
using StreamParams = StreamParamsT<kStreamMaxMats>;

struct StreamDesc {
  const void* codes;
  const uint16_t* scale;
  const uint16_t* zero;
  const uint16_t* x;
  uint16_t* y;
  int64_t N, K;
};

// Format tags of the streaming kernel: bits 4, 3 or 2 (g128 integer codes), 1 (ternary), 5
// (hierarchical int4: codes as int4, `scale` the fp16 row pairs [N, 2], `zero` the index bytes
// [N, K/32]).
constexpr int kStreamHier = 5;

// Fills p for a set of `count` matrices of one format (a tag above), each multiplied by mt
// rows of X (X [mt, K] and Y [mt, N] row-major), and returns the bytes of dynamic shared
// memory a CTA needs, or 0 if this kernel cannot serve the set (pointers not 16-byte
// aligned, or activations too long to stage).
int stream_plan(StreamParams& p, int bits, int count, const StreamDesc* d, int mt);
cudaError_t launch_gemv_stream(const StreamParams& p, int bits, int mt, int smem, cudaStream_t stream);
// One matrix (p.count == 1, mt == 1) with the fused argmax of its fp16 outputs (ties to the
// lowest row); p.am_ws / p.am_out must be set. Grid = p.ctas_per_sm * SMs CTAs.
cudaError_t launch_gemv_stream_argmax(const StreamParams& p, int bits, int smem, cudaStream_t stream);
// CTAs the streaming kernel launches for a plan (the argmax work space holds one partial each).
int stream_grid(const StreamParams& p);
// Records e as the library's last CUDA error (wq_last_cuda_error); returns the wq_status.
int note_cuda_error(cudaError_t e);

}  // namespace wq
