// wq_gemv_argmax_static: the fused product + greedy pick with the library's own scratch.
//
// wq_gemv_argmax needs a small device work space (a ticket counter and one partial result
// per CTA). Some callers cannot hand one over: engines that own all device memory through
// their own pool and forbid libraries to allocate, or decode loops where an allocation,
// which may synchronise the device, is not allowed. This entry point uses a fixed array
// that lives in libwq itself instead; it allocates nothing.
#include "gemv_stream.cuh"
#include "wq.h"

namespace {

// The scratch: a 16-byte header (ticket counter) then one (value, row) pair per CTA.
static __device__ __align__(256) unsigned char g_argmax_scratch[WQ_ARGMAX_STATIC_SCRATCH_BYTES];

// Device address of g_argmax_scratch on the current device, looked up once per device (the
// host-side symbol is not a device address). nullptr if the lookup fails.
void* scratch_address() {
  static void* addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_argmax_scratch);
    if (e != cudaSuccess) {
      wq::note_cuda_error(e);
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" int wq_gemv_argmax_static(const uint16_t* x, const void* codes, const uint16_t* scale,
                                     const uint16_t* zero, int fmt, int64_t N, int64_t K, uint16_t* y,
                                     int32_t* argmax, void* stream) {
  // every check of wq_gemv_argmax happens here first, so that a rejected call enqueues
  // nothing (not even the clearing of the scratch header)
  if (fmt != WQ_INT4 && fmt != WQ_INT2) return WQ_ERR_ARG;
  if (N < 1 || N > INT32_MAX || K < 128 || K > 32768 || K % 128 != 0) return WQ_ERR_SHAPE;
  if (!x || !codes || !scale || !zero || !argmax) return WQ_ERR_ARG;
  if ((((uintptr_t)x | (uintptr_t)codes | (uintptr_t)scale | (uintptr_t)zero) & 15) != 0 ||
      ((uintptr_t)argmax & 3) != 0 || (y && ((uintptr_t)y & 1) != 0))
    return WQ_ERR_ALIGN;
  const size_t need = wq_argmax_workspace_bytes();
  if (need == 0) return WQ_ERR_UNSUPPORTED;
  if (need > WQ_ARGMAX_STATIC_SCRATCH_BYTES) return WQ_ERR_SCRATCH;
  void* ws = scratch_address();
  if (!ws) return WQ_ERR_CUDA;
  // the array keeps the previous call's contents: start the ticket counter from zero
  const cudaError_t e = cudaMemsetAsync(ws, 0, 16, (cudaStream_t)stream);
  if (e != cudaSuccess) return wq::note_cuda_error(e);
  return wq_gemv_argmax(x, codes, scale, zero, fmt, N, K, y, argmax, ws, WQ_ARGMAX_STATIC_SCRATCH_BYTES, stream);
}
