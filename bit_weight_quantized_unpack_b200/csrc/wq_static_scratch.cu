// wq_gemv_argmax_static: the fused product + greedy pick with the library's own scratch.
//
// wq_gemv_argmax needs a small device work space (a ticket counter and one partial result
// per CTA). Some callers cannot hand one over: engines that own all device memory through
// their own pool and forbid libraries to allocate, or decode loops where an allocation,
// which may synchronise the device, is not allowed. This entry point uses a fixed array
// that lives in libwq itself instead; it allocates nothing.
#include <atomic>

#include "api_internal.cuh"
#include "gemv_stream.cuh"
#include "host_util.cuh"
#include "wq.h"

namespace {

// The scratch: a 16-byte header (ticket counter) then one (value, row) pair per CTA.
static __device__ __align__(256) unsigned char g_argmax_scratch[WQ_ARGMAX_STATIC_SCRATCH_BYTES];

// Device address of g_argmax_scratch on the current device, looked up once per device (the
// host-side symbol is not a device address); threads racing on a first call store the same
// value. The cache assumes the module stays loaded: after cudaDeviceReset the address is
// not looked up again. nullptr if the lookup fails.
void* scratch_address() {
  static std::atomic<void*> addr[wq::kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= wq::kMaxDevices) return nullptr;
  void* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    const cudaError_t e = cudaGetSymbolAddress(&a, g_argmax_scratch);
    if (e != cudaSuccess) {
      wq::note_cuda_error(e);
      return nullptr;
    }
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}

}  // namespace

extern "C" int wq_gemv_argmax_static(const uint16_t* x, const void* codes, const uint16_t* scale,
                                     const uint16_t* zero, int fmt, int64_t N, int64_t K, uint16_t* y,
                                     int32_t* argmax, void* stream) {
  // every check and the launch plan come first, so that a rejected call enqueues nothing
  // (not even the clearing of the scratch header)
  size_t need = 0;
  const int st = wq::argmax_prepare(x, codes, scale, zero, fmt, N, K, y, argmax, &need);
  if (st != WQ_OK) return st;
  if (need > WQ_ARGMAX_STATIC_SCRATCH_BYTES) return WQ_ERR_SCRATCH;
  void* ws = scratch_address();
  if (!ws) return WQ_ERR_CUDA;
  // the array keeps the previous call's contents: start the ticket counter from zero
  const cudaError_t e = cudaMemsetAsync(ws, 0, 16, (cudaStream_t)stream);
  if (e != cudaSuccess) return wq::note_cuda_error(e);
  return wq::argmax_launch(ws, (cudaStream_t)stream);
}
