// Internal entry points shared by the C ABI's translation units (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace wq {

// Every check of wq_gemv_argmax except those on the work space, then the launch plan; on
// WQ_OK, *workspace_needed is the work-space size the launch needs and the plan is kept
// (per host thread) for argmax_launch. Enqueues nothing.
int argmax_prepare(const uint16_t* x, const void* codes, const uint16_t* scale, const uint16_t* zero, int fmt,
                   int64_t N, int64_t K, uint16_t* y, int32_t* argmax, size_t* workspace_needed);
// Launches the plan of this thread's last successful argmax_prepare with `workspace`.
int argmax_launch(void* workspace, cudaStream_t stream);

}  // namespace wq
