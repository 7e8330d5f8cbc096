// C ABI of libwq (declared in include/wq.h): argument checks, launch planning, launches.
// Every check happens before the first launch; no device memory is ever allocated here.
#include <limits.h>
#include <string.h>

#include "gemm_skinny.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "api_internal.cuh"
#include "gemv_rows.cuh"
#include "gemv_stream.cuh"
#include "host_util.cuh"
#include "wq.h"

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return WQ_OK;
  g_last_cuda_error = (int)e;
  return WQ_ERR_CUDA;
}

}  // namespace

namespace wq {
int note_cuda_error(cudaError_t e) { return cuda_status(e); }
}  // namespace wq

namespace {

// The kernels are built for sm_100a only: refuse any other device up front instead of
// failing inside a launch. Cached per device ordinal.
int check_device() {
  static std::atomic<int> cached[wq::kMaxDevices];  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= wq::kMaxDevices) return WQ_ERR_UNSUPPORTED;
  int c = cached[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_status(e);
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_status(e);
    c = (major == 10 && minor == 0) ? 1 : 2;
    cached[dev].store(c, std::memory_order_relaxed);
  }
  return c == 1 ? WQ_OK : WQ_ERR_UNSUPPORTED;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

constexpr int64_t kMaxK = (int64_t)1 << 20;

int check_shape(int fmt, int64_t N, int64_t K) {
  if (fmt < WQ_INT4 || fmt > WQ_INT4H) return WQ_ERR_ARG;
  if (N < 1 || N > INT_MAX || K < 128 || K > kMaxK || K % 128 != 0) return WQ_ERR_SHAPE;
  return WQ_OK;
}

int check_weights(int fmt, const void* codes, const uint16_t* scale, const uint16_t* zero) {
  if (!codes || !scale) return WQ_ERR_ARG;
  if ((fmt == WQ_TERNARY) != (zero == nullptr)) return WQ_ERR_ARG;
  if (fmt == WQ_INT4H)  // row pairs read as 4-byte words, index bytes bulk-copied
    return aligned(codes, 16) && aligned(scale, 4) && aligned(zero, 16) ? WQ_OK : WQ_ERR_ALIGN;
  if (!aligned(codes, 16) || !aligned(scale, 2) || (zero && !aligned(zero, 2))) return WQ_ERR_ALIGN;
  return WQ_OK;
}

// Hierarchical int4 is served by the streaming kernel only: M rows of X of K values each
// staged in shared memory, M * K <= kHierMaxMK (with M <= 4).
constexpr int64_t kHierMaxMK = 92160;

// Fill one SetMat; returns its item count (rows per item = 32 >> lanes_log2).
int64_t plan_mat(wq::SetMat& m, int fmt, const void* codes, const uint16_t* scale,
                 const uint16_t* zero, const uint16_t* x, uint16_t* y, int64_t N, int64_t K,
                 int64_t M) {
  m.codes = codes;
  m.scale = scale;
  m.zero = zero;
  m.x = x;
  m.y = y;
  m.N = (int)N;
  m.K = (int)K;
  m.M = (int)M;
  m.ldx = (int)K;
  m.ldy = (int)N;
  m.lanes_log2 = wq::gemv_lanes_log2(fmt, K);
  const int64_t rows = 32 >> m.lanes_log2;
  return (N + rows - 1) / rows;
}

// Streaming kernel for a set (int4 / int2 / ternary / int4h) with M = 1 .. 4 rows of X: needs
// 16-byte aligned codes, metadata and activations, and activations short enough to stage in
// shared memory.
// Failure-detection test hook (wq_debug_arm_timeout): poll bound for the next streaming launch
// on this thread, with one of its ring slots never filled; 0 = disarmed.
thread_local uint32_t g_arm_polls = 0;

int try_stream(int fmt, int count, const wq_linear_desc* d, int64_t M, cudaStream_t stream, bool* done) {
  *done = false;
  if (count > wq::kStreamMaxMats || M > wq::kStreamMaxRows) return WQ_OK;
  static thread_local wq::StreamParams sp;
  static thread_local wq::StreamDesc sd[wq::kStreamMaxMats];
  for (int i = 0; i < count; ++i) sd[i] = {d[i].codes, d[i].scale, d[i].zero, d[i].x, d[i].y, d[i].N, d[i].K};
  // format tag: 4 / 3 / 2 bits, 1 ternary, kStreamHier
  const int bits = fmt == WQ_INT4 ? 4 : fmt == WQ_INT3 ? 3 : fmt == WQ_INT2 ? 2 : fmt == WQ_INT4H ? wq::kStreamHier : 1;
  const int smem = wq::stream_plan(sp, bits, count, sd, (int)M);
  if (smem == 0) return WQ_OK;
  *done = true;
  if (g_arm_polls) {
    sp.max_polls = g_arm_polls;
    sp.skip_first_copy = 1;
    g_arm_polls = 0;
  }
  return cuda_status(wq::launch_gemv_stream(sp, bits, (int)M, smem, stream));
}

// int3 set: one warp per output row (any M).
int launch_int3(const wq_linear_desc* d, int count, cudaStream_t stream) {
  static thread_local wq::SetParams p;
  int64_t total = 0;
  for (int i = 0; i < count; ++i) {
    wq::SetMat& m = p.m[i];
    memset(&m, 0, sizeof(m));
    m.codes = d[i].codes;
    m.scale = d[i].scale;
    m.zero = d[i].zero;
    m.x = d[i].x;
    m.y = d[i].y;
    m.N = (int)d[i].N;
    m.K = (int)d[i].K;
    m.M = (int)d[i].M;
    m.ldx = (int)d[i].K;
    m.ldy = (int)d[i].N;
    m.item_begin = (int)total;
    total += d[i].N;
    if (total > INT_MAX) return WQ_ERR_SHAPE;
    m.item_end = (int)total;
  }
  p.count = count;
  p.total_items = (int)total;
  return cuda_status(wq::launch_gemv_int3(p, stream));
}

// Skinny-batch GEMM for an int4 set with kSkMinM <= M <= kSkMaxM: needs 16-byte aligned
// codes and activations.
int try_skinny(int fmt, int count, const wq_linear_desc* d, int64_t M, cudaStream_t stream, bool* done) {
  *done = false;
  if (fmt != WQ_INT4 || count > wq::kSkMaxMats || M < wq::kSkMinM || M > wq::kSkMaxM) return WQ_OK;
  static thread_local wq::SkParams kp;
  static thread_local wq::SkDesc kd[wq::kSkMaxMats];
  for (int i = 0; i < count; ++i) kd[i] = {d[i].codes, d[i].scale, d[i].zero, d[i].x, d[i].y, d[i].N, d[i].K};
  const int smem = wq::skinny_plan(kp, count, kd, (int)M);
  if (smem == 0) return WQ_OK;
  *done = true;
  return cuda_status(wq::launch_gemm_skinny(kp, smem, stream));
}

// Row-per-lane kernel for a batch-1 set (int4 / int2): needs 32-byte aligned codes
// (its loads are whole 32-byte sectors) and K small enough to stage x in shared memory.
int try_rows(int fmt, int count, const wq_linear_desc* d, cudaStream_t stream, bool* done) {
  *done = false;
  if (fmt == WQ_TERNARY || count > wq::kRowsMaxMats) return WQ_OK;
  static thread_local wq::RowParams rp;
  static thread_local wq::RowMatDesc rd[wq::kRowsMaxMats];
  for (int i = 0; i < count; ++i) {
    if (((uintptr_t)d[i].codes & 31) != 0) return WQ_OK;
    rd[i] = {d[i].codes, d[i].scale, d[i].zero, d[i].x, d[i].y, d[i].N, d[i].K};
  }
  int max_k = 0;
  if (!wq::rows_plan(rp, fmt == WQ_INT4 ? 4 : 2, count, rd, &max_k)) return WQ_OK;
  *done = true;
  return cuda_status(wq::launch_gemv_rows(rp, fmt == WQ_INT4 ? 4 : 2, max_k, stream));
}

}  // namespace

namespace wq {

namespace {
// The plan of the last argmax_prepare on this thread (consumed by argmax_launch).
thread_local StreamParams g_am_stream;
thread_local int g_am_bits = 0;  // 0: no plan; else the streaming kernel's format tag
thread_local int g_am_smem = 0;
}  // namespace

int argmax_prepare(const uint16_t* x, const void* codes, const uint16_t* scale, const uint16_t* zero, int fmt,
                   int64_t N, int64_t K, uint16_t* y, int32_t* argmax, size_t* workspace_needed) {
  g_am_bits = 0;
  int st = check_shape(fmt, N, K);
  if (st != WQ_OK) return st;
  if (fmt == WQ_TERNARY || fmt == WQ_INT3 || !x || !argmax) return WQ_ERR_ARG;
  if ((st = check_weights(fmt, codes, scale, zero)) != WQ_OK) return st;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scale, fmt == WQ_INT4H ? 4 : 16) || !aligned(zero, 16) ||
      (y && !aligned(y, 2)) || !aligned(argmax, 4))
    return WQ_ERR_ALIGN;
  if (K > 32768) return WQ_ERR_SHAPE;
  if ((st = check_device()) != WQ_OK) return st;
  const int bits = fmt == WQ_INT4 ? 4 : fmt == WQ_INT4H ? kStreamHier : 2;
  const StreamDesc d = {codes, scale, zero, x, y, N, K};
  g_am_smem = stream_plan(g_am_stream, bits, 1, &d, 1);
  if (g_am_smem == 0) return WQ_ERR_SHAPE;
  g_am_stream.am_out = reinterpret_cast<int*>(argmax);
  *workspace_needed = 16 + 8 * (size_t)stream_grid(g_am_stream);
  g_am_bits = bits;
  return WQ_OK;
}

int argmax_launch(void* workspace, cudaStream_t stream) {
  const int bits = g_am_bits;
  g_am_bits = 0;
  if (bits == 0) return WQ_ERR_ARG;
  g_am_stream.am_ws = static_cast<unsigned int*>(workspace);
  return note_cuda_error(launch_gemv_stream_argmax(g_am_stream, bits, g_am_smem, stream));
}

}  // namespace wq

extern "C" {

size_t wq_codes_bytes(int fmt, int64_t N, int64_t K) {
  if (check_shape(fmt, N, K) != WQ_OK) return 0;
  if (fmt == WQ_INT4 || fmt == WQ_INT4H) return (size_t)(N * K / 2);
  if (fmt == WQ_INT2) return (size_t)(N * K / 4);
  if (fmt == WQ_INT3) return (size_t)(N * K * 3 / 8);
  return (size_t)(N * 26 * (K / 128));
}

size_t wq_meta_count(int64_t N, int64_t K) {
  if (check_shape(WQ_INT4, N, K) != WQ_OK) return 0;
  return (size_t)(N * (K / 128));
}

size_t wq_scale_bytes(int fmt, int64_t N, int64_t K) {
  if (check_shape(fmt, N, K) != WQ_OK) return 0;
  return fmt == WQ_INT4H ? (size_t)(4 * N) : (size_t)(2 * N * (K / 128));
}

size_t wq_zero_bytes(int fmt, int64_t N, int64_t K) {
  if (check_shape(fmt, N, K) != WQ_OK || fmt == WQ_TERNARY) return 0;
  return fmt == WQ_INT4H ? (size_t)(N * (K / 32)) : (size_t)(2 * N * (K / 128));
}

int wq_quantize(const float* W, int64_t N, int64_t K, int fmt, int group, void* codes,
                uint16_t* scale, uint16_t* zero, void* stream) {
  int st = check_shape(fmt, N, K);
  if (st != WQ_OK) return st;
  if (group != (fmt == WQ_INT4H ? 32 : 128) || !W) return WQ_ERR_ARG;
  if ((st = check_weights(fmt, codes, scale, zero)) != WQ_OK) return st;
  if (!aligned(W, 16)) return WQ_ERR_ALIGN;
  if ((st = check_device()) != WQ_OK) return st;
  return cuda_status(wq::launch_quantize(W, N, K, fmt, codes, scale, zero, (cudaStream_t)stream));
}

int wq_gemm(const uint16_t* X, int64_t M, const void* codes, const uint16_t* scale,
            const uint16_t* zero, int fmt, int64_t N, int64_t K, uint16_t* Y, void* stream) {
  int st = check_shape(fmt, N, K);
  if (st != WQ_OK) return st;
  if (M < 1 || M > 2048) return WQ_ERR_SHAPE;
  if (!X || !Y) return WQ_ERR_ARG;
  if ((st = check_weights(fmt, codes, scale, zero)) != WQ_OK) return st;
  if (!aligned(X, 16) || !aligned(Y, 2)) return WQ_ERR_ALIGN;
  if ((st = check_device()) != WQ_OK) return st;
  if (fmt == WQ_INT4H) {
    if (M > wq::kStreamMaxRows || M * K > kHierMaxMK) return WQ_ERR_UNSUPPORTED;
    const wq_linear_desc d = {codes, scale, zero, X, Y, N, K, M};
    bool done = false;
    const int r = try_stream(fmt, 1, &d, M, (cudaStream_t)stream, &done);
    return done ? r : WQ_ERR_UNSUPPORTED;
  }
  if (fmt == WQ_INT3) {  // streaming kernel for M <= 4 where it applies, else one warp per row
    const wq_linear_desc d = {codes, scale, zero, X, Y, N, K, M};
    if (M <= wq::kStreamMaxRows) {
      bool done = false;
      const int r = try_stream(fmt, 1, &d, M, (cudaStream_t)stream, &done);
      if (done) return r;
    }
    return launch_int3(&d, 1, (cudaStream_t)stream);
  }
  {
    const wq_linear_desc d = {codes, scale, zero, X, Y, N, K, M};
    bool done = false;
    const int r = try_skinny(fmt, 1, &d, M, (cudaStream_t)stream, &done);
    if (done) return r;
  }
  if (fmt == WQ_INT4 && M >= wq::kTcMinM) {
    // tensor-core path: 128-row weight tiles x up to 256 tokens
    static thread_local wq::TcParams tp;  // ~20 KB: kept off the stack, one per thread
    const int bn = wq::tc_bn_for((int)M);
    if (!wq::tc_plan_mat(tp.m[0], X, (int)M, codes, scale, zero, Y, (int)N, (int)K, bn))
      return WQ_ERR_CUDA;
    tp.m[0].tile_begin = 0;
    tp.m[0].tile_end = tp.m[0].tiles_n * tp.m[0].tiles_m;
    tp.m[0].cost_begin = 0;
    tp.count = 1;
    tp.total_tiles = tp.m[0].tile_end;
    tp.total_cost = (int64_t)tp.total_tiles * tp.m[0].tile_cost;
    return cuda_status(wq::launch_gemm_tc(tp, (cudaStream_t)stream));
  }
  if (M <= wq::kStreamMaxRows) {
    const wq_linear_desc d = {codes, scale, zero, X, Y, N, K, M};
    bool done = false;
    int r = try_stream(fmt, 1, &d, M, (cudaStream_t)stream, &done);
    if (done) return r;
    if (M == 1) {
      r = try_rows(fmt, 1, &d, (cudaStream_t)stream, &done);
      if (done) return r;
    }
  }
  wq::SetParams p;
  p.count = 1;
  const int64_t items = plan_mat(p.m[0], fmt, codes, scale, zero, X, Y, N, K, M);
  p.m[0].item_begin = 0;
  p.m[0].item_end = (int)items;
  p.total_items = (int)items;
  return cuda_status(wq::launch_gemv_set(p, fmt, (int)M, (cudaStream_t)stream));
}

int wq_gemv(const uint16_t* x, const void* codes, const uint16_t* scale, const uint16_t* zero,
            int fmt, int64_t N, int64_t K, uint16_t* y, void* stream) {
  return wq_gemm(x, 1, codes, scale, zero, fmt, N, K, y, stream);
}

int wq_linear_set(const wq_linear_desc* descs, int count, int fmt, void* stream) {
  if (!descs || count < 1 || count > WQ_LINEAR_SET_MAX) return WQ_ERR_ARG;
  if (fmt < WQ_INT4 || fmt > WQ_INT4H) return WQ_ERR_ARG;
  static_assert(WQ_LINEAR_SET_MAX == wq::kSetMax, "set size");
  static thread_local wq::SetParams p;
  p.count = count;
  int64_t total = 0;
  const int64_t M = descs[0].M;
  for (int i = 0; i < count; ++i) {
    const wq_linear_desc& d = descs[i];
    int st = check_shape(fmt, d.N, d.K);
    if (st != WQ_OK) return st;
    if (d.M < 1 || d.M > 2048) return WQ_ERR_SHAPE;
    if (d.M != M) return WQ_ERR_ARG;
    if (!d.x || !d.y) return WQ_ERR_ARG;
    if ((st = check_weights(fmt, d.codes, d.scale, d.zero)) != WQ_OK) return st;
    if (!aligned(d.x, 16) || !aligned(d.y, 2)) return WQ_ERR_ALIGN;
    const int64_t items = plan_mat(p.m[i], fmt, d.codes, d.scale, d.zero, d.x, d.y, d.N, d.K, d.M);
    p.m[i].item_begin = (int)total;
    total += items;
    if (total > INT_MAX) return WQ_ERR_SHAPE;
    p.m[i].item_end = (int)total;
  }
  int st0 = check_device();
  if (st0 != WQ_OK) return st0;
  if (fmt == WQ_INT4H) {
    if (M > wq::kStreamMaxRows) return WQ_ERR_UNSUPPORTED;
    for (int i = 0; i < count; ++i)
      if (M * descs[i].K > kHierMaxMK) return WQ_ERR_UNSUPPORTED;
    bool done = false;
    const int r = try_stream(fmt, count, descs, M, (cudaStream_t)stream, &done);
    return done ? r : WQ_ERR_UNSUPPORTED;
  }
  if (fmt == WQ_INT3) {
    if (M <= wq::kStreamMaxRows) {
      bool done = false;
      const int r = try_stream(fmt, count, descs, M, (cudaStream_t)stream, &done);
      if (done) return r;
    }
    return launch_int3(descs, count, (cudaStream_t)stream);
  }
  {
    bool done = false;
    const int r = try_skinny(fmt, count, descs, M, (cudaStream_t)stream, &done);
    if (done) return r;
  }
  if (fmt == WQ_INT4 && M >= wq::kTcMinM) {
    // tensor-core GEMM: persistent launches of up to kTcMaxMats matrices each
    static thread_local wq::TcParams tp;
    // as few launches as the parameter block allows. Matrices are ordered by the cost of
    // their tiles (K), largest first, and dealt to the launches round robin, so that every
    // launch, whose CTAs take its tiles round robin, ends with small tiles on all SMs.
    const int launches = (count + wq::kTcMaxMats - 1) / wq::kTcMaxMats;
    static thread_local int order[WQ_LINEAR_SET_MAX];
    for (int i = 0; i < count; ++i) order[i] = i;
    for (int i = 1; i < count; ++i) {  // stable insertion sort by K, descending
      const int v = order[i];
      int j = i;
      while (j > 0 && descs[order[j - 1]].K < descs[v].K) {
        order[j] = order[j - 1];
        --j;
      }
      order[j] = v;
    }
    for (int l = 0; l < launches; ++l) {
      const int n = (count - l + launches - 1) / launches;  // matrices l, l + launches, ...
      int tiles = 0;
      int64_t cost = 0;
      for (int j = 0; j < n; ++j) {
        const wq_linear_desc& d = descs[order[l + j * launches]];
        wq::TcMat& t = tp.m[j];
        if (!wq::tc_plan_mat(t, d.x, (int)M, d.codes, d.scale, d.zero, d.y, (int)d.N, (int)d.K, wq::tc_bn_for((int)M)))
          return WQ_ERR_CUDA;
        t.tile_begin = tiles;
        t.cost_begin = cost;
        tiles += t.tiles_n * t.tiles_m;
        cost += (int64_t)t.tiles_n * t.tiles_m * t.tile_cost;
        t.tile_end = tiles;
      }
      tp.count = n;
      tp.total_tiles = tiles;
      tp.total_cost = cost;
      const int st = cuda_status(wq::launch_gemm_tc(tp, (cudaStream_t)stream));
      if (st != WQ_OK) return st;
    }
    return WQ_OK;
  }
  if (M <= wq::kStreamMaxRows) {
    bool done = false;
    int r = try_stream(fmt, count, descs, M, (cudaStream_t)stream, &done);
    if (done) return r;
    if (M == 1) {
      r = try_rows(fmt, count, descs, (cudaStream_t)stream, &done);
      if (done) return r;
    }
  }
  for (int i = count; i < wq::kSetMax; ++i) {
    memset(&p.m[i], 0, sizeof(p.m[i]));
    p.m[i].item_begin = p.m[i].item_end = (int)total;
  }
  p.total_items = (int)total;
  int st = check_device();
  if (st != WQ_OK) return st;
  return cuda_status(wq::launch_gemv_set(p, fmt, (int)M, (cudaStream_t)stream));
}

size_t wq_argmax_workspace_bytes(void) {
  if (check_device() != WQ_OK) return 0;
  const int sms = wq::device_sm_count();
  if (sms == 0) return 0;
  return 16 + 8 * (size_t)wq::kStreamMaxCtasPerSm * (size_t)sms;
}

int wq_gemv_argmax(const uint16_t* x, const void* codes, const uint16_t* scale, const uint16_t* zero, int fmt,
                   int64_t N, int64_t K, uint16_t* y, int32_t* argmax, void* workspace, size_t workspace_bytes,
                   void* stream) {
  if (!workspace) return WQ_ERR_ARG;
  if (!aligned(workspace, 16)) return WQ_ERR_ALIGN;
  size_t need = 0;
  const int st = wq::argmax_prepare(x, codes, scale, zero, fmt, N, K, y, argmax, &need);
  if (st != WQ_OK) return st;
  if (workspace_bytes < need) return WQ_ERR_ARG;
  return wq::argmax_launch(workspace, (cudaStream_t)stream);
}

const char* wq_status_str(int status) {
  switch (status) {
    case WQ_OK: return "WQ_OK";
    case WQ_ERR_ARG: return "WQ_ERR_ARG: invalid argument (null pointer, format or group)";
    case WQ_ERR_SHAPE: return "WQ_ERR_SHAPE: N, K or M outside the supported range";
    case WQ_ERR_ALIGN: return "WQ_ERR_ALIGN: pointer not aligned as required";
    case WQ_ERR_CUDA: return "WQ_ERR_CUDA: a CUDA call or launch failed";
    case WQ_ERR_UNSUPPORTED:
      return "WQ_ERR_UNSUPPORTED: not served here (needs an sm_100 (B200) device; WQ_INT4H needs M <= 4 and "
             "M * K <= 92160)";
    case WQ_ERR_SCRATCH: return "WQ_ERR_SCRATCH: the launch needs more scratch than the library's static array holds";
    default: return "unknown wq_status";
  }
}

int wq_last_cuda_error(void) { return g_last_cuda_error; }

int wq_debug_arm_timeout(unsigned int polls) {
  g_arm_polls = polls;
  return WQ_OK;
}

int wq_device_errors(unsigned int* flags, int clear, void* stream) {
  if (!flags) return WQ_ERR_ARG;
  int st = check_device();
  if (st != WQ_OK) return st;
  return cuda_status(wq::read_device_errors(flags, clear != 0, (cudaStream_t)stream));
}

}  // extern "C"
