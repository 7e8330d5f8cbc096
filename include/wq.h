/*
 * wq.h -- C ABI of libwq: group-quantised sub-byte weights times fp16 activations, on
 * NVIDIA B200 (sm_100a).
 *
 * What it computes.  A linear layer y = x . W^T whose weight W [N, K] (N output rows, K
 * along the reduction) is stored quantised in groups of 128 consecutive k of one row:
 *   - WQ_INT4 / WQ_INT3 / WQ_INT2: asymmetric round-to-nearest b-bit codes q in
 *     [0, 2^b - 1] with one fp16 scale s and one fp16 integer zero point z per group,
 *     w_hat = (q - z) * s (Whetstone README, "What the weights can actually survive":
 *     round-to-nearest, group 128, fp16 scale and zero per group; format table rows
 *     "int4 g128" 4.25, "int3 g128" 3.25 and "int2 g128" 2.25 bits/weight);
 *   - WQ_TERNARY: trits t in {-1, 0, +1} with one fp16 absmean scale per group,
 *     w_hat = t * s, five trits per byte in base 3 (format table row "ternary g128";
 *     TKintegers K5, "What is K5?": five balanced-ternary digits make a one-byte code).
 *   - WQ_INT4H: hierarchical int4 in groups of 32: 4-bit codes q in [0, 15]; per group g
 *     two 4-bit indices a_g, b_g; per row one fp16 pair (d, dm);
 *     w_hat = (d a_g) q - (dm b_g) (Whetstone README, "What the weights can actually
 *     survive": two 4-bit indices per group of 32 against an f16 pair per row, the GGUF
 *     Q4_K idea of "Prior art"; format table row "int4 hier-g32", 4.28 bits/weight).
 * Products accumulate in fp32; y is rounded to fp16 once, to nearest-even.
 * Batch-1 decode is bound by memory bandwidth (Whetstone README, "The one fact that
 * shapes everything": tok/s ceiling = bandwidth / bytes read per token), so the
 * matrix-vector kernels stream the packed codes once and never materialise w_hat.
 *
 * Quantiser definition (bit-exact between the GPU and the float64 reference), per
 * (row, group), all in float64 with correctly rounded division and rint = ties-to-even:
 *   int-b:   lo = min w, hi = max w, Q = 2^b - 1
 *            s = fp16_rne((hi - lo) / Q), s := 1 if s == 0
 *            z = clamp(rint(-lo / s), 0, Q),  q = clamp(rint(w / s) + z, 0, Q)
 *   ternary: a = (|w_0| + |w_1| + ... + |w_127|) / 128, summed left to right
 *            s = fp16_rne(a), s := 1 if s == 0,  t = clamp(rint(w / s), -1, 1)
 *   int4h (per row; groups of 32):
 *            per group: lo = min w, hi = max w, m_g = max(0, -lo), s_g = (hi + m_g) / 15
 *            d = rs(max_g s_g), dm = rs(max_g m_g), where rs(v) = fp16_rne(v / 15), except
 *            rs(0) = 1 and rs(v) = 2^-24 (smallest positive binary16) if v > 0 rounds to 0
 *            (Whetstone README, "New in 0.6.0": the shared row scale must not underflow)
 *            a_g = clamp(rint(s_g / d), 0, 15), b_g = clamp(rint(m_g / dm), 0, 15)
 *            S = d a_g, Z = dm b_g (exact), q = clamp(rint((w + Z) / S), 0, 15), q = 0 if S == 0
 * fp16_rne is the direct float64 -> binary16 rounding (never through float32).
 * Inputs must be finite.
 *
 * Layouts (all row-major, rows contiguous; G = K / 128):
 *   int4 codes   uint32 [N, K/8]    code k in word k/8,  bits 4*(k%8)..4*(k%8)+3
 *   int2 codes   uint32 [N, K/16]   code k in word k/16, bits 2*(k%16)..2*(k%16)+1
 *   int3 codes   uint32 [N, 3K/32]  code k at bits 3k..3k+2 of the row's little-endian
 *                                   bit stream (word j = stream bits 32j..32j+31; codes
 *                                   10 and 21 of every 32 straddle two words; a group is
 *                                   12 words)
 *   ternary      uint8  [N, 26*G]   group g of a row at bytes 26g..26g+25; byte j of a
 *                                   group = sum_{i<5} (t_{5j+i} + 1) * 3^i; byte 25 holds
 *                                   trits 125..127 and two pad trits 0 (digit 1); every
 *                                   byte is in 0..242
 *   scale, zero  fp16 bits (uint16) [N, G]; zero is unused (NULL) for WQ_TERNARY; a zero
 *                point is an integer in [0, 2^b - 1] (as wq_quantize writes it); the
 *                kernels use its nearest integer
 *   int4h        codes as int4 (uint32 [N, K/8]); `scale` is the row pair, fp16 bits
 *                uint16 [N, 2] = (d, dm); `zero` points to the index BYTES, uint8
 *                [N, K/32], byte g of a row = a_g | b_g << 4 (passed through the
 *                uint16_t* parameter); scale 4-byte and zero 16-byte aligned
 *   x, X, y, Y   fp16 bits (uint16), X [M, K] and Y [M, N] row-major
 *
 * Conventions.
 *   - Every pointer argument except `stream` is a DEVICE pointer owned by the caller;
 *     the library allocates no device memory and keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Work is enqueued asynchronously; a call returns once its kernels are launched.
 *   - Errors are returned as wq_status, never thrown. All argument checks happen before
 *     any launch: on a non-WQ_OK return from a check, nothing was enqueued and no
 *     output was touched. WQ_ERR_CUDA means a launch failed; outputs are then undefined.
 *   - Requirements: 1 <= N <= 2^31 - 1, 128 <= K <= 2^20 - 128 and K % 128 == 0;
 *     W (for wq_quantize), codes, x/X and y/Y 16-byte aligned; scale and zero 2-byte
 *     aligned; buffers may not overlap except inputs shared between calls.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { WQ_INT4 = 0, WQ_INT2 = 1, WQ_TERNARY = 2, WQ_INT3 = 3, WQ_INT4H = 4 } wq_fmt;

typedef enum {
  WQ_OK = 0,
  WQ_ERR_ARG = 1,          /* null pointer, unknown format, group != 128 */
  WQ_ERR_SHAPE = 2,        /* N, K or M outside the supported range, K % 128 != 0 */
  WQ_ERR_ALIGN = 3,        /* a pointer is not aligned as required above */
  WQ_ERR_CUDA = 4,         /* a CUDA call or launch failed (see wq_last_cuda_error) */
  WQ_ERR_UNSUPPORTED = 5,  /* valid request the library cannot serve here (no sm_100 GPU, or
                              WQ_INT4H outside its product range, see wq_gemm) */
  WQ_ERR_SCRATCH = 6       /* needs more scratch than the library's static array holds */
} wq_status;

/* Bytes of packed codes for an [N, K] weight in format fmt (0 on invalid arguments):
 * int4 and int4h N*K/2, int3 N*K*3/8, int2 N*K/4, ternary N*26*(K/128). */
size_t wq_codes_bytes(int fmt, int64_t N, int64_t K);

/* Number of fp16 entries of the scale array (and of the zero array) of the g128 formats:
 * N * K / 128. */
size_t wq_meta_count(int64_t N, int64_t K);

/* Bytes of the scale and of the zero array of an [N, K] weight in format fmt (0 on invalid
 * arguments, and wq_zero_bytes is 0 for WQ_TERNARY): 2 N K / 128 each for the g128 formats;
 * int4h 4 N (the row pairs) and N K / 32 (the index bytes). */
size_t wq_scale_bytes(int fmt, int64_t N, int64_t K);
size_t wq_zero_bytes(int fmt, int64_t N, int64_t K);

/* Quantise W (fp32 [N, K], device) into codes / scale / zero as defined above.
 * group must be 128 (32 for WQ_INT4H). zero must be NULL for WQ_TERNARY and non-NULL
 * otherwise. Whetstone README, "What the weights can actually survive" (round-to-nearest
 * group quantisation, hierarchical group-32 metadata) and TKintegers K5, "What is K5?"
 * (base-3 trit bytes). */
int wq_quantize(const float* W, int64_t N, int64_t K, int fmt, int group,
                void* codes, uint16_t* scale, uint16_t* zero, void* stream);

/* y[n] = fp16( sum_k x[k] * w_hat[n, k] ), fp32 accumulation, for one activation vector
 * x (fp16 [K]); y is fp16 [N]. Whetstone README, "The one fact that shapes everything"
 * (each weight read once, one multiply-add per weight). */
int wq_gemv(const uint16_t* x, const void* codes, const uint16_t* scale,
            const uint16_t* zero, int fmt, int64_t N, int64_t K, uint16_t* y,
            void* stream);

/* Y[m, n] = fp16( sum_k X[m, k] * w_hat[n, k] ) for M activation rows, 1 <= M <= 2048.
 * WQ_INT4H (a decode format) is served for M <= 4 and M * K <= 92160 only, with codes, zero
 * and X 16-byte aligned; other M or K give WQ_ERR_UNSUPPORTED (before any launch).
 * M = 1 runs the wq_gemv kernel. Small M streams the weights once and reuses each
 * dequantised weight for every row of X (int4 with 2 <= M <= 32: warp-level tensor-core
 * MMAs fed from registers); large M dequantises weight tiles into shared memory as fp16
 * tensor-core operands with fp32 accumulators (TKintegers K5, "What is K5?": tiles
 * expanded to fp16 tensor-core operands, fp32 accumulation). */
int wq_gemm(const uint16_t* X, int64_t M, const void* codes, const uint16_t* scale,
            const uint16_t* zero, int fmt, int64_t N, int64_t K, uint16_t* Y,
            void* stream);

/* One matrix of a linear set: Y = X . w_hat^T with this matrix's own X and Y. */
typedef struct {
  const void* codes;
  const uint16_t* scale;
  const uint16_t* zero;   /* NULL for WQ_TERNARY */
  const uint16_t* x;      /* fp16 [M, K] row-major (M = 1: one vector) */
  uint16_t* y;            /* fp16 [M, N] row-major */
  int64_t N;
  int64_t K;
  int64_t M;              /* rows of x and y, 1 <= M <= 2048 */
} wq_linear_desc;

/* Largest count accepted by wq_linear_set. */
#define WQ_LINEAR_SET_MAX 256

/* Run `count` independent products of one format as ONE persistent kernel launch per kind
 * of kernel (streaming kernel for M = 1 and for int2 / ternary up to M = 4, skinny-batch
 * kernel for int4 with 2 <= M <= 32, tensor-core GEMM for int4 with larger M -- split into
 * launches of at most 80 matrices --, the generic set kernel otherwise). `descs` is a
 * HOST array (read during the call, not kept); the pointers inside are device pointers.
 * Equivalent to count wq_gemm calls, without count launches: at batch 1 a whole decoded
 * token reads every weight once, and per-launch overhead dominates small matrices
 * (Whetstone README, "The baseline, and where the opportunity actually is": dispatch and
 * launch overhead, not bytes, set the baseline's speed). All entries must have the same
 * M. 1 <= count <= WQ_LINEAR_SET_MAX; each entry obeys the wq_gemm requirements. Results equal
 * the single calls' up to the fp32 summation order of rows whose groups straddle two units of
 * work (in practice the fp16 outputs are nearly always bit-identical); each call is
 * deterministic. */
int wq_linear_set(const wq_linear_desc* descs, int count, int fmt, void* stream);

/* Bytes of device work space wq_gemv_argmax needs on the current device (one 8-byte partial
 * per CTA of its launch plus a 16-byte header); 0 if no supported device is current. */
size_t wq_argmax_workspace_bytes(void);

/* Greedy pick fused into the output-projection product: y = x . w_hat^T exactly as wq_gemv
 * computes it (fp16, rounded once), and *argmax = the row n with the largest y[n], compared
 * as fp16 values, ties to the lowest n -- in one launch, with no read-back of y (Whetstone
 * README, notes on --temperature 0: greedy decoding stays on the GPU because the argmax is
 * written where the next step reads it).
 *   fmt        WQ_INT4, WQ_INT2 or WQ_INT4H (WQ_ERR_ARG otherwise).
 *   y          device fp16 [N], or NULL to skip storing the outputs.
 *   argmax     device int32, written with the row index.
 *   workspace  device buffer of at least wq_argmax_workspace_bytes() bytes, 16-byte aligned,
 *              zero-filled by the caller before its first use; every call leaves its first
 *              4 bytes zero again. Two calls that share a work space must not overlap on the
 *              GPU (same stream, or ordered by events).
 * codes, scale, zero and x must be 16-byte aligned (WQ_ERR_ALIGN; for WQ_INT4H scale 4-byte)
 * and K at most 32768 (WQ_ERR_SHAPE); other requirements as for wq_gemv. Inputs must be
 * finite. */
int wq_gemv_argmax(const uint16_t* x, const void* codes, const uint16_t* scale,
                   const uint16_t* zero, int fmt, int64_t N, int64_t K, uint16_t* y,
                   int32_t* argmax, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the library's own device array that wq_gemv_argmax_static uses as its scratch. */
#define WQ_ARGMAX_STATIC_SCRATCH_BYTES 16384

/* wq_gemv_argmax for callers that cannot give the library a work space: an engine that owns
 * all device memory through its own pool and does not let libraries call cudaMalloc, or a
 * decode loop in which an allocation (which can synchronise the device) is not acceptable.
 * There is no counterpart on the pages; this is a deployment convenience.
 * Same arguments and results as wq_gemv_argmax, without workspace / workspace_bytes. The
 * scratch is a static array of WQ_ARGMAX_STATIC_SCRATCH_BYTES bytes inside libwq, held by
 * every GPU that loads the library until the process exits; the call allocates nothing.
 * It returns WQ_ERR_SCRATCH, before any launch, if its launch on the current device would
 * need more (16 + 8 bytes per CTA, i.e. more than 2046 CTAs).
 * The first call on a device looks up the array's address on that device (make that first
 * call before any stream capture). Each call clears the array's header on `stream` before
 * its kernel runs. All calls share the one array: two calls whose work overlaps on the GPU
 * (different streams, not ordered by events) race and may return a wrong row. */
int wq_gemv_argmax_static(const uint16_t* x, const void* codes, const uint16_t* scale,
                          const uint16_t* zero, int fmt, int64_t N, int64_t K, uint16_t* y,
                          int32_t* argmax, void* stream);

/* Largest candidate count of wq_gemv_rescore. */
#define WQ_RESCORE_MAX_TOPK 64

/* Work-space bytes wq_gemv_rescore needs for N rows and topk candidates (0 if N or topk is
 * out of range: 1 <= N <= 524288, 1 <= topk <= WQ_RESCORE_MAX_TOPK). */
size_t wq_rescore_workspace_bytes(int64_t N, int topk);

/* Head rescoring (Whetstone README, feature list: --head-rescore keeps an fp16 copy of the
 * output projection and recomputes only the logits that decide the token).
 *   y           = the quantised head's logits, exactly as wq_gemv (fp16 [N]);
 *   cand[i]     = the rows of the topk largest y, largest first, equal y: lower row first
 *                 (int32 [topk]; only the first min(topk, N) entries are written);
 *   cand_logits = fp32 sum over k of x[k] * w16[cand[i], k] (float [topk]), each product exact;
 *   *token      = the candidate with the largest cand_logits, equal values: the lower row.
 * w16: the fp16 head, [N, K] row-major, 16-byte aligned (e.g. the fp32 weights rounded to
 * fp16). workspace: device memory of at least wq_rescore_workspace_bytes(N, topk) bytes,
 * 8-byte aligned, owned by the caller; no state is kept in it between calls. The other
 * arguments and requirements are wq_gemv's. All checks run before the first launch; three
 * launches on `stream` (the GEMV, a per-chunk top-k, one merge-and-recompute CTA). */
int wq_gemv_rescore(const uint16_t* x, const void* codes, const uint16_t* scale,
                    const uint16_t* zero, int fmt, const uint16_t* w16, int64_t N, int64_t K,
                    int topk, uint16_t* y, int32_t* cand, float* cand_logits, int32_t* token,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Static string naming a status code. */
const char* wq_status_str(int status);

/* The cudaError_t value of the last WQ_ERR_CUDA in this thread (0 if none). */
int wq_last_cuda_error(void);

/* Device-side error flags of this library on the current device, OR-ed over every kernel
 * since the last clear: bit 0 (WQ_DEVERR_TIMEOUT) = a bounded wait on an mbarrier inside a
 * kernel (the streaming matrix-vector kernel, the tensor-core GEMM) gave up; that launch's
 * outputs are undefined, and the kernel stopped computing, waited (bounded) for its copies
 * still in flight, freed its tensor memory and returned instead of hanging. Kernels run
 * after their call has returned, so a timeout cannot be a wq_status of that call; it is
 * reported here. `flags` is a HOST pointer. Synchronises `stream`; clears the flags if
 * clear != 0. */
#define WQ_DEVERR_TIMEOUT 1u
int wq_device_errors(unsigned int* flags, int clear, void* stream);

/* Failure-detection test hook (no counterpart on the pages). Arms the next wq_gemv / wq_gemm /
 * wq_linear_set call made on this host thread that launches the streaming matrix-vector
 * kernel (int4 / int2 / ternary with M = 1 .. 4): in that launch, one ring slot of warp 0 of
 * CTA 0 is never filled and every mbarrier wait gives up after `polls` polls. The wait on
 * the unfilled slot therefore runs out, and the kernel takes its error path (WQ_DEVERR_TIMEOUT
 * in wq_device_errors, outputs of that call undefined) without any GPU fault, trap or hang.
 * The next call runs normally. polls = 0 disarms. Always returns WQ_OK. */
int wq_debug_arm_timeout(unsigned int polls);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */
