/*
 * qlora.h — C ABI of the B200 (sm_100a) QLoRA NF4 + LoRA quantized linear.
 *
 * The operation, as the sources state it:
 *
 *   h = dequant(W_NF4, c_block) x + (alpha/r) B A x
 *     «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나» (iq-universe blog),
 *     § "QLoRA의 수식: 두 항의 결합".
 *   Storage: blocks of 64 weights, one absmax scale per block, each weight a
 *   4-bit index of the nearest normal-quantile level; the scales themselves
 *   re-quantized to 8 bits ("double quantization"), about 4.13 bits/param;
 *   weights restored to bf16 just before each matmul.
 *     "48GB GPU Fine-Tuning a 65B Model: Where QLoRA Saves GPU Memory",
 *     § "Quantization Keeps the Patterns and Reduces Bits per Number";
 *     «QLoRA는 …», § "메모리 회계: 세 겹의 최적화" (restore formula
 *     c(q) * q2/256 * s_max, error at most s_max/256).
 *   Backward: W is frozen, gradients flow through the restored W to x and to
 *   A and B only.
 *     «QLoRA는 …», § "명제 1 · QLoRA Backward Unbiasedness";
 *     "48GB GPU …", § "QLoRA Puts the Two Methods in Different Places".
 *
 * Notation (row-major everywhere, tokens in rows):
 *   W  [N x K] bf16   frozen base weight (N = d_out, K = d_in, K % 64 == 0)
 *   x  [M x K] bf16   input tokens
 *   A  [r x K] bf16   LoRA down projection
 *   B  [N x r] bf16   LoRA up projection
 *   s = alpha / r
 *   y  = x W_hat^T + s (x A^T) B^T                         [M x N] bf16
 *   u' = bf16(s * x A^T)                                    [M x r] bf16
 *   dX = dY W_hat + s (dY B) A                              [M x K] bf16
 *   dA = s (dY B)^T x                                       [r x K] fp32
 *   dB = s dY^T (x A^T)                                     [N x r] fp32
 *
 * Stored format (readings where the sources are silent):
 *   codes       [N x K/2] u8   byte i of a row = (q[2i] << 4) | q[2i+1]
 *   scale_codes [N*K/64]  u8   q2 = min(255, rint(fl32(256 * absmax / s_max)))
 *   absmax      [ceil(N*K/64 / 256)] fp32   s_max per group of 256
 *                              consecutive blocks (row-major block order)
 *   restore:    w_hat = bf16_rne(fl32(c[q] * (fl32(q2 * s_max) * 2^-8)))
 *
 * Conventions for every call:
 *   - Memory is owned by the CALLER. The library never allocates, frees or
 *     synchronises; every device pointer must be 16-byte aligned.
 *   - Calls are asynchronous and ordered on the given CUDA stream
 *     (a cudaStream_t passed as void*; NULL = legacy default stream).
 *   - Argument, shape, alignment and device errors are returned
 *     synchronously, before anything is launched. A failed launch returns
 *     QLORA_ERR_CUDA. No C++ exception crosses the ABI.
 *   - Kernels never wait without a bound: a pipeline wait that exceeds about
 *     two seconds ends the kernel and sets a device status bit that
 *     qlora_device_status() reports as QLORA_ERR_TIMEOUT.
 *   - Inputs must be finite; results for non-finite weights are unspecified.
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, alpha/r not finite   */
  QLORA_ERR_SHAPE = 2,             /* K % 64 != 0, empty where not allowed, r range */
  QLORA_ERR_ALIGNMENT = 3,         /* a device pointer not 16-byte aligned          */
  QLORA_ERR_WORKSPACE = 4,         /* ws too small (see qlora_workspace_bytes)      */
  QLORA_ERR_UNSUPPORTED_DEVICE = 5,/* current device is not sm_100                 */
  QLORA_ERR_CUDA = 6,              /* a CUDA runtime / launch error                 */
  QLORA_ERR_TIMEOUT = 7            /* a kernel gave up on a bounded wait            */
} qlora_status_t;

/* Code of the 8-bit block-scale code under double quantization (the
 * 8-bit scale codes with 32-bit constants per group of 256 scales of
 * «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "메모리 회계: 세 겹의
 * 최적화"; the sources print the first, the other two are readings of the
 * same paragraph). Per group of 256 consecutive block scales s:
 *   QLORA_DQ_U8_256: one fp32 constant s_max = max s;
 *     q2 = min(255, rint(fl32(fl32(256 s) / s_max))) (unsigned),
 *     s_hat = fl32(q2 * s_max) * 2^-8; error at most s_max / 256.
 *   QLORA_DQ_U8_255: one fp32 constant s_max;
 *     q2 = min(255, rint(fl32(fl32(255 s) / s_max))) (unsigned),
 *     s_hat = fl32(fl32(q2 * s_max) / 255); error at most s_max / 510.
 *   QLORA_DQ_S8_MID: two fp32 constants mid = fl32(fl32(lo + hi) / 2) and
 *     half = fl32(fl32(hi - lo) / 2) (lo, hi = min, max s), stored as
 *     [mid, half] per group; q2 = clamp(rint(fl32(fl32(127 fl32(s - mid)) /
 *     half)), -127, 127) stored as an int8 byte (0 when half is 0),
 *     s_hat = fl32(mid + fl32(fl32(q2 * half) / 127)); error at most
 *     half / 254. rint rounds half to even. */
typedef enum { QLORA_DQ_U8_256 = 0, QLORA_DQ_U8_255 = 1, QLORA_DQ_S8_MID = 2 } qlora_dq_code_t;

/* Packed NF4 weight. All pointers are device pointers owned by the caller;
 * sizes from qlora_nf4_bytes_ex(). Formats («QLoRA는 어떻게 65B 모델을 GPU 한
 * 장에 올렸나», § "메모리 회계: 세 겹의 최적화"):
 *   dq_group = 256: double quantization (~4.13 bits/param): scale_codes holds
 *     one 8-bit code q2 per 64-weight block, absmax the group constants of
 *     dq_code (one float per 256 consecutive blocks, or two for
 *     QLORA_DQ_S8_MID); with QLORA_DQ_U8_256 the block scale is
 *     s_hat = fl32(q2 * s_max) * 2^-8;
 *   dq_group = 0: no double quantization (4.5 bits/param): absmax holds the
 *     fp32 block scale s_b itself, one per block; scale_codes is unused and
 *     may be NULL; dq_code is ignored. */
typedef struct {
  int64_t n_out;         /* N rows (d_out)                                     */
  int64_t k_in;          /* K columns (d_in), K % 64 == 0                      */
  int32_t block;         /* weights per absmax block: must be 64               */
  int32_t dq_group;      /* 256 (double quantization) or 0 (none)              */
  uint8_t *codes;        /* N*K/2 bytes                                        */
  uint8_t *scale_codes;  /* N*K/64 bytes (dq_group 256), unused for 0          */
  float *absmax;         /* group constants (dq_group 256: 1 or 2 floats per
                            ceil(N*K/64/256) groups), or N*K/64 block scales
                            (dq_group 0); 4-byte aligned                       */
  int32_t dq_code;       /* qlora_dq_code_t (dq_group 256)                     */
  int32_t reserved;      /* must be 0                                          */
} qlora_nf4_t;

/* Forward path selection for qlora_linear_fwd_ex. AUTO takes the decode GEMV
 * for m <= 16 and the tensor-core GEMM otherwise. */
typedef enum { QLORA_FWD_AUTO = 0, QLORA_FWD_GEMM = 1, QLORA_FWD_GEMV = 2 } qlora_fwd_path_t;

/* Byte sizes of the three stored arrays (codes, scale codes, fp32 scales or
 * group constants) for dq_group 256 or 0 and scale code dq_code; returns
 * their sum (0 on bad shape, dq_group or dq_code). out may be NULL. Host
 * only, no device work. */
QLORA_API size_t qlora_nf4_bytes_ex(int64_t n_out, int64_t k_in, int32_t dq_group, int32_t dq_code, size_t out[3]);

/* qlora_nf4_bytes_ex with dq_code QLORA_DQ_U8_256. */
QLORA_API size_t qlora_nf4_bytes(int64_t n_out, int64_t k_in, int32_t dq_group, size_t out[3]);

/* The library's own fp32 NF4 table (16 ascending levels in [-1, 1] with an
 * exact zero at index 7), computed on the host by Newton iteration on erfc:
 * 8 positive levels Phi^-1(d + j(1/2 - d)/8), j = 0..7, 7 negative levels
 * -Phi^-1(d + j(1/2 - d)/7), j = 0..6, and 0, d = ((1-1/30)+(1-1/32))/2,
 * divided by Phi^-1(d). Host only. */
QLORA_API qlora_status_t qlora_nf4_codebook(float out[16]);

/* Quantize a bf16 weight W [N x K] (device) into q (device buffers). One pass
 * over W: per-block absmax, nearest-level encode, nibble packing, and the
 * 8-bit double quantization of the scales. Bit-exact with the definition in
 * the stored-format paragraph above. */
QLORA_API qlora_status_t qlora_quantize_nf4(const void *w_bf16, const qlora_nf4_t *q, void *stream);

/* Restore W_hat [N x K] bf16 (device) from q. Bit-exact. */
QLORA_API qlora_status_t qlora_dequantize(const qlora_nf4_t *q, void *w_bf16_out, void *stream);

/* Workspace bytes for qlora_linear_fwd / _bwd at these sizes: covers both
 * calls, every forward path, and the stream-K schedule's fp32 partial slots
 * (up to 256 KB per SM) wherever some setting of qlora_set_gemm_schedule
 * could run stream-K, so the answer does not change with that setting. 0 for
 * arguments out of range. The size depends on the SM count of the current
 * device: ask with the device current that the calls will run on. A smaller
 * workspace, down to what qlora_fwd_workspace_bytes reports for the
 * forward, is accepted; the GEMMs then run data-parallel. */
QLORA_API size_t qlora_workspace_bytes(int64_t m, int64_t n_out, int64_t k_in, int32_t r);

/* The least workspace that qlora_linear_fwd accepts for these sizes (at most
 * qlora_workspace_bytes for the same sizes; without the stream-K slots). */
QLORA_API size_t qlora_fwd_workspace_bytes(int64_t m, int64_t n_out, int64_t k_in, int32_t r);

/* Forward: y [m x N] = x W_hat^T + s (x A^T) B^T, bf16 out, fp32 accumulate.
 * x [m x K], A [r x K], B [N x r] bf16 (device); 1 <= r <= 256; m >= 0
 * (m == 0 is a no-op). u_out [m x r] bf16 receives u' = bf16(s x A^T) for
 * the backward pass; it may be NULL. ws/ws_bytes: caller-owned scratch. */
QLORA_API qlora_status_t qlora_linear_fwd(const qlora_nf4_t *q, const void *x_bf16, int64_t m,
                                const void *a_bf16, const void *b_bf16, int32_t r, float alpha,
                                void *y_bf16, void *u_out_bf16, void *ws, size_t ws_bytes,
                                void *stream);

/* As qlora_linear_fwd, with the forward path chosen explicitly. */
QLORA_API qlora_status_t qlora_linear_fwd_ex(const qlora_nf4_t *q, const void *x_bf16, int64_t m,
                                   const void *a_bf16, const void *b_bf16, int32_t r,
                                   float alpha, void *y_bf16, void *u_out_bf16, void *ws,
                                   size_t ws_bytes, int32_t path, void *stream);

/* Size of the library-owned scratch array used by qlora_linear_fwd_noalloc
 * (8 MiB per GPU that loads the library, held until the process exits). */
#define QLORA_NOALLOC_SCRATCH_BYTES (8u << 20)

/* Forward for callers that cannot provide a workspace. The sources describe
 * no counterpart: it is a convenience of this library. Some callers have no
 * way to hand over scratch memory: a runtime whose device memory all belongs
 * to its own pool, code running where a device allocation is forbidden or
 * would stall other work (cudaMalloc may synchronise the device), or a plain
 * C caller with no device allocator. This call takes the arguments of
 * qlora_linear_fwd minus ws/ws_bytes and uses instead one fixed device array
 * of QLORA_NOALLOC_SCRATCH_BYTES owned by the library. It allocates and
 * frees nothing.
 *   - Results: it is qlora_linear_fwd given that array as a workspace of
 *     QLORA_NOALLOC_SCRATCH_BYTES bytes, and so bit-identical to
 *     qlora_linear_fwd called with a caller workspace of that same size. The
 *     array is too small for the stream-K slots, so the GEMM always runs the
 *     data-parallel schedule; where qlora_linear_fwd with a larger
 *     workspace would run stream-K (qlora_set_gemm_schedule), results agree
 *     within the forward's tolerance, not bit for bit.
 *   - Problems whose qlora_fwd_workspace_bytes() exceeds the array are
 *     rejected with QLORA_ERR_WORKSPACE before anything is launched. Ask
 *     that function beforehand: the need follows the split plan and is not
 *     monotone in m. On a 148-SM B200 at r <= 64 every m up to 2,304 tokens
 *     fits for 4096 x 11008 and 8192 x 22016 weights of either orientation
 *     (up to 6,272 for 11008 x 4096 and 4096 x 4096); at r = 256 up to 384.
 *   - The first call on each device (and the first after a cudaDeviceReset)
 *     looks up the array's device address with that device current; make
 *     that first call before any stream capture.
 *   - Every call shares the one array and leaves its contents behind; no part
 *     of it needs to start at zero (each call writes all it reads). Calls
 *     that overlap on the GPU (other streams, other host threads) race on it:
 *     keep them ordered, e.g. on one stream. */
QLORA_API qlora_status_t qlora_linear_fwd_noalloc(const qlora_nf4_t *q, const void *x_bf16, int64_t m,
                                                  const void *a_bf16, const void *b_bf16, int32_t r,
                                                  float alpha, void *y_bf16, void *u_out_bf16, void *stream);

/* Backward: dX [m x K] bf16 (may be NULL to skip), dA [r x K] fp32 and
 * dB [N x r] fp32 (overwritten, not accumulated). u_bf16 is the u' that the
 * forward produced ([m x r], may be NULL: then it is recomputed). No gradient
 * into W. Any N: when N % 8 != 0 the call first copies dY into the workspace
 * with its rows padded to a multiple of 8 (qlora_workspace_bytes counts it).
 * m == 0: dA and dB are set to zero; x, u, dY, A, B and dX are not read
 * (they may be NULL) and no workspace is needed. */
QLORA_API qlora_status_t qlora_linear_bwd(const qlora_nf4_t *q, const void *x_bf16, const void *u_bf16,
                                const void *dy_bf16, int64_t m, const void *a_bf16,
                                const void *b_bf16, int32_t r, float alpha, void *dx_bf16,
                                float *da, float *db, void *ws, size_t ws_bytes, void *stream);

/* LoRA merge for export: w_out [N x K] bf16 (device, row-major, caller-owned)
 * receives bf16(W_hat + (alpha/r) B A), with W_hat the restored weight of q
 * (exactly what qlora_dequantize writes), the rank-r product accumulated in
 * fp32 and one rounding to bf16 at the end. This is the export path of
 * "48GB GPU Fine-Tuning a 65B Model: Where QLoRA Saves GPU Memory":
 * § "LoRA Freezes the Original Weights ..." (B A has W's shape and is added
 * to it, so inference pays nothing extra) and § "QLoRA Puts the Two Methods
 * in Different Places" (with a 4-bit base the adapters are merged into the
 * restored 16-bit weights, not into the codes). A [r x K] and w_out must be
 * 16-byte aligned; B [N x r] 16-byte aligned when r % 8 == 0, else 2-byte
 * aligned. 1 <= r <= 256. */
QLORA_API qlora_status_t qlora_merge_lora(const qlora_nf4_t *q, const void *a_bf16, const void *b_bf16,
                                          int32_t r, float alpha, void *w_out_bf16, void *stream);

/* AdamW step for the LoRA adapters (A and B are the only trained
 * parameters; their Adam states m and v may live in CPU pinned memory:
 * «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "메모리 회계: 세 겹의 최적화",
 * Paged Optimizer). The update runs on the GPU; `master`, `m` and `v` may be
 * device memory or pinned host memory the GPU can address (then each step
 * moves 16 bytes per parameter over the host link and keeps nothing of it on
 * the device). Update, with t = step (1-based):
 *   m <- b1 m + (1-b1) g;  v <- b2 v + (1-b2) g^2;  p <- p (1 - lr wd)
 *   p <- p - (lr / (1-b1^t)) m / (sqrt(v) / sqrt(1-b2^t) + eps)
 * master (fp32, n), m, v (fp32, n) are updated in place; grad (fp32, n) is
 * read (e.g. dA or dB from qlora_linear_bwd); param_bf16 (n, may be NULL)
 * receives bf16(master) for the next forward. All fp32 pointers 4-byte
 * aligned (16-byte aligned ones take the vector path). Asynchronous on
 * `stream`: launch it on a second stream to overlap it with other work. */
typedef struct {
  float lr, beta1, beta2, eps, weight_decay;
  int32_t step;
} qlora_adamw_t;
QLORA_API qlora_status_t qlora_adamw_step(float *master, void *param_bf16, const float *grad, float *m,
                                          float *v, int64_t n, const qlora_adamw_t *hp, void *stream);

/* The same update on the host CPU (the page's paged optimizer: states in
 * CPU pinned memory, update on the CPU). All pointers are host memory;
 * param_bf16 (may be NULL) receives bf16(master) as uint16 bit patterns.
 * Synchronous; runs on a fixed pool of worker threads owned by the library.
 * Never touches the GPU. */
QLORA_API qlora_status_t qlora_adamw_host(float *master, void *param_bf16, const float *grad, float *m,
                                          float *v, int64_t n, const qlora_adamw_t *hp);

/* One paged optimizer step, enqueued on `stream` and fully asynchronous:
 * copy grad_dev (device, n fp32) to grad_host (pinned), run
 * qlora_adamw_host on the pinned master/m/v as a host function of the
 * stream, then copy param_host_bf16 (pinned, n bf16) to param_dev_bf16
 * (device; both NULL to skip). Issue it on a second stream once the
 * gradient is complete (cudaStreamWaitEvent) so that the copies and the CPU
 * update overlap the GPU's other work. All host buffers stay owned by the
 * caller and must outlive the step. */
QLORA_API qlora_status_t qlora_adamw_paged(const float *grad_dev, void *param_dev_bf16, float *master_host,
                                           float *m_host, float *v_host, float *grad_host,
                                           void *param_host_bf16, int64_t n, const qlora_adamw_t *hp,
                                           void *stream);

/* AdamW with m and v kept in pinned host memory and staged through device
 * memory (the paged optimizer with the copy engines doing the paging): on
 * `stream`, copy m_host, v_host (pinned, n fp32 each) into m_stage, v_stage
 * (device, n fp32 each, caller-owned scratch), run qlora_adamw_step on the
 * staged states, and copy them back. The transfers hold no SMs, so issued on
 * a second stream the update overlaps the kernels of other streams; two
 * such streams used in turn overlap the host-to-device and device-to-host
 * copies of consecutive updates. master, grad, param_bf16 as in
 * qlora_adamw_step (device). Arguments are checked before anything is
 * enqueued; m_stage and v_stage must not be in use by other work meanwhile.
 * Results are bit-identical to qlora_adamw_step on device-resident states. */
QLORA_API qlora_status_t qlora_adamw_staged(float *master, void *param_bf16, const float *grad, float *m_host,
                                            float *v_host, float *m_stage, float *v_stage, int64_t n,
                                            const qlora_adamw_t *hp, void *stream);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device. Returns QLORA_OK, QLORA_ERR_TIMEOUT (a kernel gave up on a
 * bounded wait; *bits, if non-NULL, gets which role), or QLORA_ERR_CUDA. */
QLORA_API qlora_status_t qlora_device_status(void *stream, uint32_t *bits);

/* Status bits that qlora_device_status() may return in *bits: which kind
 * of wait ran out of time. */
#define QLORA_STATUS_BIT_PRODUCER 0x1u  /* a load producer waited for a free stage */
#define QLORA_STATUS_BIT_MMA      0x2u  /* the MMA issuer waited for operands      */
#define QLORA_STATUS_BIT_RESTORE  0x4u  /* a restore warp waited for codes/scales  */
#define QLORA_STATUS_BIT_EPILOGUE 0x8u  /* the epilogue waited for an accumulator  */
#define QLORA_STATUS_BIT_SELFTEST 0x10u /* qlora_selftest_wait_timeout             */

/* Diagnostic for the failure-detection path (not part of the method): one
 * tiny kernel waits on a shared-memory barrier that nothing ever completes,
 * gives up after limit_us microseconds (clamped to [1, 2000000]), sets
 * QLORA_STATUS_BIT_SELFTEST and returns normally. The CUDA context stays
 * usable; qlora_device_status() then returns QLORA_ERR_TIMEOUT with that bit.
 * Lets a caller check that its error handling sees a timed-out wait without
 * any GPU fault. */
QLORA_API qlora_status_t qlora_selftest_wait_timeout(uint32_t limit_us, void *stream);

/* Work schedule of the CTA-pair GEMMs (forward y and backward dX); one
 * setting for the whole process, read once per call. Not part of the method
 * (the sources define what is computed, not how the work is split): a
 * performance choice of this library that changes results only in the order
 * of fp32 additions.
 *   QLORA_SCHED_AUTO (default): stream-K when the GEMM's reduction runs over
 *     at least 128 k-tiles of 64 (K >= 8192 for the forward, d_out >= 8192
 *     for dX) and its output tiles do not divide evenly over the SM pairs;
 *     otherwise data-parallel. Measured on B200: with shorter reductions the
 *     pairs' lockstep reuse of the input tiles in L2 is worth more than a
 *     balanced last wave; with longer ones stream-K is 5-13 % faster.
 *   QLORA_SCHED_DATA_PARALLEL: always data-parallel (tile q, q + pairs, ...).
 *   QLORA_SCHED_STREAM_K: stream-K whenever the tiles do not divide evenly.
 * Stream-K: all but the last full wave of tiles stay data-parallel, the rest
 * is cut into equal (tile, k-tile) ranges, one per SM pair, and a tile cut
 * between two pairs is finished from an fp32 partial passed through the
 * workspace. It needs the workspace size that qlora_workspace_bytes reports
 * under the same setting, and an output row stride that is a multiple of 8
 * elements; otherwise the call runs data-parallel. Both schedules give the
 * same results up to the order of fp32 additions. QLORA_ERR_INVALID_ARG for
 * an unknown mode. */
typedef enum {
  QLORA_SCHED_AUTO = 0,
  QLORA_SCHED_DATA_PARALLEL = 1,
  QLORA_SCHED_STREAM_K = 2
} qlora_sched_t;
QLORA_API qlora_status_t qlora_set_gemm_schedule(int32_t mode);
QLORA_API int32_t qlora_get_gemm_schedule(void);

/* Static description of a status code. */
QLORA_API const char *qlora_status_string(qlora_status_t s);

/* Number of kernels this library has launched in this process (all devices,
 * all streams) since it was loaded. Host only; lets a caller count the
 * device work behind a sequence of calls. */
QLORA_API uint64_t qlora_launch_count(void);

/* Library version as major*10000 + minor*100 + patch (1.1.0: qlora_nf4_t
 * gained dq_code and reserved; 1.2.0: qlora_adamw_staged). */
QLORA_API int32_t qlora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
