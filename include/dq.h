/*
 * dq.h — C ABI of the DualQuant dual-scale solver for NVIDIA B200 (sm_100a).
 *
 * What is computed is the DualQuant hot path ("DualQuant: Dual-scale Calibration-free
 * Weight-and-Activation Quantization for LLMs"): for each weight matrix W (m x n,
 * out_features x in_features) a row-block scale r, a column scale c and 4-bit codes Q with
 * W ~ diag(r) Q diag(c), fitted by block coordinate descent with closed-form updates
 * (Abstract), the quantizer used as a black box and the scales projected onto the
 * format's admissible set after every update (acceptodds.com abstract of the same paper);
 * and the activation rescale by the column scales followed by 4-bit quantization
 * (Abstract; appendix Table 11, "Activation quantization (incl. beta)").
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" are CUDA device pointers; "host" are host pointers.
 *  - The caller allocates every buffer, including the workspace; the library never
 *    allocates, frees or keeps a pointer after the call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream). Outputs are valid once the stream has been synchronised.
 *  - Argument errors are returned synchronously before any work is queued. Conditions
 *    found on the device (non-finite input) raise a per-device error word that
 *    dq_last_device_error() reads and clears.
 *  - Layouts are row-major. Element codes are packed two per byte, the low nibble holding
 *    the even column. Block scales are stored one code per block: INT4 -> uint16 bf16 bit
 *    pattern, MXINT4/MXFP4 -> uint8 E8M0 (2^(code-127)), NVFP4 -> uint8 E4M3 multiplied by
 *    the fp32 tensor scale.
 */
#ifndef DQ_H_
#define DQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DQ_API __attribute__((visibility("default")))
#else
#define DQ_API
#endif

typedef enum {
  DQ_OK = 0,
  DQ_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad stride or alignment      */
  DQ_ERR_SHAPE = 2,         /* n not a multiple of the format's block length, too large  */
  DQ_ERR_DTYPE = 3,         /* unknown dtype / format / codec                            */
  DQ_ERR_WORKSPACE = 4,     /* workspace smaller than the *_workspace_bytes() figure     */
  DQ_ERR_NONFINITE = 5,     /* a NaN or Inf was found in an input (device-detected)      */
  DQ_ERR_TIMEOUT = 6,       /* a bounded device wait gave up (device-detected)           */
  DQ_ERR_CUDA = 7,          /* a CUDA runtime call failed                                */
  DQ_ERR_UNSUPPORTED = 8    /* a shape the kernels do not handle (e.g. rows too many)    */
} dq_status;

typedef enum {
  DQ_INT4 = 0, DQ_MXINT4 = 1, DQ_MXFP4 = 2, DQ_NVFP4 = 3, DQ_INT8 = 4, DQ_MXINT8 = 5
} dq_kind;

/* Format: kind plus block length along a row. INT4: group 64 or 128 (bf16 block scale,
 * elements -7..7). MXINT4: 32 (E8M0, elements -7..7). MXFP4: 32 (E8M0, E2M1 elements).
 * NVFP4: 16 (E4M3 block scale times an fp32 tensor scale, E2M1 elements). The 8-bit formats
 * of the DualQuant appendix's 8-bit table: INT8: group 128 (64 allowed), bf16 block scale,
 * elements -127..127; MXINT8: 32 (E8M0, elements -127..127). 4-bit codes are packed two per
 * byte (low nibble = even column), 8-bit codes one per byte (two's complement). */
typedef struct {
  int32_t kind;
  int32_t group;
} dq_format;

typedef enum { DQ_F32 = 0, DQ_BF16 = 1 } dq_dtype;

/* One matrix of a solve. All pointers are device pointers.
 *   W            [m, ldw] input weights (dtype of the call), 16-byte aligned, ldw*esize % 16 == 0
 *   r0           optional warm-start row-block scales [m, n/B] fp32 (projected on entry), or NULL
 *   c0           optional warm-start column scales [n] fp32 (finite, > 0), or NULL
 *   q_packed     out [m, n/2] uint8 (8-bit formats: [m, n], 16-byte aligned), the codes of
 *                the returned state
 *   r            out [m, n/B] fp32, decoded row-block scales
 *   c            out [n] fp32, column scales
 *   block_scales out [m, n/B] codes of r (uint16 bf16 bits for INT4/INT8, uint8 otherwise)
 *   tensor_scale out [1] fp32, NVFP4 only (may be NULL for the other formats)
 *   mse_trace    out [iters+1] fp64, ||W - W_hat||^2/||W||^2 after init and each iteration */
typedef struct {
  const void* W;
  int64_t m, n, ldw;
  const float* r0;
  const float* c0;
  uint8_t* q_packed;
  float* r;
  float* c;
  void* block_scales;
  float* tensor_scale;
  double* mse_trace;
} dq_matrix;

/* Workspace (device bytes) needed by dq_solve_batched for these shapes. `m`, `n` are host
 * arrays of `count` entries. Returns 0 for invalid arguments. */
DQ_API size_t dq_solve_workspace_bytes(int64_t count, const int64_t* m, const int64_t* n,
                                       dq_format fmt, int32_t iters);

/* Dual-scale BCD solve of `count` independent matrices (a full layer set in one call).
 * `mats` is a host array of descriptors. Per matrix: iteration 0 sets c = 1 (or c0) and
 * r = Pi_S(absmax/q_max) (or Pi_S(r0)); then `iters` iterations of
 *   Q-step  q = RNE_E(fl32(fl32(W * fl32(1/c)) * fl32(1/r)))
 *   r-step  r = Pi_S(sum_b W q c / sum_b (q c)^2)     per (row, block)
 *   c-step  c = sum_i W q r / sum_i (q r)^2           per column
 * (DualQuant Abstract: BCD with closed-form updates; acceptodds abstract: projection of the
 * scales after each update; Figure 2 (b): the trace, monotone by Theorem 1 (i)).
 * Returns DQ_ERR_SHAPE if some n is not a multiple of fmt.group, DQ_ERR_UNSUPPORTED if a
 * matrix has more rows than the kernel holds (see dq_solve_max_rows). */
DQ_API dq_status dq_solve_batched(const dq_matrix* mats, int64_t count, int32_t dtype,
                                  dq_format fmt, int32_t iters, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Which scales the iterations update: both (the method), only r (the c-step is skipped, c
 * stays at c0 or 1) or only c (the r-step and its projection are skipped, r stays at its
 * initial projected value). The ablation of the ai4snews summary of DualQuant, paragraph 2
 * (turning on only the row or only the column scales). */
typedef enum { DQ_UPDATE_BOTH = 0, DQ_UPDATE_ROW_ONLY = 1, DQ_UPDATE_COL_ONLY = 2 } dq_update;

/* Options of dq_solve_batched_ex. A NULL options pointer means {DQ_UPDATE_BOTH, NULL}.
 *   update   dq_update
 *   qchange  NULL, or a host array of `count` device pointers, each to [iters+1] fp64 that
 *            receive ||Q^t - Q^(t-1)||_F / ||Q^(t-1)||_F (DualQuant paper, Figure 2 (a)),
 *            with Q^t the Q-step result of iteration t and entries 0 and 1 equal to 0. The
 *            trace costs a second quantization of every element per iteration from t = 2
 *            on; it changes no other output. */
typedef struct {
  int32_t update;
  double* const* qchange;
} dq_solve_options;

/* Workspace for dq_solve_batched_ex with these options (the Q-change trace needs more). */
DQ_API size_t dq_solve_workspace_bytes_ex(int64_t count, const int64_t* m, const int64_t* n,
                                          dq_format fmt, int32_t iters,
                                          const dq_solve_options* options);

/* dq_solve_batched with options. DQ_ERR_INVALID_ARG for an unknown `update` or a null
 * pointer inside `qchange`. */
DQ_API dq_status dq_solve_batched_ex(const dq_matrix* mats, int64_t count, int32_t dtype,
                                     dq_format fmt, int32_t iters,
                                     const dq_solve_options* options, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* Single-matrix form of dq_solve_batched (same semantics, flat arguments). */
DQ_API dq_status dq_solve(const void* W, int32_t dtype, int64_t m, int64_t n, int64_t ldw,
                          dq_format fmt, int32_t iters, const float* r0, const float* c0,
                          uint8_t* q_packed, float* r, float* c, void* block_scales,
                          float* tensor_scale, double* mse_trace, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Bytes of the fixed scratch array that dq_solve_noalloc uses (per device). */
#define DQ_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

/* dq_solve without a workspace argument, for callers that cannot allocate device memory
 * (for example a host that hands all device memory to its own pool allocator and does not
 * allow a library to call cudaMalloc or any other allocating routine). The DualQuant pages
 * have no counterpart to this call; it exists only for such callers.
 * Same arguments, semantics and outputs as dq_solve, minus workspace and workspace_bytes.
 * Scratch: a fixed DQ_NOALLOC_SCRATCH_BYTES array inside libdq.so, held by every device
 * that loads it until the process exits. The driver places it in device memory when the
 * array's code module loads: at process start under CUDA_MODULE_LOADING=EAGER, otherwise
 * (lazy loading, the default) during the first call on the device. A host that hands all
 * device memory to its own pool should therefore make one call before doing so; once the
 * pool owns every byte, that first call fails with DQ_ERR_CUDA. The first call in each CUDA
 * context looks up the array's device address (cudaGetSymbolAddress) in that context and
 * keeps it for the context (keyed by the context's id, so a context created after a device
 * reset, or a second context on the device, looks it up afresh); make that first call before
 * any stream capture. The call allocates and frees nothing.
 * Every call on a device shares the one array and leaves its contents behind; the call
 * clears what must start at zero itself. Calls whose GPU work overlaps (different streams,
 * or different host threads, on the same device) race on the array: serialise them.
 * Returns DQ_ERR_WORKSPACE, before touching the device, when the shape and iteration count
 * need more scratch than DQ_NOALLOC_SCRATCH_BYTES (dq_solve_workspace_bytes tells how much). */
DQ_API dq_status dq_solve_noalloc(const void* W, int32_t dtype, int64_t m, int64_t n,
                                  int64_t ldw, dq_format fmt, int32_t iters, const float* r0,
                                  const float* c0, uint8_t* q_packed, float* r, float* c,
                                  void* block_scales, float* tensor_scale, double* mse_trace,
                                  void* stream);

/* Largest m the solver handles for a given n, format and dtype (0 if the format is bad). */
DQ_API int64_t dq_solve_max_rows(int64_t n, dq_format fmt, int32_t dtype);

/* Workspace (device bytes) needed by dq_act_quant: for NVFP4, one slot per CTA of the
 * amax pre-pass (16 KB; every call writes all the slots it reads, nothing needs clearing),
 * otherwise 256 bytes. */
DQ_API size_t dq_act_quant_workspace_bytes(int64_t tokens, int64_t n, dq_format fmt);

/* Activation rescale + block quantization (DualQuant Abstract: the column scales are
 * per-channel activation rescalings applied before activation quantization; appendix
 * Table 6: activation SQNR with and without them). With W_hat = diag(r) Q diag(c), the
 * quantized GEMM consumes c * x, so x~ = fl32(X * c) per channel (c NULL: x~ = X). Per
 * (token, block of B channels): a = max|x~|, d = Pi_S(a / q_max) (0 for a = 0; NVFP4 with
 * s_t = amax(x~)/2688), q = RNE_E(fl32(x~ * fl32(1/d))).
 *   X            device [tokens, ldx] (dtype), 16-byte aligned, ldx*esize % 16 == 0
 *   c            device [n] fp32 or NULL
 *   x_packed     device out [tokens, n/2] uint8, 4-byte aligned (8-bit formats: [tokens, n],
 *                8-byte aligned)
 *   scales       device out [tokens, n/B] (uint16 bf16 bits for INT4/INT8, uint8 otherwise)
 *   tensor_scale device out [1] fp32 (NVFP4; may be NULL otherwise) */
DQ_API dq_status dq_act_quant(const void* X, int32_t dtype, int64_t tokens, int64_t n,
                              int64_t ldx, const float* c, dq_format fmt, uint8_t* x_packed,
                              void* scales, float* tensor_scale, void* workspace,
                              size_t workspace_bytes, void* stream);

/* W4A4 GEMM on the quantized operands: the deployment side of the dual-scale model (the
 * ai4snews summary of DualQuant, paragraph 4: a real packed W4A4 inference path). With
 * W_hat = diag(r) Q diag(c) and the activation x~ = c * x quantized per (token, block) as
 * d * q_x, the layer output is
 *   y[t, i] = sum_j (d q_x)[t, j] * (r q)[i, j]
 * computed on the tensor cores (block-scaled FP4 MMA, fp32 accumulation). NVFP4 only:
 * E2M1 elements, E4M3 block scales per 16 elements, one fp32 tensor scale per operand.
 *   x_packed        device [T, K/2] uint8 (dq_act_quant's x_packed), 16-byte aligned
 *   x_scales        device [T, K/16] uint8 (its scales; code 0 = an all-zero block), 4-byte
 *                   aligned
 *   x_tensor_scale  device [1] fp32
 *   w_packed        device [N, K/2] uint8 (dq_solve's q_packed), 16-byte aligned
 *   w_scales        device [N, K/16] uint8 (its block_scales), 4-byte aligned
 *   w_tensor_scale  device [1] fp32 (its tensor_scale)
 *   y               device out [T, ldy] fp32, ldy >= N
 *   workspace       device scratch of dq_w4a4_gemm_workspace_bytes(T, N, K) bytes,
 *                   16-byte aligned (the scale factors re-laid for the tensor core)
 * Returns DQ_ERR_SHAPE if K is not a multiple of 64, DQ_ERR_UNSUPPORTED for another format,
 * DQ_ERR_WORKSPACE for a missing or small workspace; a bounded wait that gives up raises
 * DQ_ERR_TIMEOUT in the device error word. */
DQ_API size_t dq_w4a4_gemm_workspace_bytes(int64_t T, int64_t N, int64_t K);
DQ_API dq_status dq_w4a4_gemm(const uint8_t* x_packed, const uint8_t* x_scales,
                              const float* x_tensor_scale, int64_t T, const uint8_t* w_packed,
                              const uint8_t* w_scales, const float* w_tensor_scale, int64_t N,
                              int64_t K, dq_format fmt, float* y, int64_t ldy, void* workspace,
                              size_t workspace_bytes, void* stream);

/* W4A4 linear layer from the unquantized activation: the activation rescale + quantization
 * (dq_act_quant, NVFP4) as the producer of the W4A4 GEMM (dq_w4a4_gemm) in one call. One
 * pass over X forms x~ = fl32(X * c), quantizes it per (token, 16 channels) and writes the
 * codes and scale factors straight in the layouts the tensor core reads (no re-layout of the
 * activation's scale factors); the GEMM then consumes them with the solver's weight codes.
 * The result is bit-identical to dq_act_quant followed by dq_w4a4_gemm.
 *   X               device [T, ldx] (dtype), 16-byte aligned, ldx*esize % 16 == 0, ldx >= K
 *   c               device [K] fp32 (the solver's c) or NULL, 16-byte aligned
 *   w_packed, w_scales, w_tensor_scale, N, fmt, y, ldy: as for dq_w4a4_gemm (K = in
 *                   features, a multiple of 64)
 *   workspace       device scratch of dq_w4a4_linear_workspace_bytes(T, N, K, fmt) bytes,
 *                   16-byte aligned (the quantized activation and both operands' scale
 *                   factors in the tensor core's layout)
 * Errors as for dq_act_quant and dq_w4a4_gemm; a non-finite x~ raises DQ_ERR_NONFINITE in
 * the device error word. dq_w4a4_linear_workspace_bytes returns 0 for an unsupported format
 * or shape. */
DQ_API size_t dq_w4a4_linear_workspace_bytes(int64_t T, int64_t N, int64_t K, dq_format fmt);
DQ_API dq_status dq_w4a4_linear(const void* X, int32_t dtype, int64_t T, int64_t K,
                                int64_t ldx, const float* c, const uint8_t* w_packed,
                                const uint8_t* w_scales, const float* w_tensor_scale, int64_t N,
                                dq_format fmt, float* y, int64_t ldy, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Codecs used by the kernels, exposed for bit-exact tests (one code per output element). */
typedef enum {
  DQ_CODEC_INT4 = 0,   /* RNE to -7..7, saturating; code = two's-complement nibble (uint8) */
  DQ_CODEC_E2M1 = 1,   /* RNE to E2M1, saturating at 6; code = sign<<3 | magnitude (uint8) */
  DQ_CODEC_E4M3 = 2,   /* RNE to E4M3 (FN), saturating at 448 (uint8)                      */
  DQ_CODEC_E8M0 = 3,   /* nearest power of two, tie up, clamped to 2^-127..2^127 (uint8)  */
  DQ_CODEC_BF16 = 4,   /* RNE to bfloat16 (uint16 bit pattern)                             */
  DQ_CODEC_INT8 = 5    /* RNE to -127..127, saturating; code = two's-complement byte       */
} dq_codec;

/* x: device fp32 [count]; codes: device [count] of the codec's code type. */
DQ_API dq_status dq_encode(const float* x, int64_t count, int32_t codec, void* codes,
                           void* stream);
/* codes: device [count]; x: device fp32 [count] decoded values. */
DQ_API dq_status dq_decode(const void* codes, int64_t count, int32_t codec, float* x,
                           void* stream);

/* Synchronises `stream`, then returns and clears the device error word of the current
 * device: DQ_ERR_NONFINITE, DQ_ERR_TIMEOUT or DQ_OK (DQ_ERR_CUDA if a CUDA call fails). */
DQ_API dq_status dq_last_device_error(void* stream);

/* Measurement hooks (no computation). dq_set_timing_events: before the i-th launch of the
 * solve kernel made by this host thread the library records start_events[i] on the launch
 * stream and after it stop_events[i], for i < capacity; the events (cudaEvent_t, created by
 * the caller with timing enabled) stay the caller's. NULL / 0 disables. Returns
 * DQ_ERR_INVALID_ARG for a negative capacity or a NULL array with capacity > 0. */
DQ_API dq_status dq_set_timing_events(void* const* start_events, void* const* stop_events,
                                      int32_t capacity);
/* Number of solve-kernel launches recorded since the last dq_set_timing_events call. */
DQ_API int32_t dq_timing_events_used(void);
/* Kernels this library has launched from this process so far (all entry points). */
DQ_API int64_t dq_kernel_launches(void);

/* Human-readable name of a status code (static storage). */
DQ_API const char* dq_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* DQ_H_ */
