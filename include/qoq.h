/*
 * qoq.h -- C ABI of the B200 (sm_100a) W4A8 GEMM library with progressive
 * group quantization (QoQ).
 *
 * The method: "QServe: W4A8KV4 Quantization and System Co-design for
 * Efficient LLM Serving".  Weights are quantized in two levels (Methods,
 * 1) Algorithm: QoQ): first per output channel to symmetric INT8 with an
 * FP16 scale s1, inside a protective range, then per group of G input
 * channels to asymmetric UINT4 codes q with an INT8 group scale s2 and a UINT4
 * zero z.  Inside the GEMM the codes are turned back into INT8 with
 * register-level parallelism as dq = q*s2 - z*s2 (Methods, 2) System: QServe,
 * "subtraction after multiplication"), the products run on INT8 tensor cores
 * with INT32 accumulation, and the per-token x per-channel FP16 scaling is
 * applied once after the whole K reduction, so no partial sum is ever
 * dequantized (Background: the per-group W4A4 main loop that must dequantize
 * INT32 partial sums; "Part5 LLM部署技术", 3. 实践扩展：QServe（W4A8KV4）).
 *
 * Conventions for every entry point:
 *  - Pointers named as device pointers must point to device memory of the
 *    current CUDA device; the caller owns all memory.  The library allocates
 *    no device memory (the GEMM's split-K workspace is the caller's); the
 *    only state it keeps between calls is the
 *    device error word (qoq_device_error), the fixed scratch array of
 *    qoq_w4a8_gemm_static_ws, and host-side caches of device attributes, of
 *    the driver's tensor-map entry point and of that array's address.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    compute entry point only enqueues work on `stream` and returns without
 *    synchronizing, except the ones marked "synchronous".
 *  - Arguments are validated before anything is launched.  A violated
 *    precondition returns QOQ_ERR_INVALID_ARG, QOQ_ERR_UNSUPPORTED or
 *    QOQ_ERR_WORKSPACE and launches nothing.  A CUDA launch or driver error
 *    returns QOQ_ERR_CUDA.  No exception or abort crosses the ABI.
 *  - FP16 arrays hold IEEE binary16 values (`__half` / `torch.float16`).
 *    Inputs must be finite; this is not checked on the device.
 *  - Every device pointer must be 16-byte aligned.
 *  - Shapes: N % 128 == 0, K % 128 == 0, group in {64, 128}, K % group == 0,
 *    1 <= M, K <= 133120 (127 * 127 * K stays below 2^31, so INT32
 *    accumulation cannot overflow).
 *  - Requires a compute capability 10.0 device (B200); other devices get
 *    QOQ_ERR_UNSUPPORTED.
 */
#ifndef QOQ_H_
#define QOQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QOQ_API __attribute__((visibility("default")))
#else
#define QOQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  QOQ_OK = 0,
  QOQ_ERR_INVALID_ARG = 1,  /* bad pointer, shape or alignment */
  QOQ_ERR_UNSUPPORTED = 2,  /* valid but not supported (device, group, size) */
  QOQ_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  QOQ_ERR_WORKSPACE = 4,    /* the split-K workspace given is too small */
};

/* Human-readable text for a status code (static storage, never NULL). */
QOQ_API const char* qoq_status_str(int status);

/* Library ABI version (increments on any signature or layout change). */
QOQ_API int qoq_version(void);

/* Protective range of level 1 (119) and the UINT4 code range (15), so that
 * callers can check their own offline quantizers against the library. */
QOQ_API int qoq_protective_range(void);

/* ------------------------------------------------------------------------
 * Packed weight format
 *
 * The packed buffer is a sequence of blocks, one per (n-tile of 128 output
 * channels, k-tile of 128 input channels), n-tile major: block (nt, kt) starts
 * at byte (nt * (K/128) + kt) * qoq_packed_block_bytes(group).  A block holds
 *   codes : 8192 bytes = [j = 0..3][row = 0..127][16 bytes], the 16 bytes
 *           covering k = 32j .. 32j+31 of that row as four 32-bit words; word
 *           w (k0 = 32j + 8w) holds in byte b the codes q[k0+b] (low nibble)
 *           and q[k0+4+b] (high nibble), so one AND gives four codes in K
 *           order and one shift + AND the next four;
 *   s2    : 128 * (128/group) bytes = [g = group within tile][row], INT8;
 *   z     : 64 * (128/group) bytes  = [g][row/2], UINT4 zero of the even row
 *           in the low nibble and of the odd row in the high nibble.
 * This is the library's own answer to the pages' "compute-aware weight
 * reordering" (Methods, 2) System: QServe): each block is one contiguous
 * bulk copy, and the order matches the dequantizing threads' reads.
 * ---------------------------------------------------------------------- */

/* Bytes of one (128 x 128) block: 8192 + 192 for group 128, 8192 + 384 for
 * group 64.  Returns 0 for an unsupported group.  The block holds the
 * level-2 result of Methods, 1) Algorithm: QoQ (UINT4 codes, INT8 group
 * scales, UINT4 zeros per group of input channels). */
QOQ_API size_t qoq_packed_block_bytes(int group);

/* Bytes of the whole packed buffer for an N x K weight (0 if the shape is
 * invalid): N*K/2 bytes of UINT4 codes plus 1.5 bytes per group (s2, z),
 * the W4 storage of Methods, 1) Algorithm: QoQ. */
QOQ_API size_t qoq_packed_weight_bytes(int N, int K, int group);

/* ------------------------------------------------------------------------
 * Offline: progressive group quantization of a weight matrix.
 *   W      : device, FP16, N x K row-major (the [out, in] layout of a
 *            linear layer), read only.
 *   packed : device, qoq_packed_weight_bytes(N, K, group) bytes, written.
 *   s1     : device, FP16[N], written: per-output-channel level-1 scale.
 * Level 1: s1[n] = fp16(max_k |W[n,k]| / 119) (1.0 for an all-zero row, the
 * smallest positive FP16 if the quotient rounds to 0);
 * W8 = clamp(rne(W / s1), -119, 119) with an IEEE binary32 division.
 * Level 2, per group: mn = min(0, min W8), mx = max(0, max W8),
 * s2 = max(1, ceil((mx - mn) / 15)), z = rne(-mn / s2),
 * q = clamp(rne(W8 / s2) + z, 0, 15) (exact integer round-half-even).
 * Source: Methods, 1) Algorithm: QoQ and 2) System: QServe (protective
 * range).  Asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
QOQ_API int qoq_quantize_weights(const void* W, int N, int K, int group,
                         void* packed, void* s1, void* stream);

/* Pack already-quantized codes into the packed format (no quantization).
 *   q  : device, uint8 N x K, values 0..15;
 *   s2 : device, int8 N x (K/group), values 1..16;
 *   z  : device, uint8 N x (K/group), values 0..15;
 *   packed : device, written.
 * The caller guarantees |(q - z) * s2| <= 127 (true for every output of
 * qoq_quantize_weights); values outside the ranges give unspecified codes.
 * Asynchronous on `stream`. */
QOQ_API int qoq_pack_codes(const uint8_t* q, const int8_t* s2, const uint8_t* z,
                   int N, int K, int group, void* packed, void* stream);

/* Debug / inspection: unpack the packed format.  Any of q, s2, z, dq may be
 * NULL to skip it.  q: uint8 N x K; s2: int8 N x (K/group);
 * z: uint8 N x (K/group); dq: int8 N x K with dq = q*s2 - z*s2, computed
 * with the same byte-lane arithmetic as the GEMM main loop.
 * Source: Methods, 1) Algorithm: QoQ (the level-2 codes, scales and zeros)
 * and 2) System: QServe (dequantization to INT8, the zero subtracted after
 * the scale multiply).  q and dq must be 16-byte aligned.
 * Asynchronous on `stream`. */
QOQ_API int qoq_unpack_weights(const void* packed, int N, int K, int group,
                       uint8_t* q, int8_t* s2, uint8_t* z, int8_t* dq,
                       void* stream);

/* ------------------------------------------------------------------------
 * Online: per-token symmetric INT8 activation quantization.
 *   X  : device, FP16, M x K row-major, read only.
 *   X8 : device, int8 M x K row-major, written.
 *   sx : device, FP16[M], written.
 * sx[m] = fp16(max_k |X[m,k]| / 127) (1.0 for an all-zero row, the smallest
 * positive FP16 if the quotient rounds to 0);
 * X8 = clamp(rne(X / sx), -127, 127) with an IEEE binary32 division.
 * Source: the 8-bit activations of W4A8 (Insight; abstract of the QServe
 * page); per-token granularity as in the Background's W4A16 / W8A8
 * families.  Asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
QOQ_API int qoq_quantize_act_per_token(const void* X, int M, int K, int8_t* X8,
                               void* sx, void* stream);

/* ------------------------------------------------------------------------
 * Per-input-channel smoothing, SmoothQuant style ("Part5 LLM部署技术",
 * 1.1 权重-激活联合量化：SmoothQuant): part of the activations' outliers are
 * moved onto the weights with one factor s[k] per input channel, so that
 * X . W^T = (X / s) . (W * s)^T.  The factors are folded into the offline
 * weight quantization (so into s1) and into the per-token quantizer.
 * Readings where the page's formula is lost: migration strength 0.5 (the
 * default), s[k] = fp16(clamp(sqrt(max|Xcal[:,k]| / max|W[:,k]|), 2^-14,
 * 2^14)) with binary32 operations, 1 where either maximum is 0; the smoothed
 * operands are FP16: W' = fp16(W * s) (one rounding of the exact product),
 * X' = fp16(X / s) (binary32 quotient, then FP16).
 *
 * qoq_smooth_factors: s (device, FP16[K], written) from a calibration batch
 *   Xcal (device, FP16 Mc x K row-major) and W (device, FP16 N x K).
 * qoq_quantize_weights_smoothed: qoq_quantize_weights of W' = W * s.
 * qoq_quantize_act_per_token_smoothed: qoq_quantize_act_per_token of
 *   X' = X / s; feed X8 / sx to the GEMM with the smoothed weights.
 * s is 16-byte aligned.  As for every input, the smoothed values must be
 * finite (X / s overflows FP16 for |X| > 65504 * s).  Asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
QOQ_API int qoq_smooth_factors(const void* Xcal, int Mc, const void* W, int N, int K,
                               void* smooth, void* stream);
QOQ_API int qoq_quantize_weights_smoothed(const void* W, const void* smooth, int N, int K,
                                          int group, void* packed, void* s1, void* stream);
QOQ_API int qoq_quantize_act_per_token_smoothed(const void* X, const void* smooth, int M,
                                                int K, int8_t* X8, void* sx, void* stream);

/* ------------------------------------------------------------------------
 * The hot path: Y = (X8 . dq^T) * sx[m] * s1[n], FP16 out.
 *   X8     : device, int8 M x K row-major (from qoq_quantize_act_per_token).
 *   sx     : device, FP16[M].
 *   packed : device, packed weights (qoq_quantize_weights / qoq_pack_codes).
 *   s1     : device, FP16[N].
 *   Y      : device, FP16 M x N row-major, written (rows >= M untouched).
 *   ws, ws_bytes : device workspace for splitting K over several CTAs
 *            through L2, at least qoq_gemm_workspace_bytes(M, N, K, group)
 *            bytes (0 for shapes that are not split that way: a split of K
 *            into at most 8 parts for token tiles of 16, or 3 for tiles of
 *            32, runs on a thread-block cluster whose CTAs add their INT32
 *            partial tiles up in the leader CTA's shared memory and needs no
 *            workspace).  Owned by the caller, who fills it
 *            with zeros once before its first use (e.g. cudaMemset); every
 *            call that completes leaves its first 16 KiB (arrival counters,
 *            one per 32-channel slice of an output tile; K is split only when
 *            there are at most 1024 output tiles) at zero again, so it can be
 *            reused by later calls on the same stream whatever their shape.
 *            After a call that reported a device error (qoq_device_error) it
 *            must be zeroed again.  The rest holds INT32 partial sums.  Calls
 *            that can run at the same time (different streams) need
 *            different workspaces.  ws == NULL (with any ws_bytes) is an
 *            explicit request not to split K: the call runs unsplit (slower
 *            for small M).  A non-NULL ws smaller than the plan needs
 *            returns QOQ_ERR_WORKSPACE and launches nothing.
 * The UINT4 codes are dequantized to INT8 inside the main loop
 * (dq = q*s2 - z*s2, four byte lanes per 32-bit operation), multiplied on the
 * INT8 tensor cores (tcgen05, INT32 accumulators in tensor memory), and the
 * FP16 scaling runs once in the epilogue: Y = fp16_rn(float(acc) *
 * (float(sx[m]) * float(s1[n]))).  The token tile and the number of K splits
 * are chosen per (M, N, K); split partials are added exactly in INT32 (in a
 * cluster's leader CTA, or by the last CTA of an output tile to arrive)
 * before its epilogue.  The kernel may start as a programmatic dependent of
 * the preceding kernel on `stream`: it reads and writes nothing that kernel
 * may write before that kernel has completed.  Sources: Methods, 1) and 2);
 * Background.  Asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
QOQ_API int qoq_w4a8_gemm(const int8_t* X8, const void* sx, const void* packed,
                          const void* s1, int M, int N, int K, int group, void* Y,
                          void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * qoq_w4a8_gemm without a caller workspace, for callers that cannot allocate
 * device memory (for instance code that runs inside an allocator's own
 * callbacks, or a runtime that reserved all device memory up front and hands
 * out no scratch).  The method described in the pages has no counterpart to
 * this entry point; it exists only for such callers.
 *
 * Arguments and results are those of qoq_w4a8_gemm, with the same automatic
 * launch plan.  The K-split scratch is a fixed array of QOQ_STATIC_WS_BYTES
 * (16 MiB) in this library's device memory, one per device; the library
 * allocates nothing.
 *   - The first call on each device (with that device current) looks up the
 *     array's device address once; make that first call before any stream
 *     capture begins on that device.
 *   - A shape whose plan needs more scratch than the array holds
 *     (qoq_gemm_workspace_bytes(M, N, K, group) > QOQ_STATIC_WS_BYTES) is
 *     rejected with QOQ_ERR_UNSUPPORTED and nothing is launched; use
 *     qoq_w4a8_gemm with a workspace for it.  The automatic plan splits K
 *     through this scratch only for token tiles of 32 (more than 3 splits)
 *     and into at most 4 units per SM, so it needs at most 16 KiB + 4 * SMs
 *     * 32 * 128 * 4 bytes (about 9.7 MB with 148 SMs): on such a GPU no
 *     valid shape is rejected.  Plans that split K across a cluster, or do
 *     not split it, leave the array untouched.
 *   - Every call on a device uses the same array, and it keeps the last
 *     call's contents.  Each call that splits K clears the array's arrival
 *     counters on `stream` before its GEMM, so nothing from an earlier call
 *     (even one that failed) leaks into it.  Calls that may overlap in time
 *     (different streams, or several host threads) race on the array and give
 *     wrong results: order them on one stream or with events.
 * Asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
#define QOQ_STATIC_WS_BYTES ((size_t)16 << 20)
QOQ_API int qoq_w4a8_gemm_static_ws(const int8_t* X8, const void* sx, const void* packed,
                                    const void* s1, int M, int N, int K, int group,
                                    void* Y, void* stream);

/* Workspace bytes qoq_w4a8_gemm, qoq_w4a8_gemm_i32 and qoq_w4a8_linear use
 * for this shape (0 if K is not split, or if the shape is invalid): 16 KiB
 * of arrival counters plus the INT32 partial sums of the K splits.  Partial
 * sums stay INT32 and are added exactly before the single FP16 scaling
 * (Background: no dequantization of partial sums; Methods, 1) Algorithm:
 * QoQ, INT32 accumulation on INT8 tensor cores). */
QOQ_API size_t qoq_gemm_workspace_bytes(int M, int N, int K, int group);

/* Workspace bytes for an explicit configuration of qoq_w4a8_gemm_config
 * (tok_tile / splits as there, 0 = auto).  Same layout and source as
 * qoq_gemm_workspace_bytes. */
QOQ_API size_t qoq_gemm_workspace_bytes_config(int M, int N, int K, int group,
                                               int tok_tile, int splits);

/* Debug: the same main loop, storing the raw INT32 accumulator
 * acc[m, n] = sum_k X8[m,k] * dq[n,k] (device, int32 M x N row-major,
 * 16-byte aligned) instead of the scaled FP16 output.  This is the INT8 x
 * INT8 -> INT32 product of Methods, 1) Algorithm: QoQ (every GEMM on INT8
 * tensor cores) over the dequantized weights of 2) System: QServe, before
 * the per-token x per-channel scaling.  ws / ws_bytes and the errors as for
 * qoq_w4a8_gemm.  Asynchronous on `stream`. */
QOQ_API int qoq_w4a8_gemm_i32(const int8_t* X8, const void* packed, int M, int N,
                              int K, int group, int32_t* acc, void* ws,
                              size_t ws_bytes, void* stream);

/* The same GEMM with an explicit launch configuration (tuning and tests).
 *   tok_tile : token tile (MMA N): 16, 32, 64, 128, 176, 192 or 256, or 0
 *              for auto; 1 asks for the CUDA-core matrix-vector product
 *              (M <= 4 and the token rows within its shared memory, else
 *              QOQ_ERR_UNSUPPORTED), with `splits` its K ranges;
 *   splits   : K splits per output tile, 1..8 (at most K/128), or 0 for auto.
 * Exactly one of Y (FP16 output, needs sx and s1) and acc (INT32 output) is
 * non-NULL.  An explicit split count > 1 needs its workspace
 * (qoq_gemm_workspace_bytes_config), else QOQ_ERR_WORKSPACE (also for
 * ws == NULL).
 * Asynchronous on `stream`. */
QOQ_API int qoq_w4a8_gemm_config(const int8_t* X8, const void* sx, const void* packed,
                                 const void* s1, int M, int N, int K, int group,
                                 void* Y, int32_t* acc, int tok_tile, int splits,
                                 void* ws, size_t ws_bytes, void* stream);

/* The whole online path of one linear layer: per-token activation
 * quantization of X followed by the W4A8 GEMM, Y = X . W^T in FP16.
 *   X      : device, FP16 M x K row-major, read only.
 *   packed, s1 : the quantized weight (qoq_quantize_weights), N x K.
 *   X8, sx : device buffers of M x K int8 and M FP16 for the quantized
 *            activations (written; owned by the caller, reusable between
 *            calls on the same stream).
 *   Y      : device, FP16 M x N row-major, written.
 *   ws, ws_bytes : as for qoq_w4a8_gemm.
 * Same results (X8, sx and Y, bit for bit) as qoq_quantize_act_per_token
 * followed by qoq_w4a8_gemm.  Here the GEMM is launched as a programmatic
 * dependent of the quantizer, so it starts streaming weights while the
 * activations are still being quantized.  For M <= 2 x SMs the quantizer is
 * itself launched as a programmatic dependent of whatever kernel precedes
 * it on `stream`: it may be scheduled while that kernel drains, but touches
 * no memory before that kernel has completed.
 * Asynchronous on `stream`. */
QOQ_API int qoq_w4a8_linear(const void* X, int M, int K, const void* packed, const void* s1,
                            int N, int group, int8_t* X8, void* sx, void* Y, void* ws,
                            size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The MLP's gate_up projection with its output step fused into the GEMM
 * epilogue (kernel fusion, "Part5 LLM部署技术", 3. 实践扩展：QServe
 * （W4A8KV4）), for the SwiGLU MLP of the served models: the pages name the
 * models (Llama-3-8B, Qwen1.5-72B), not the formula, so the step taken is
 * H = fp16(silu(gate) * up), silu(x) = x / (1 + exp(-x)), and H is then
 * quantized per token to INT8 for the down projection.
 *
 * qoq_quantize_weights_gate_up: offline, the fused weight W (device, FP16,
 *   2I x K row-major: gate rows 0 .. I-1, then up rows I .. 2I-1; I % 64 ==
 *   0) quantized as qoq_quantize_weights, packed so that every 128-row tile
 *   t holds the gate rows 64t .. 64t+63 in its rows 0..63 and the up rows of
 *   the same channels in rows 64..127; s1 (FP16[2I]) in that packed order.
 * qoq_w4a8_gate_up_silu: X8 / sx (M x K, from qoq_quantize_act_per_token)
 *   times that weight; the epilogue writes H (device, FP16 M x I) instead of
 *   the 2I outputs, gate and up each formed exactly as qoq_w4a8_gemm forms
 *   an output (fp16 of acc * sx * s1), h = fp16(silu(g) * u) in binary32
 *   with the C library's expf.  K is not split.  Then H8 / sh (M x I INT8,
 *   FP16[M]) = qoq_quantize_act_per_token(H), launched as the GEMM's
 *   programmatic dependent: the operands of the down projection's
 *   qoq_w4a8_gemm.  Asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
QOQ_API int qoq_quantize_weights_gate_up(const void* W, int I, int K, int group, void* packed,
                                         void* s1, void* stream);
QOQ_API int qoq_w4a8_gate_up_silu(const int8_t* X8, const void* sx, const void* packed,
                                  const void* s1, int M, int I, int K, int group, void* H,
                                  int8_t* H8, void* sh, void* stream);

/* qoq_w4a8_linear as one kernel, for a few decode rows: the activation
 * quantizer fused into the GEMM ("Part5 LLM部署技术", 3. 实践扩展：QServe
 * （W4A8KV4）, kernel fusion).  Same arguments and the same results (X8, sx
 * and Y, bit for bit) as qoq_w4a8_linear.  Every CTA copies the FP16 rows
 * into its shared memory, computes each row's scale with the arithmetic of
 * qoq_quantize_act_per_token, writes all of X8 (every CTA writes the same
 * bytes; CTA 0 writes sx) and then runs the GEMM on it.
 *   - Applies when the rows fit 48 KiB (M * K * 2 <= 49152) and the GEMM's
 *     plan takes 16-token tiles without a cluster split; for one to four rows
 *     (where the automatic plan is the CUDA-core GEMV) it runs its own
 *     16-token plan, whose workspace size is
 *     qoq_gemm_workspace_bytes_config(M, N, K, group, 16, 0).  Otherwise
 *     QOQ_ERR_UNSUPPORTED and nothing is launched.
 *   - Measured on B200 in back-to-back decode it is slower than
 *     qoq_w4a8_linear's two kernels (the quantizer overlaps the GEMM's start,
 *     while here the rows are quantized inside the GEMM before its first
 *     MMA), so qoq_w4a8_linear does not use it.
 * Asynchronous on `stream`. */
QOQ_API int qoq_w4a8_linear_fused(const void* X, int M, int K, const void* packed,
                                  const void* s1, int N, int group, int8_t* X8, void* sx,
                                  void* Y, void* ws, size_t ws_bytes, void* stream);

/* The launch configuration qoq_w4a8_gemm picks for a shape: token tile,
 * K splits, CTAs in the grid and pipeline stages.  Host only: no CUDA call
 * beyond reading the SM count of the current device and (once per device)
 * how many thread-block clusters of the kernel fit on it; without a device
 * 148 SMs and 148 / splits clusters are assumed.  The
 * pages fix no tiling; this reports the library's own choice for the GEMM of
 * Methods, 1) Algorithm: QoQ.  For one to four tokens (when their INT8 rows
 * fit, with the per-warp copy rings, 227 KiB of shared memory) the product
 * may run on the CUDA cores as a matrix-vector product
 * with the same integer sums and epilogue: tok_tile = 0, stages = the
 * depth of each warp's weight copy ring (2 or 4), a CTA per 32 output
 * channels and K range (ctas = N / 32 * splits); a K split keeps an INT32
 * slice per range in the workspace.  It is taken for one token, and for two
 * to four when a launch-time model fitted on B200 prefers it to the 16-token
 * tensor-core tile (small weights). */
QOQ_API int qoq_gemm_plan(int M, int N, int K, int group, int* tok_tile, int* splits,
                  int* ctas, int* stages);

/* ------------------------------------------------------------------------
 * 4-bit KV cache and decode attention over it.
 * Source: "QServe: Cuantificación W4A8KV4 y Co-diseño del Sistema para un
 * Servicio Eficiente de LLM", abstract (W4A8KV4: the KV cache in 4 bits);
 * "QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM
 * Serving" (velog notes), Insight (the fused attention made memory-bound).
 * The pages give no cache format; this library's: every (token, KV head)
 * vector x of d = 128 FP16 values has UINT4 codes q, an FP16 scale s and an
 * FP16 offset m (the vector's minimum), x^ = s * q + m, with
 * s = fp16((max - min) / 15) and q = clamp(rne((x - min) / s), 0, 15)
 * computed in IEEE binary32 (q = 0 when s = 0).
 *
 * A cache of B sequences, Hkv KV heads and L token slots (L % 16 == 0) is
 * three caller-owned device arrays, 16-byte aligned, sizes from
 * qoq_kv4_cache_bytes:
 *   k_codes, v_codes  [B][Hkv][L / 16][1024] bytes each: per block of 16
 *            tokens, 32 runs of 32 bytes; run r (gid = r >> 2, tig = r & 3),
 *            32-bit word w (0..7), nibble p (bits 4p..4p+3; j = p & 3,
 *            e = p >> 2) holds
 *              K: token gid + 8 (j & 1), dimension 16w + 2 tig + e + 8 (j >> 1)
 *              V: token 2 tig + e + 8 (j >> 1), dimension 16w + gid + 8 (j & 1)
 *            of the block;
 *   scales   [B][Hkv][L][4] FP16: s_K, m_K, s_V, m_V of the token.
 * (The nibble orders are the operand layouts of the attention kernel's
 * tensor-core fragments, so each lane loads its 32 bytes in two pieces.)
 * Only d = 128 is supported (QOQ_ERR_UNSUPPORTED otherwise), and at most
 * 65535 (B * Hkv) pairs.
 * ---------------------------------------------------------------------- */
QOQ_API int qoq_kv4_cache_bytes(int B, int Hkv, int L, int d, size_t* k_bytes, size_t* v_bytes,
                                size_t* scale_bytes);

/* Quantize T new tokens of every (sequence, KV head) pair into cache slots
 * t0 .. t0 + T - 1 (0 <= t0, t0 + T <= L).  K, V: [B][Hkv][T][128] FP16
 * (device, 16-byte aligned).  Slots outside the range keep their codes and
 * scales (a block of 16 tokens that is written in part is read, merged and
 * written back).  Asynchronous on `stream`.  Errors: QOQ_ERR_INVALID_ARG for
 * NULL / misaligned pointers or a range outside the cache,
 * QOQ_ERR_UNSUPPORTED for d != 128 or L % 16 != 0. */
QOQ_API int qoq_kv4_quantize(const void* K, const void* V, int B, int Hkv, int T, int d, int L,
                             int t0, uint8_t* k_codes, uint8_t* v_codes, void* scales,
                             void* stream);

/* Workspace of qoq_kv4_decode_attention (its per-split partial results);
 * 0 for an unsupported shape. */
QOQ_API size_t qoq_kv4_attention_workspace_bytes(int B, int Hq, int Hkv, int L, int d);

/* Decode attention of one query token per sequence over the 4-bit cache:
 * out[b][h] = softmax_t(Q[b][h] . k^[b][h / g][t] / sqrt(128)) . v^[b][h / g]
 * over t < seqlen[b], with g = Hq / Hkv query heads per KV head (grouped-query
 * attention, g <= 8).  Q, out: [B][Hq][128] FP16 (device, 16-byte aligned);
 * seqlen: B int32 on the device, each clamped to [0, L]; a sequence of length
 * 0 gives out = 0.  The scores and sums are FP32, the softmax weights enter
 * the tensor cores as an FP16 pair (high and low part) per weight.  ws: at
 * least qoq_kv4_attention_workspace_bytes, 16-byte aligned (no zeroing
 * needed); QOQ_ERR_WORKSPACE when it is NULL or too small.  On `stream`: the
 * attention kernel, then a kernel that merges its splits of the sequence
 * when there is more than one. */
QOQ_API int qoq_kv4_decode_attention(const void* Q, const uint8_t* k_codes, const uint8_t* v_codes,
                                     const void* scales, const int* seqlen, int B, int Hq, int Hkv,
                                     int L, int d, void* out, void* ws, size_t ws_bytes,
                                     void* stream);

/* ------------------------------------------------------------------------
 * Device-side error word.  Every wait inside the kernels is bounded; a wait
 * that runs out sets a bit in this word and the kernel returns early
 * instead of hanging.  Synchronous (device-wide): reads the word of the
 * current device and, if `clear` is non-zero, resets it to 0.
 * Bits: 1 = producer wait, 2 = MMA wait, 4 = dequantizer wait,
 *       8 = epilogue wait, 16 = split-K arrival counter,
 *       64 = qoq_selftest_wait_timeout, 128 = a GEMM kernel launched with
 *       less shared memory than its layout needs (it did nothing).
 * ---------------------------------------------------------------------- */
QOQ_API int qoq_device_error(unsigned int* value, int clear);

/* Self-test of the bounded waits: launches one warp that waits, with the
 * same bounded mbarrier wait as every kernel of this library, on a barrier
 * that nothing arrives at.  The wait gives up after its SM-clock limit
 * (about 2 s at full clock), sets bit 64 in the device error word and the
 * kernel returns; the CUDA context stays usable.  It makes a stuck wait
 * observable without faulting or hanging the GPU.  Asynchronous on `stream`
 * (the kernel runs for about two seconds). */
QOQ_API int qoq_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QOQ_H_ */
