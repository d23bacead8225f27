/*
 * qg.h -- C ABI of the B200 (sm_100a) quantized-GEMM library (libqg.so).
 *
 * Computes Y = (x_scale * Xq) @ (w_scale * Wq) + bias and its weight-only
 * forms.  Every entry point takes plain pointers and sizes; no C++ or PyTorch
 * type crosses this boundary.
 *
 * Conventions shared by all entry points
 * --------------------------------------
 * Layout.  X is row-major [M, K] with leading dimension ldx >= K (elements).
 *   W is column-major [K, N] with stride [1, ldw], i.e. its storage is the
 *   row-major [N, K] matrix whose row n is output column n (what
 *   torch.empty(N, K).t() gives).  Y is row-major [M, N] with ldy >= N.
 *   (Page "量化算法的本质": X row-major stride [K,1], W column-major stride [1,K].)
 * Memory.  All array arguments are DEVICE pointers owned by the caller; the
 *   library allocates no device memory per call and keeps no pointer after
 *   returning, except a launch plan (qg_plan_*, below), a small host object
 *   that keeps the pointers it binds until qg_plan_destroy.
 * Stream.  Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and runs asynchronously; nothing synchronizes the host.
 * Errors.  Arguments are checked before anything is enqueued; a failed check
 *   returns a non-zero qg_status and enqueues nothing.  A launch failure
 *   returns QG_ERR_CUDA.  Kernels never trap: a device wait that exceeds its
 *   time limit records QG_ERR_TIMEOUT in a device status word and the kernel
 *   returns; qg_check_device_errors() reads (and clears) that word.
 *   qg_last_error_message() gives a one-line description of the last failure
 *   on the calling host thread.
 * Alignment.  Pointers to matrices (X, Xq, W, Wq, qweight, Y) must be 16-byte
 *   aligned and their leading dimensions must be multiples of 16 bytes
 *   (ldx*sizeof(elem) % 16 == 0); scale, zero, bias vectors need natural
 *   alignment.  Violations return QG_ERR_ALIGNMENT.
 * Sizes.  M, N, K >= 0 and below 2^31.  M == 0 or N == 0 is a no-op (QG_OK).
 *   K == 0 gives the empty sum: Y = bias (or 0).
 * Overflow.  int8 products accumulate in int32.  With |q| <= 127 the sum is
 *   exact for K <= 133144 (2^31 / 127^2); larger K returns QG_ERR_UNSUPPORTED.
 * Workspace.  The GEMM calls take an optional caller-owned device workspace
 *   (qg_gemm_workspace_size() bytes, 16-byte aligned, zero-filled before its
 *   first use).  With workspace == NULL (the fastest choice on B200 for the
 *   LLaMA-7B decode shapes) decode shapes (M <= 64) run the cluster split-K
 *   kernel, which needs no scratch memory.  With a workspace they run the
 *   stream-K kernel instead: one CTA per SM with equal shares of the weight
 *   stream; tiles shared by several CTAs are combined through the workspace,
 *   and the kernel leaves its counters zeroed again on exit.  A workspace
 *   must not be used by two calls that may execute at the same time; after a
 *   QG_ERR_TIMEOUT it must be zero-filled again.  Larger M takes no
 *   workspace: qg_gemm_w8a8 and its variants run persistent 128 x 256 tiles,
 *   or for M > 128 256-row tiles of 224..256 columns on two-CTA clusters (one
 *   tile per SM pair); the weight-only GEMMs run 128 x 128/256 tiles with K
 *   split over a cluster while the tiles leave SMs idle.
 */
#ifndef QG_H
#define QG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (binary-compatible with cudaStream_t). */
typedef struct CUstream_st *qg_stream_t;

typedef enum {
    QG_OK = 0,
    QG_ERR_INVALID_ARG = 1,  /* null pointer, negative or inconsistent size */
    QG_ERR_ALIGNMENT = 2,    /* pointer or leading dimension misaligned      */
    QG_ERR_UNSUPPORTED = 3,  /* valid request outside what is implemented     */
    QG_ERR_CUDA = 4,         /* CUDA runtime/driver error at launch           */
    QG_ERR_TIMEOUT = 5,      /* a kernel's bounded wait expired (device word) */
    QG_ERR_NO_DEVICE = 6,    /* no sm_100 device is current                   */
    QG_ERR_DEBUG_CHECK = 7   /* debug library only: a device-side check found an
                                index outside its buffer or a TMA coordinate
                                off its 16-byte rule; the access was skipped   */
} qg_status;

typedef enum {
    QG_F32 = 0,   /* float32 output                                           */
    QG_F16 = 1,   /* IEEE binary16 output (round to nearest even)              */
    QG_BF16 = 2,  /* bfloat16 output (round to nearest even)                   */
    QG_I32 = 3    /* raw int32 accumulator, W8A8 only (exactness checks)       */
} qg_dtype;

/* Activation applied in the GEMM epilogue to the fp32 value, before the
 * conversion to the output type (the *_act entry points below). */
typedef enum {
    QG_ACT_NONE = 0,
    QG_ACT_GELU = 1  /* gelu(v) = 0.5 v (1 + erf(v / sqrt 2)), the exact form */
} qg_activation;

/* Flags of the *_ex GEMM entry points (bitwise or). */
typedef enum {
    /* The caller guarantees that no kernel that may still be running when the
     * call's kernel starts writes the weight operand (codes, scales, zero
     * points): the weights were written, and completed, before any kernel
     * still in flight on the device was launched (for example, quantized once
     * at load time and followed by a synchronize).  The decode kernels (M <= 64,
     * no workspace) then load their first weight tiles -- and dequantize them --
     * before waiting on the preceding kernel of the stream, so a chain of
     * decode GEMMs streams weights across kernel boundaries.  Results are the
     * same bits as without the flag.  Other paths ignore it.  Breaking the
     * contract can read stale weights (wrong results, no fault). */
    QG_FLAG_STATIC_WEIGHTS = 1
} qg_flags;

/* 1 in the debug library (libqg_debug.so, built with QG_DEBUG), 0 in libqg.so.
 * The debug library checks, on the device, every TMA coordinate against the
 * 16-byte rule for its innermost coordinate and the hand-computed shared and
 * tensor memory offsets of the split-K exchanges against their areas; a failed
 * check records QG_ERR_DEBUG_CHECK (with the check's site) in the kernel's
 * status word, read by qg_check_device_errors, and skips the access (a wait on
 * a skipped copy then times out): no trap.  It computes the same results as
 * libqg.so.  A stand-in for a memory checker on small cases. */
int qg_debug_checks(void);

/* Human-readable name of a status code (static string). */
const char *qg_status_string(int status);

/* Description of the last failed call on this host thread ("" if none). */
const char *qg_last_error_message(void);

/* Library version as 10000*major + 100*minor + patch. */
int qg_version(void);

/* Bytes of workspace the GEMM calls use for an M x N x K problem on the
 * current device (0 if the shape never uses one).  The same size serves
 * qg_gemm_w8a8, qg_gemm_w8a16 and qg_gemm_w4a16. */
size_t qg_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/* Kernel families for qg_debug_inject_timeout. */
typedef enum {
    QG_DEBUG_WEIGHT_ONLY = 1,  /* cluster split-K weight-only kernel: qg_gemm_w8a16 / qg_gemm_w4a16 (and
                                  their _act and _sym forms) without a workspace */
    QG_DEBUG_STREAM_K = 2      /* stream-K decode kernel: the GEMM calls given a workspace, and
                                  qg_gemm_w4a16_noalloc */
} qg_debug_family;

/* Fault injection for tests; the library never arms it itself.  Arms the NEXT
 * launch of one kernel family (from any host thread) to fail in a controlled
 * way: its first CTA skips the copy of its first K block, so the waits on that
 * copy can never complete, and every bounded wait of that launch gives up after
 * `wait_limit_us` microseconds (100 .. 1000000) instead of one second.  The
 * launch then ends by itself: its waits expire, it records QG_ERR_TIMEOUT in the
 * device status word, waits (bounded) for the copies it did issue, frees its
 * tensor memory and exits; qg_check_device_errors() then returns
 * QG_ERR_TIMEOUT.  Its output is undefined, and a workspace it used must be
 * zero-filled again before reuse (qg_gemm_w4a16_noalloc does that itself).
 * Nothing faults or traps; later launches run normally.  This is how the
 * timeout path is tested ("INT4/FP16混合精度GEMM" §7.1 lists the checks to make
 * when a kernel misbehaves).  Returns QG_ERR_INVALID_ARG for an unknown family
 * or a limit out of range. */
qg_status qg_debug_inject_timeout(int family, int wait_limit_us);

/* Sets a tuning switch for the rest of the process (or until set again) and
 * returns QG_OK, or QG_ERR_INVALID_ARG for an unknown name.  Each switch starts
 * from the environment variable of the same name, read once per process;
 * unset, the library uses its measured defaults.  Switches choose among
 * kernels and launch shapes that give the same results (the parity tests
 * compare them this way); none changes what is computed.
 *   "QG_W8A8_PAIR"     1 (default): W8A8 with M > 128 on two-SM CTA-pair tiles;
 *                      0: one-SM 128 x 256 tiles
 *   "QG_PAIR_STAGES"   7: seven ring stages in the CTA-pair kernel (default 6)
 *   "QG_W8A8_SPLITS", "QG_W8A16_SPLITS", "QG_W4A16_SPLITS"
 *                      decode cluster size (K splits, 1..8); 0 (default): automatic
 *   "QG_WONLY_BN"      weight-only token tile width 16/32/64/128/256; 0: automatic
 *   "QG_PAIR_N"        CTA-pair tile width in output columns (a multiple of 16,
 *                      128..256); 0 (default): chosen by waves
 * Not synchronized with launches already enqueued (they keep their choice);
 * set switches before the calls they should affect. */
qg_status qg_set_tuning(const char *name, int value);

/* Synchronizes `stream`, then reads and clears the device status word that
 * kernels set when a bounded wait expires.  Returns QG_OK, QG_ERR_TIMEOUT or
 * QG_ERR_CUDA. */
qg_status qg_check_device_errors(qg_stream_t stream);

/*
 * qg_quantize_rowwise_int8 -- symmetric per-row int8 quantization (dynamic,
 * per token).  Page "量化算法的本质", per_channel_quant_int8, symmetric branch;
 * page "量化与多精度算子" §二 (z = 0, range [-127, 127]) and §六 (rounding).
 *
 * For every row m of X (IEEE binary16):
 *   a = max(max_k |x[m,k]|, 1e-10)         (binary32)
 *   q[m,k] = clamp(rint(x[m,k] * (127/a)), -127, 127)
 *           (127/a and the product rounded to binary32, rint = half to even)
 *   x_scale[m] = a / 127                    (binary32 division)
 * Results are bit-exact IEEE binary32 operations.
 *
 *   x        [in]  device, fp16 [M, ldx] row-major, 16-byte aligned, ldx % 8 == 0
 *   xq       [out] device, int8 [M, ldxq] row-major, 16-byte aligned, ldxq % 16 == 0
 *   x_scale  [out] device, float32 [M]
 * Applied to the [N, K] storage of a column-major weight, the same call is the
 * per-output-column weight quantizer (w_scale[N]).
 */
qg_status qg_quantize_rowwise_int8(const void *x, int64_t ldx, int8_t *xq, int64_t ldxq,
                                   float *x_scale, int64_t M, int64_t K, qg_stream_t stream);

/*
 * qg_quantize_rowwise_asym_int8 -- asymmetric per-row int8 quantization (the
 * asymmetric branch of per_channel_quant_int8 on page "量化算法的本质"; page
 * "量化与多精度算子" §二: x ~= s (q - z)).  For every row m of X (binary16):
 *   mn, mx = min and max of the row            (0, 0 for K == 0)
 *   s = max((mx - mn) / 255, 1e-8)             (binary32 division)
 *   z = -mn / s - 128                          (binary32; z is not rounded)
 *   q[m,k] = clamp(rint(x[m,k] / s + z), -128, 127)  (binary32 divide, add;
 *                                              rint = half to even)
 *   qsum[m] = sum_k q[m,k]                     (exact)
 * Results are bit-exact IEEE binary32 operations.  Applied to the [N,K]
 * storage of a weight it is the per-output-column weight quantizer.
 *
 *   x      [in]  device, fp16 [M, ldx] row-major, 16-byte aligned, ldx % 8 == 0
 *   xq     [out] device, int8 [M, ldxq], ldxq % 16 == 0
 *   scale, zero  [out] device, float32 [M]
 *   qsum   [out] device, int32 [M], or NULL
 * K must be <= 131071.
 */
qg_status qg_quantize_rowwise_asym_int8(const void *x, int64_t ldx, int8_t *xq, int64_t ldxq,
                                        float *scale, float *zero, int32_t *qsum, int64_t M, int64_t K,
                                        qg_stream_t stream);

/*
 * qg_quantize_block_asym4 -- block-wise asymmetric 4-bit weight quantization
 * and packing (offline step for qg_gemm_w4a16).  Page "从零实现大语言模型 INT8
 * 量化", 第一步/第二步 (block of 64, scale = (max-min)/(levels-1),
 * zero = round(-min/scale), q = round(w/scale) + zero) with 16 levels; scale
 * floor 1e-5 as in page "量化算法的本质", GPTQ MARLIN (clamp(min=1e-5));
 * packing as page "INT4/FP16混合精度GEMM" §4.1-4.2 ((w >> 4i) & 0xF, (K/8, N)).
 *
 * For every output column n and block b of `group` consecutive k:
 *   s = fp16(max((max - min) / 15, 1e-5))   (binary32, then nearest-even fp16)
 *   z = clamp(rint(-min / s), 0, 15)        (stored as fp16 integer)
 *   q = clamp(rint(w / s) + z, 0, 15)       (quantized with the fp16 s)
 * Bit-exact.
 *
 *   w        [in]  device, fp16 [N, ldw] (storage of column-major [K, N]), ldw % 8 == 0
 *   qweight  [out] device, int32 [N, K/8]: word p of row n holds k = 8p..8p+7,
 *                  code j in bits 4j..4j+3 (low nibble first)
 *   scale    [out] device, fp16 [K/group, N] row-major
 *   zero     [out] device, fp16 [K/group, N] row-major (integers 0..15)
 *   group    must be 64 (QG_ERR_UNSUPPORTED otherwise); K % 64 == 0
 */
qg_status qg_quantize_block_asym4(const void *w, int64_t ldw, int32_t *qweight, void *scale,
                                  void *zero, int64_t N, int64_t K, int64_t group,
                                  qg_stream_t stream);

/*
 * qg_gemm_w8a8 -- Y = (x_scale * Xq) @ (w_scale * Wq) + bias with int8 x int8
 * products accumulated in int32 in tensor memory and the dequantization fused
 * into the epilogue (the int32 accumulator is never written to global memory).
 * Page "量化算法的本质", W8A8矩阵乘法; page "量化与多精度算子" §四 (int32
 * accumulate, dequant in the epilogue); page "Ascend C per-channel INT8 GEMM"
 * §5.4 (scale at write-back).
 *
 *   y[m,n] = float(acc[m,n]) * (x_scale[m] * w_scale[n]) + bias[n]
 *   acc[m,n] = sum_k xq[m,k] * wq[k,n]  (exact int32)
 *
 *   xq       [in]  device, int8 [M, ldx] row-major, ldx % 16 == 0
 *   wq       [in]  device, int8 column-major [K, N] stored [N, ldw], ldw % 16 == 0
 *   x_scale  [in]  device, float32 [M]
 *   w_scale  [in]  device, float32 [N]
 *   bias     [in]  device, float32 [N], or NULL for none
 *   y        [out] device, [M, ldy] row-major of type y_dtype (qg_dtype):
 *                  QG_F32, QG_F16, QG_BF16, or QG_I32 (raw acc; scales and
 *                  bias ignored and may be NULL)
 *   workspace, workspace_bytes  optional, see "Workspace" above
 */
qg_status qg_gemm_w8a8(const int8_t *xq, int64_t ldx, const int8_t *wq, int64_t ldw,
                       const float *x_scale, const float *w_scale, const float *bias,
                       void *y, int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K,
                       void *workspace, size_t workspace_bytes, qg_stream_t stream);

/*
 * qg_gemm_w8a8_zp -- W8A8 with zero points (asymmetric operands).  Page
 * "量化与多精度算子" §二: with x ~= s_x (q_x - z_x) and w ~= s_w (q_w - z_w),
 * the product is the integer dot product plus correction terms; page
 * "量化算法的本质" (zero optional: present = asymmetric).
 *   y[m,n] = x_scale[m] * w_scale[n] * (acc[m,n] - w_zero[n] * x_qsum[m]
 *            - x_zero[m] * w_qsum[n] + K * x_zero[m] * w_zero[n]) + bias[n]
 *   acc[m,n] = sum_k xq[m,k] * wq[k,n]   (exact int32)
 * The bracket is formed in fp64 and rounded once to fp32; then, as in
 * qg_gemm_w8a8, fp32 multiply by x_scale * w_scale and add bias.
 *
 *   xq, ldx, wq, ldw, x_scale, w_scale, bias, y, y_dtype, ldy  as qg_gemm_w8a8
 *   x_zero, w_zero  [in] device float32 [M] / [N], or NULL (that operand symmetric)
 *   x_qsum, w_qsum  [in] device int32 [M] / [N]: the code row sums of Xq and of
 *                   the [N,K] Wq storage (qg_quantize_rowwise_asym_int8 writes
 *                   them).  w_zero requires x_qsum; x_zero requires w_qsum.
 * Codes may span [-128, 127]; K must be <= 131071.  QG_I32 returns acc.
 */
qg_status qg_gemm_w8a8_zp(const int8_t *xq, int64_t ldx, const float *x_scale, const float *x_zero,
                          const int32_t *x_qsum, const int8_t *wq, int64_t ldw, const float *w_scale,
                          const float *w_zero, const int32_t *w_qsum, const float *bias, void *y,
                          int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K, qg_stream_t stream);

/*
 * qg_quantize_gemm_w8a8 -- qg_quantize_rowwise_int8 of X followed by
 * qg_gemm_w8a8, as ONE kernel for decode batches (M <= 64).  Page "量化算法的
 * 本质", W8A8矩阵乘法 (one operator should be one kernel; the separate
 * quantize / post-process kernels are the slow variant); page "量化与多精度
 * 算子" §四 (convert late, on chip).  Every CTA computes the row scales of X
 * itself and quantizes the K blocks it multiplies straight into shared memory,
 * so Xq never goes through global memory.
 *
 * Results are bit-identical to the two calls: the same binary32 operations
 * decide every code and scale, and the int32 accumulation is exact.
 *
 *   x        [in]  device, fp16 [M, ldx] row-major, 16-byte aligned, ldx % 8 == 0
 *   wq, w_scale, bias, y, y_dtype, ldy   as qg_gemm_w8a8
 *   xq       [out] optional (NULL): int8 [M, ldxq], ldxq % 16 == 0 -- the codes
 *   x_scale  [out] optional (NULL): float32 [M] -- the row scales
 * M > 64 returns QG_ERR_UNSUPPORTED (use the two calls).  With K == 0 or
 * N == 0 there is no product: Y = bias (or 0), and the requested xq / x_scale
 * are still written (with N == 0 and K > 0 they must be requested together).
 */
qg_status qg_quantize_gemm_w8a8(const void *x, int64_t ldx, const int8_t *wq, int64_t ldw,
                                const float *w_scale, const float *bias, void *y, int y_dtype,
                                int64_t ldy, int8_t *xq, int64_t ldxq, float *x_scale, int64_t M,
                                int64_t N, int64_t K, qg_stream_t stream);

/*
 * qg_gemm_w8a16 -- weight-only int8: Y = X @ (w_scale * Wq) + bias, X fp16.
 * Page "量化算法的本质" (W8A16 naming: fp16 activations, int8 weights); page
 * "量化与多精度算子" §四 (weights stored int8, dequantized on chip, fp16 GEMM
 * with fp32 accumulation).  Int8 codes convert to fp16 exactly on chip; the
 * per-column scale is applied to the fp32 accumulator in the epilogue.
 *
 *   y[m,n] = fp16( w_scale[n] * sum_k x[m,k] * wq[k,n] + bias[n] )
 *
 *   x        [in]  device, fp16 [M, ldx] row-major, ldx % 8 == 0
 *   wq       [in]  device, int8 column-major [K, N] stored [N, ldw], ldw % 16 == 0
 *   w_scale  [in]  device, float32 [N]
 *   bias     [in]  device, float32 [N] or NULL
 *   y        [out] device, fp16 [M, ldy] row-major
 *   workspace, workspace_bytes  optional, see "Workspace" above
 */
qg_status qg_gemm_w8a16(const void *x, int64_t ldx, const int8_t *wq, int64_t ldw,
                        const float *w_scale, const float *bias, void *y, int64_t ldy,
                        int64_t M, int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                        qg_stream_t stream);

/*
 * qg_gemm_w4a16 -- weight-only 4-bit block-asymmetric: Y = X @ Wdq + bias with
 * Wdq[k,n] = (q[k,n] - zero[k/group, n]) * scale[k/group, n].  Page
 * "INT4/FP16混合精度GEMM" §3.2, §4.2 (unpack, (q - zp) * scale, fp16 matmul
 * with fp32 accumulate, fp16 out); page "从零实现大语言模型 INT8 量化" (block
 * dequant); page "量化与多精度算子" §三 §四 (per-group, on-chip dequant).
 * The dequantized weight is formed in fp16 on chip (one rounding of (q-z)*s).
 *
 *   x        [in]  device, fp16 [M, ldx] row-major, ldx % 8 == 0
 *   qweight  [in]  device, int32 [N, K/8] as produced by qg_quantize_block_asym4
 *   scale    [in]  device, fp16 [K/group, N]
 *   zero     [in]  device, fp16 [K/group, N]
 *   group    must be 64; K % 64 == 0
 *   bias     [in]  device, float32 [N] or NULL
 *   y        [out] device, fp16 [M, ldy] row-major
 *   workspace, workspace_bytes  optional, see "Workspace" above
 */
qg_status qg_gemm_w4a16(const void *x, int64_t ldx, const int32_t *qweight, const void *scale,
                        const void *zero, int64_t group, const float *bias, void *y, int64_t ldy,
                        int64_t M, int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                        qg_stream_t stream);

/*
 * qg_gemm_w8a8_ex, qg_gemm_w8a16_ex, qg_gemm_w4a16_ex -- qg_gemm_w8a8,
 * qg_gemm_w8a16 and qg_gemm_w4a16 with a `flags` argument (qg_flags bits; 0
 * is the plain call).  Same arguments, layouts, results and errors otherwise;
 * an unknown flag bit returns QG_ERR_INVALID_ARG.  QG_FLAG_STATIC_WEIGHTS is
 * the serving case of the pages' weight-only decode ("量化与多精度算子" §四:
 * weights quantized offline and only read at inference): the decode kernels
 * start streaming the weights before the preceding kernel has finished.
 */
qg_status qg_gemm_w8a8_ex(const int8_t *xq, int64_t ldx, const int8_t *wq, int64_t ldw,
                          const float *x_scale, const float *w_scale, const float *bias,
                          void *y, int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K,
                          void *workspace, size_t workspace_bytes, unsigned flags, qg_stream_t stream);
qg_status qg_gemm_w8a16_ex(const void *x, int64_t ldx, const int8_t *wq, int64_t ldw,
                           const float *w_scale, const float *bias, void *y, int64_t ldy,
                           int64_t M, int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                           unsigned flags, qg_stream_t stream);
qg_status qg_gemm_w4a16_ex(const void *x, int64_t ldx, const int32_t *qweight, const void *scale,
                           const void *zero, int64_t group, const float *bias, void *y, int64_t ldy,
                           int64_t M, int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                           unsigned flags, qg_stream_t stream);

/*
 * qg_quantize_block_sym4 -- block-wise symmetric int4 weight quantization and
 * packing.  Page "INT4/FP16混合精度GEMM" §5.1 (scale = max|w| / 7, q =
 * round(w / scale), INT4 range [-8, 7]); §3.2/§4.2 (8 codes per word, element
 * i at (w >> 4i) & 0xF).  For every column n and block b of 64 consecutive k
 * of the [N,K] storage of a column-major fp16 weight:
 *   s32 = max(max|w| / 7, 1e-5)   s = fp16(s32), stored and used to quantize
 *   q   = clamp(rint(w / s), -8, 7)        (binary32 division, half to even)
 * qweight [N, K/8] int32: nibble j of word p is k = 8p + j as a two's-
 * complement 4-bit code; scale [K/64, N] fp16.  group must be 64.
 */
qg_status qg_quantize_block_sym4(const void *w, int64_t ldw, int32_t *qweight, void *scale, int64_t N,
                                 int64_t K, int64_t group, qg_stream_t stream);

/*
 * qg_quantize_channel_sym4 -- per-output-column symmetric int4 for the int8
 * tensor path (qg_gemm_w4a8).  Same formulas with one block per column and the
 * scale kept in binary32: a = max(max_k |w|, 1e-10); s = a / 7;
 * q = clamp(rint(w / s), -8, 7).  Same packing; scale [N] float32.
 * K % 32 == 0.
 */
qg_status qg_quantize_channel_sym4(const void *w, int64_t ldw, int32_t *qweight, float *scale, int64_t N,
                                   int64_t K, qg_stream_t stream);

/*
 * qg_gemm_w4a8 -- int8 activations x int4 weights on the int8 tensor cores.
 * Page "Ascend C per-channel INT8 GEMM" §9.1 (unpack int4 to int8, then the
 * int8 GEMM; half the weight bytes); page "量化与多精度算子" §四.
 *   y[m,n] = x_scale[m] * w_scale[n] * sum_k xq[m,k] * q4[k,n] + bias[n]
 * with q4 the sign-extended codes of qg_quantize_channel_sym4; the int32
 * accumulation is exact and the epilogue is qg_gemm_w8a8's.  The packed tile
 * is unpacked to int8 in shared memory right before the MMA.
 *   xq, ldx, x_scale, w_scale, bias, y, y_dtype, ldy   as qg_gemm_w8a8
 *   qweight [in] device int32 [N, K/8] (qg_quantize_channel_sym4), K % 32 == 0
 * Tuned for decode (M <= 64); larger M runs correctly on 64-row tiles.
 */
qg_status qg_gemm_w4a8(const int8_t *xq, int64_t ldx, const int32_t *qweight, const float *x_scale,
                       const float *w_scale, const float *bias, void *y, int y_dtype, int64_t ldy,
                       int64_t M, int64_t N, int64_t K, qg_stream_t stream);

/*
 * qg_gemm_w4a16_sym -- W4A16 with symmetric group-int4 weights (no zero
 * points): y[m,n] = sum_k x[m,k] * q4[k,n] * s[k/64, n] + bias[n], q4 and s
 * from qg_quantize_block_sym4.  Same kernels as qg_gemm_w4a16: each code q is
 * read as its offset form q + 8 with zero point 8, and fp16(q * s) is the
 * dequantized weight.  Arguments as qg_gemm_w4a16 without zero and workspace.
 */
qg_status qg_gemm_w4a16_sym(const void *x, int64_t ldx, const int32_t *qweight, const void *scale,
                            int64_t group, const float *bias, void *y, int64_t ldy, int64_t M, int64_t N,
                            int64_t K, qg_stream_t stream);

/*
 * qg_gemm_w8a8_act, qg_gemm_w8a16_act, qg_gemm_w4a16_act -- the GEMMs above
 * with an activation fused into the epilogue: Y = act(GEMM(...)), the
 * activation applied to each fp32 output value before its conversion, so the
 * pre-activation result never reaches global memory.  Page
 * "INT4/FP16混合精度GEMM" §8 (fused linear_gelu: the GEMM result is not written
 * back before gelu); page "量化与多精度算子" §四 (the epilogue is where
 * elementwise work rides along).  Arguments as the base calls, without the
 * workspace pair (these run the cluster kernels), plus `activation`
 * (qg_activation).  QG_I32 output with an activation is QG_ERR_INVALID_ARG.
 */
qg_status qg_gemm_w8a8_act(const int8_t *xq, int64_t ldx, const int8_t *wq, int64_t ldw,
                           const float *x_scale, const float *w_scale, const float *bias,
                           void *y, int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K,
                           int activation, qg_stream_t stream);
qg_status qg_gemm_w8a16_act(const void *x, int64_t ldx, const int8_t *wq, int64_t ldw,
                            const float *w_scale, const float *bias, void *y, int64_t ldy,
                            int64_t M, int64_t N, int64_t K, int activation, qg_stream_t stream);
qg_status qg_gemm_w4a16_act(const void *x, int64_t ldx, const int32_t *qweight, const void *scale,
                            const void *zero, int64_t group, const float *bias, void *y,
                            int64_t ldy, int64_t M, int64_t N, int64_t K, int activation,
                            qg_stream_t stream);

/*
 * qg_gemm_w4a16_noalloc -- qg_gemm_w4a16 for decode batches (M <= 16) that
 * allocates nothing.  The pages describe no such call: it exists for callers
 * that may not allocate device memory, such as code running inside a runtime
 * that owns all device memory through its own pool and forbids allocation at
 * execute time, or latency-bound loops that cannot afford cudaMalloc/cudaFree
 * (which may synchronize the device and cost far more than the GEMM).
 *
 * Same arguments, layouts and result as qg_gemm_w4a16 without the workspace
 * pair; it runs the stream-K decode kernel with its scratch in a 4 MiB static
 * device array of the library, which every device that loads the library holds
 * until the process exits.  No cudaMalloc, cudaFree or other allocating call
 * is made.
 *   - M > 16, or a problem whose stream-K scratch on the current device is
 *     larger than 4 MiB, returns QG_ERR_UNSUPPORTED with a message.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any
 *     stream capture.
 *   - Each call zeroes the scratch's arrival counters on `stream` before the
 *     kernel; the rest of the array keeps the last call's contents.
 *   - All calls share one array per device: calls that may run at the same time
 *     on the GPU (other streams, other host threads) race and give wrong
 *     results.  Serialize them, e.g. on one stream.
 */
qg_status qg_gemm_w4a16_noalloc(const void *x, int64_t ldx, const int32_t *qweight,
                                const void *scale, const void *zero, int64_t group,
                                const float *bias, void *y, int64_t ldy, int64_t M, int64_t N,
                                int64_t K, qg_stream_t stream);

/*
 * Launch plans.  The pages describe no such call: it exists for loops that
 * issue the same call with the same preallocated buffers again and again (a
 * decode step per token), where the caller's per-call argument marshalling
 * costs as much host time as the launch itself.
 *
 * qg_plan_quantize_rowwise_int8, qg_plan_gemm_w8a8, qg_plan_gemm_w8a16,
 * qg_plan_gemm_w4a16 bind the arguments of qg_quantize_rowwise_int8,
 * qg_gemm_w8a8_ex, qg_gemm_w8a16_ex and qg_gemm_w4a16_ex (everything but the
 * stream; same meaning, layouts and flags) into a new plan stored in *plan;
 * qg_plan_launch(plan, stream) then makes that call on `stream` and returns
 * its status.
 *   - A plan holds the pointers and sizes, not the data: the caller keeps
 *     every buffer alive while the plan is launched and may rewrite the
 *     buffers' contents between launches (new activations, in place).
 *   - Creation only records the arguments (it fails only for a NULL `plan`,
 *     QG_ERR_INVALID_ARG, or when the host is out of memory, QG_ERR_UNSUPPORTED);
 *     every launch runs the argument checks of the direct call, so a launch
 *     returns exactly the status the direct call returns for these arguments.
 *   - A plan is not changed by a launch: it may be launched on any stream,
 *     from several host threads, and inside stream capture.
 *   - qg_plan_launch(NULL, ...) returns QG_ERR_INVALID_ARG;
 *     qg_plan_destroy frees the plan (NULL is a no-op); destroying a plan does
 *     not wait for its launches, which own nothing of it.
 */
typedef struct qg_plan qg_plan;
qg_status qg_plan_quantize_rowwise_int8(qg_plan **plan, const void *x, int64_t ldx, int8_t *xq, int64_t ldxq,
                                        float *x_scale, int64_t M, int64_t K);
qg_status qg_plan_gemm_w8a8(qg_plan **plan, const int8_t *xq, int64_t ldx, const int8_t *wq, int64_t ldw,
                            const float *x_scale, const float *w_scale, const float *bias, void *y,
                            int y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K, void *workspace,
                            size_t workspace_bytes, unsigned flags);
qg_status qg_plan_gemm_w8a16(qg_plan **plan, const void *x, int64_t ldx, const int8_t *wq, int64_t ldw,
                             const float *w_scale, const float *bias, void *y, int64_t ldy, int64_t M,
                             int64_t N, int64_t K, void *workspace, size_t workspace_bytes, unsigned flags);
qg_status qg_plan_gemm_w4a16(qg_plan **plan, const void *x, int64_t ldx, const int32_t *qweight,
                             const void *scale, const void *zero, int64_t group, const float *bias, void *y,
                             int64_t ldy, int64_t M, int64_t N, int64_t K, void *workspace,
                             size_t workspace_bytes, unsigned flags);
qg_status qg_plan_launch(const qg_plan *plan, qg_stream_t stream);
void qg_plan_destroy(qg_plan *plan);

#ifdef __cplusplus
}
#endif

#endif /* QG_H */
