/*
 * w4a8.h - C ABI of libw4a8.so, a B200 (sm_100a) implementation of the W4A8
 * per-output-channel quantized linear layer.
 *
 * The operation is the one the Keras guide "INT4 quantization in Keras"
 * describes in its section "How it works" (steps 1-6) and section "What Keras
 * does in INT4 mode":
 *   weights    - per-output-channel symmetric abs-max scale sw = 7 / max|W[:,n]|
 *                (1 for an all-zero column), codes q = clamp(rne(w * sw), -8, 7),
 *                packed two per byte along K, even k in the low nibble;
 *   activations- per-row dynamic abs-max INT8: sx = 127 / max|X[m,:]| (1 for an
 *                all-zero row), xq = clamp(rne(x * sx), -127, 127);
 *   product    - INT4 codes unpacked to INT8, INT8 x INT8 accumulated in INT32;
 *   output     - y = float(acc) / (sx * sw), then + bias[n], then ReLU if asked
 *                (the Dense epilogue of the guide's minimal model, section
 *                "Quantize a minimal functional model").
 * "rne" is round to nearest, ties to even; every float operation is IEEE
 * float32 round-to-nearest, so integer results are bit-exact and float32
 * outputs match a float32 statement of the same steps.
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller. The library
 *    never allocates, never frees and never synchronizes the stream; work is
 *    enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *    and the call returns once it is enqueued.
 *  - Strides ("ld") count elements of the array's type: floats for W, X, Y
 *    (f32), bf16 elements or int32 elements for Y in those formats, bytes for
 *    Wp and Xq.
 *  - Packed weights Wp and INT8 activations Xq must start on a 16-byte
 *    boundary and have a stride that is a multiple of 16 bytes.
 *  - Errors are returned as a w4a8_status; nothing is enqueued when an
 *    argument check fails. A CUDA launch failure returns W4A8_ERR_CUDA.
 *  - Kernels whose bounded wait on an asynchronous copy or tensor-core
 *    operation runs out record W4A8_ERR_TIMEOUT in a per-device status word
 *    instead of trapping, and return; read it with w4a8_get_device_status
 *    after synchronizing.
 */
#ifndef W4A8_H
#define W4A8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define W4A8_API __attribute__((visibility("default")))
#else
#define W4A8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int w4a8_status;

enum {
    W4A8_OK = 0,
    W4A8_ERR_INVALID_ARG = 1,  /* a null pointer, a bad size, stride or alignment */
    W4A8_ERR_UNSUPPORTED = 2,  /* no sm_100 device, or a path forced on a shape it cannot run */
    W4A8_ERR_WORKSPACE = 3,    /* workspace missing or smaller than w4a8_workspace_size() */
    W4A8_ERR_CUDA = 4,         /* a CUDA runtime call failed (e.g. a launch) */
    W4A8_ERR_TIMEOUT = 5       /* (device status) a bounded wait inside a kernel ran out */
};

/* Flags of w4a8_linear / w4a8_linear_q. */
#define W4A8_RELU          0x01u /* y = y > 0 ? y : +0 after the bias */
#define W4A8_OUT_F32       0x00u /* Y is float32 [M][ldy] (default) */
#define W4A8_OUT_BF16      0x02u /* Y is bfloat16 [M][ldy], rounded to nearest even */
#define W4A8_OUT_S32       0x04u /* Y is the raw INT32 accumulator [M][ldy]; no bias, no ReLU */
#define W4A8_OUT_MASK      0x06u
/* The caller guarantees that Wp, sw and bias hold their final values and that
 * no work still pending on the stream writes them (for example: the weights
 * were quantized when the layer was loaded and the stream has synchronized
 * since). The kernels may then read them before the previous kernel on the
 * stream has finished, overlapping the weight stream with its tail. Without
 * the flag they are read after it; the result is the same either way. */
#define W4A8_STATIC_WEIGHTS 0x08u
/* Kernel selection. AUTO picks by shape; the others force one kernel (tests). */
#define W4A8_PATH_AUTO     0x00u
#define W4A8_PATH_GENERIC  0x10u /* CUDA-core kernel, any shape */
#define W4A8_PATH_DECODE   0x20u /* weight-streaming kernel for few rows (M <= 16 per tile), picked by shape */
#define W4A8_PATH_TC       0x30u /* tcgen05 tensor-core GEMM (INT32 accumulators in TMEM); forced: the one-SM
                                    * k_gemm_tc. AUTO picks the CTA-pair k_gemm_tc_pair for INT4 layers of
                                    * M >= 1024, N >= 512, K <= 131072 and k_gemm_tc otherwise. */
/* One kernel of the decode family, forced (W4A8_ERR_UNSUPPORTED where it
 * cannot run the shape); w4a8_last_path reports them as W4A8_PATH_DECODE. */
#define W4A8_PATH_DECODE_RING  0x40u /* k_decode_ring: persistent TMA ring, M <= 8, K <= 131072 */
#define W4A8_PATH_DECODE_REGS  0x50u /* k_linear_decode: weights in registers, any M in tiles of 16 */
#define W4A8_PATH_DECODE_SPLIT 0x60u /* k_decode_split: cluster K-split, M <= 16, K <= 8192 */
/* Forced two-SM tensor-core GEMM (k_gemm_tc_pair: tcgen05.mma cta_group::2 on
 * a CTA pair, 256 channels x 192 tokens per tile), INT4 layers with
 * K <= 131072 only (else W4A8_ERR_UNSUPPORTED); w4a8_last_path reports it as
 * W4A8_PATH_TC. */
#define W4A8_PATH_TC_PAIR  0x70u
#define W4A8_PATH_MASK     0x70u

/* Largest K whose INT32 accumulator cannot overflow: 127 * 8 * K < 2^31. */
#define W4A8_MAX_K 2097152

/* Largest K for the W8A8 path: 127 * 127 * K < 2^31 keeps the INT32
 * accumulator exact for any codes. */
#define W8A8_MAX_K 133144

/* Bytes per packed output-channel row: ceil(K/2) rounded up to a multiple of
 * 16 (the stride every tensor-core tile load needs). Returns -1 if K < 1. */
W4A8_API int w4a8_packed_ld(int K);

/* Bytes per INT8 activation row used inside w4a8_linear: K rounded up to a
 * multiple of 16. Returns -1 if K < 1. */
W4A8_API int w4a8_act_ld(int K);

/* Workspace bytes w4a8_linear needs for M rows of K inputs (the INT8
 * activations and their scales). Returns 0 if M < 0 or K < 1. */
W4A8_API size_t w4a8_workspace_size(int M, int K);

/*
 * w4_quantize_pack - steps 1-2 of "How it works": per-output-channel abs-max
 * scale, half-even rounding to [-8, 7], two codes per byte.
 *   W   [K][ldw] float32, row k = input feature k, column n = output channel n
 *       (the Keras kernel layout), ldw >= N.
 *   Wp  [N][ldp] bytes out, ldp >= ceil(K/2) and a multiple of 16: byte j of
 *       row n = (q[n][2j] & 0xF) | (q[n][2j+1] & 0xF) << 4. Every byte past
 *       the nibble of k = K-1 (the odd-K pad nibble included) is written 0.
 *   sw  [N] float32 out: 7 / max_k |W[k][n]|, or 1 for an all-zero column.
 * Requires 1 <= K <= W4A8_MAX_K, N >= 1. Inputs must be finite.
 * Uses sw as scratch while it runs, so W and sw must not overlap.
 */
W4A8_API w4a8_status w4_quantize_pack(const float *W, int K, int N, int ldw,
                             uint8_t *Wp, int ldp, float *sw, void *stream);

/*
 * a8_quantize_rows - step 3: dynamic per-row abs-max INT8 quantization.
 *   X   [M][ldx] float32 (ldx >= K), finite.
 *   Xq  [M][ldq] int8 out (ldq >= K, multiple of 16); bytes K..ldq-1 of each
 *       row are written 0.
 *   sx  [M] float32 out: 127 / max_k |X[m][k]|, or 1 for an all-zero row.
 * M == 0 is a no-op returning W4A8_OK.
 */
W4A8_API w4a8_status a8_quantize_rows(const float *X, int M, int K, int ldx,
                             int8_t *Xq, int ldq, float *sx, void *stream);

/*
 * w4a8_linear - steps 3-6 on float32 activations: quantize each row of X to
 * INT8, multiply with the packed INT4 weights (unpacked to INT8 on chip),
 * accumulate in INT32, dequantize, add the bias, apply ReLU.
 *   X     [M][ldx] float32, ldx >= K.
 *   Wp,sw as produced by w4_quantize_pack for this K and N (pad nibbles 0).
 *   bias  [N] float32 or NULL.
 *   flags W4A8_RELU | one W4A8_OUT_* | W4A8_STATIC_WEIGHTS | one W4A8_PATH_*.
 *   Y     [M][ldy] out in the W4A8_OUT_* format, ldy >= N.
 *   workspace: device memory of at least w4a8_workspace_size(M, K) bytes,
 *       16-byte aligned; it holds the INT8 activations between kernels and
 *       must not be touched by the caller until the call's work completes.
 * M == 0 is a no-op returning W4A8_OK.
 */
W4A8_API w4a8_status w4a8_linear(const float *X, int M, int K, int ldx,
                        const uint8_t *Wp, int ldp, const float *sw, int N,
                        const float *bias, unsigned flags,
                        void *Y, int ldy,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * w4a8_linear_q - steps 4-6 on activations already quantized (by
 * a8_quantize_rows or an equivalent producer).
 *   Xq [M][ldq] int8 (ldq >= K, multiple of 16, 16-byte aligned), sx [M].
 *   Bytes of Xq past K in a row may hold anything: they always meet zero
 *   weight nibbles.
 * Other arguments as for w4a8_linear. No workspace is needed.
 */
W4A8_API w4a8_status w4a8_linear_q(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                          const uint8_t *Wp, int ldp, const float *sw, int N,
                          const float *bias, unsigned flags,
                          void *Y, int ldy, void *stream);

/*
 * w4a8_linear_noalloc - w4a8_linear for callers that cannot allocate device
 * memory: a host that hands this library only its input and output buffers
 * (a plugin or custom-op interface with no allocator of its own), or code
 * that must not call cudaMalloc because it can block or synchronize work
 * that is already running. It performs the same computation as w4a8_linear
 * (steps 3-6), but keeps the INT8 activations and their scales in scratch
 * memory the library owns: one static device array of
 * W4A8_NOALLOC_SCRATCH_BYTES bytes per GPU, which every GPU that loads the
 * library holds until the process exits. The pages (Keras INT4 guide) have
 * no counterpart of this entry point; it is an addition for such callers.
 *   Arguments as for w4a8_linear, without the workspace.
 *   Returns W4A8_ERR_WORKSPACE when w4a8_workspace_size(M, K) exceeds
 *   W4A8_NOALLOC_SCRATCH_BYTES (nothing is enqueued then).
 *   The first call on each device looks up the array's device address with
 *   that device current (the set-up is done once per device); make that first
 *   call before any stream capture on the device.
 *   Every call shares the one array: calls whose work can overlap on the GPU
 *   (different streams, or different host threads) race on it and corrupt
 *   each other's results; order them on one stream. Each call rewrites every
 *   byte it reads, so nothing left by an earlier call leaks into the result.
 */
#define W4A8_NOALLOC_SCRATCH_BYTES (16u << 20)
W4A8_API w4a8_status w4a8_linear_noalloc(const float *X, int M, int K, int ldx,
                                         const uint8_t *Wp, int ldp, const float *sw, int N,
                                         const float *bias, unsigned flags,
                                         void *Y, int ldy, void *stream);

/* The size in bytes of w4a8_linear_noalloc's scratch array as this library
 * was built (W4A8_NOALLOC_SCRATCH_BYTES), for callers that do not compile
 * against this header. */
W4A8_API size_t w4a8_noalloc_scratch_bytes(void);

/*
 * Layer chaining - one Dense layer feeding the next (the guide's minimal model,
 * section "Quantize a minimal functional model": each layer quantizes its own
 * float32 input dynamically, step 3 of "How it works"). The activation step
 * of a layer needs the abs-max of each of its input rows, which is a
 * reduction over the previous layer's whole output row. w4a8_linear_chain
 * lets the previous layer hand it over: with y_amax it also writes, for
 * every output row m and every 16 consecutive output channels p,
 *   y_amax[m][p] = max over n in [16 p, 16 p + 16) of |Y[m][n]|
 * (of the stored float32 outputs, after bias and ReLU), so that the next
 * layer's row abs-max is max_p y_amax[m][p] - exactly max_n |Y[m][n]| - and it
 * can quantize its rows inside its product kernel without a pass over them.
 * The pages have no API of their own for this; the results are those of
 * w4a8_linear bit for bit.
 */

/* Parts per output row of y_amax for N output channels: ceil(N / 16); -1 if N < 1. */
W4A8_API int w4a8_amax_parts(int N);

/*
 * w4a8_linear_chain - w4a8_linear with float32 output that takes and gives
 * per-row abs-max parts.
 *   X, Wp, sw, bias, Y, workspace: as for w4a8_linear; Y is float32.
 *   x_amax  [M][x_parts] float32 or NULL: parts whose max over a row equals
 *           max_k |X[m][k]| (such as the y_amax of the layer that wrote X);
 *           NULL: the call reduces the rows itself. A wrong x_amax gives
 *           wrong scales, not an error.
 *   y_amax  [M][w4a8_amax_parts(N)] float32 out, or NULL.
 *   flags   W4A8_RELU | W4A8_STATIC_WEIGHTS | one W4A8_PATH_*; any output
 *           format other than W4A8_OUT_F32 is W4A8_ERR_INVALID_ARG.
 * Launches: one on the generic and the cluster K-split decode kernels (the
 * activation step runs inside the product kernel); otherwise the activation
 * pass and the product, plus one pass over Y when y_amax is asked for.
 */
W4A8_API w4a8_status w4a8_linear_chain(const float *X, int M, int K, int ldx,
                                       const float *x_amax, int x_parts,
                                       const uint8_t *Wp, int ldp, const float *sw, int N,
                                       const float *bias, unsigned flags,
                                       float *Y, int ldy, float *y_amax,
                                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * w4a8_linear_grouped - many independent few-row linears (steps 3-6 each) in
 * as few launches as possible: one persistent launch per 64 problems. Meant
 * for batches of small layers whose separate launches would each pay the
 * dependency latency of a kernel: the projections of a model that do not
 * feed each other, or the experts of a mixture-of-experts layer at decode.
 * The pages have no counterpart; each problem's output holds the same bits as
 * w4a8_linear on that problem alone.
 *   probs[i]: X [M][ldx] float32 with 0 <= M <= 4 (M == 0: nothing to do),
 *       Wp [N][ldp] and sw [N] as from w4_quantize_pack, bias [N] or NULL,
 *       Y [M][ldy] in the W4A8_OUT_* format of `flags`; per-problem argument
 *       rules as for w4a8_linear. The array is read during the call only.
 *   flags: W4A8_RELU | one W4A8_OUT_* | W4A8_STATIC_WEIGHTS, for every problem.
 * Returns W4A8_ERR_UNSUPPORTED when a problem's INT8 rows do not fit a
 * block's shared memory (M x round_up(K, 4096) + 16 bytes beyond about
 * 68 KB); nothing is enqueued then. No workspace is needed.
 */
typedef struct w4a8_problem {
    const float *X;
    const uint8_t *Wp;
    const float *sw;
    const float *bias;
    void *Y;
    int M, K, ldx, ldp, N, ldy;
} w4a8_problem;

W4A8_API w4a8_status w4a8_linear_grouped(const w4a8_problem *probs, int count, unsigned flags, void *stream);

/*
 * W8A8 - the INT8 path that the guide's INT4 scheme extends ("How it works",
 * closing paragraph: the INT4 path is the INT8 path plus an unpack). Read as
 * the same steps with one 8-bit weight code per byte:
 *   weights - sw = 127 / max|W[:,n]| (1 for an all-zero column),
 *             q = clamp(rne(w * sw), -127, 127), rows of ldw8 bytes;
 *   activations, product and output - as for w4a8_linear (steps 3, 5, 6).
 * Kernels: decode for M <= 16, the tcgen05 GEMM otherwise (the weight tile
 * goes to the tensor cores as it is, no unpack), the generic kernel for tiny
 * problems; the W4A8_PATH_* flags force one as for the INT4 layer.
 */

/* Bytes per INT8 weight row: K rounded up to a multiple of 16 (-1 if K < 1). */
W4A8_API int w8a8_ld(int K);

/*
 * w8_quantize - W8A8 steps 1-2.
 *   W   [K][ldw] float32 (the Keras kernel layout), ldw >= N, finite.
 *   Wq  [N][ldw8] int8 out, ldw8 >= K and a multiple of 16, 16-byte aligned;
 *       bytes K..ldw8-1 of every row are written 0.
 *   sw  [N] float32 out: 127 / max_k |W[k][n]|, or 1 for an all-zero column.
 * Requires 1 <= K <= W8A8_MAX_K, N >= 1. Uses sw as scratch while it runs.
 */
W4A8_API w4a8_status w8_quantize(const float *W, int K, int N, int ldw,
                        int8_t *Wq, int ldw8, float *sw, void *stream);

/*
 * w8a8_linear - W8A8 steps 3, 5, 6 on float32 activations: quantize each row
 * of X to INT8 (into the workspace), multiply with the INT8 weights,
 * accumulate in INT32, dequantize, add the bias, apply ReLU. Arguments,
 * flags, workspace and errors as for w4a8_linear, with Wq/ldw8 as produced by
 * w8_quantize (bytes K..round_up(K,16)-1 of each row must be 0; bytes past
 * that are never read) and 1 <= K <= W8A8_MAX_K. Always two launches: the
 * activation pass, then the product.
 */
W4A8_API w4a8_status w8a8_linear(const float *X, int M, int K, int ldx,
                        const int8_t *Wq, int ldw8, const float *sw, int N,
                        const float *bias, unsigned flags,
                        void *Y, int ldy,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * w8a8_linear_q - steps 5-6 on INT8 activations Xq [M][ldq] (ldq >= K, a
 * multiple of 16, 16-byte aligned) with scales sx [M], natural k order.
 * Other arguments as for w8a8_linear; no workspace.
 */
W4A8_API w4a8_status w8a8_linear_q(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                          const int8_t *Wq, int ldw8, const float *sw, int N,
                          const float *bias, unsigned flags, void *Y, int ldy, void *stream);

/*
 * Zero-point INT4 - asymmetric per-output-channel weights (the uniform
 * asymmetric quantization of the "INT4" concept page, section 4.1, and the
 * formulas of the "4-bit Integer Quantization for LLMs" page, section "Weight
 * quantization"), with the activation step, product and epilogue of the W4A8
 * layer:
 *   sa[n] = 15 / (max_k W[k][n] - min_k W[k][n])  (1 when they are equal),
 *   zp[n] = -rne(min_k W[k][n] * sa[n]),  q = clamp(rne(w * sa[n]) + zp[n], 0, 15),
 *   acc = sum_k xq[m][k] * (q - zp[n]),  y = float(acc) / (sx[m] * sa[n]).
 * Storage: Wp as for w4_quantize_pack ([N][ldp] bytes, two nibbles per byte,
 * even k low) holding each code as the signed nibble q - 8 (q XOR 8), pad
 * nibbles 0; the W4A8 kernels multiply those and their epilogue adds
 * -(zp - 8) * sum_k xq[m][k]. Results are defined while acc fits INT32.
 */

/*
 * w4z_quantize_pack - steps 1-2 of the zero-point form.
 *   W  [K][ldw] float32 (the Keras kernel layout), ldw >= N, finite.
 *   Wp [N][ldp] bytes out (ldp >= ceil(K/2), a multiple of 16, 16-byte aligned).
 *   sa [N] float32 out, zp [N] int32 out (both used as scratch while it runs).
 * Requires 1 <= K <= W4A8_MAX_K, N >= 1.
 */
W4A8_API w4a8_status w4z_quantize_pack(const float *W, int K, int N, int ldw, uint8_t *Wp, int ldp,
                              float *sa, int32_t *zp, void *stream);

/* Workspace bytes of w4z_linear / w4z_linear_q for M rows, K inputs and N
 * outputs (INT8 rows, scales and row sums); 0 if M < 0, K < 1 or N < 1. */
W4A8_API size_t w4z_workspace_size(int M, int K, int N);

/*
 * w4z_linear - the zero-point layer on float32 activations: the activation
 * pass (which also writes the row sums), then the W4A8 product on the stored
 * codes with the zero-point correction in its epilogue (two launches).
 * Arguments, flags and errors as for w4a8_linear, with
 * sa/zp from w4z_quantize_pack in place of sw and a workspace of at least
 * w4z_workspace_size(M, K, N) bytes.
 */
W4A8_API w4a8_status w4z_linear(const float *X, int M, int K, int ldx,
                       const uint8_t *Wp, int ldp, const float *sa, const int32_t *zp, int N,
                       const float *bias, unsigned flags, void *Y, int ldy,
                       void *workspace, size_t workspace_bytes, void *stream);

/* w4z_linear_q - the same on INT8 activations Xq [M][ldq] with scales sx [M]
 * (two launches: the row sums, then the product; the workspace holds the
 * row sums). */
W4A8_API w4a8_status w4z_linear_q(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                         const uint8_t *Wp, int ldp, const float *sa, const int32_t *zp, int N,
                         const float *bias, unsigned flags, void *Y, int ldy,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * Group-wise INT4 - the zero-point rule above applied to every group of 128
 * consecutive k of each output channel ("INT4" concept page, section 4.2,
 * group quantization with group_size 128); sa and zp are [N][ng] with
 * ng = ceil(K / 128), the last group ragged. The output is
 *   y = sum_g float(acc_g) / (sx[m] * sa[n][g]),
 *   acc_g = sum_{k in g} xq[m][k] * (q - zp[n][g]) (exact INT32 partial sums),
 * summed in float32, then bias and ReLU. The kernel adds the group terms in
 * another order than a sequential loop, so outputs agree with that loop
 * within (2 ng + 2) * 2^-24 * sum_g |term_g| rather than bit for bit.
 * Storage: as for the zero-point form (nibbles q - 8, pad 0).
 * Output formats: W4A8_OUT_F32 or _BF16 (W4A8_OUT_S32 is rejected: there is no
 * single integer accumulator). Path: the decode-style kernel for any M
 * (W4A8_PATH_AUTO or _DECODE; other paths return W4A8_ERR_UNSUPPORTED).
 */

/* Groups per output channel for K inputs: ceil(K / 128); -1 if K < 1. */
W4A8_API int w4g_groups(int K);

/* w4g_quantize_pack - W [K][ldw] float32 -> Wp [N][ldp] (as w4z_quantize_pack),
 * sa [N][ng] float32, zp [N][ng] int32. Requires 1 <= K <= W4A8_MAX_K, N >= 1. */
W4A8_API w4a8_status w4g_quantize_pack(const float *W, int K, int N, int ldw, uint8_t *Wp, int ldp,
                              float *sa, int32_t *zp, void *stream);

/* w4g_linear - activation pass and the group-wise product (two launches);
 * arguments and workspace (w4a8_workspace_size(M, K)) as for w4a8_linear. */
W4A8_API w4a8_status w4g_linear(const float *X, int M, int K, int ldx,
                       const uint8_t *Wp, int ldp, const float *sa, const int32_t *zp, int N,
                       const float *bias, unsigned flags, void *Y, int ldy,
                       void *workspace, size_t workspace_bytes, void *stream);

/* w4g_linear_q - the group-wise product on INT8 activations (one launch). */
W4A8_API w4a8_status w4g_linear_q(const int8_t *Xq, int M, int K, int ldq, const float *sx,
                         const uint8_t *Wp, int ldp, const float *sa, const int32_t *zp, int N,
                         const float *bias, unsigned flags, void *Y, int ldy, void *stream);

/* Which kernel path (W4A8_PATH_GENERIC / _DECODE / _TC) the calling thread's
 * last successful w4a8_linear / w4a8_linear_q / w8a8_linear / w8a8_linear_q
 * call enqueued (grouped calls: _DECODE); 0 if none. */
W4A8_API unsigned w4a8_last_path(void);

/* How many kernels the calling thread's last successful w4a8_linear /
 * w4a8_linear_q / w4a8_linear_noalloc / w4a8_linear_chain call enqueued
 * (1 to 3; 0 if none, or if that call had M == 0). */
W4A8_API unsigned w4a8_last_launch_count(void);

/* Name of the product kernel that the calling thread's last successful
 * w4a8_linear / w4a8_linear_q / w4a8_linear_noalloc / w4a8_linear_chain /
 * w4a8_linear_grouped / w8a8_linear / w8a8_linear_q
 * call enqueued ("k_decode_split", "k_decode_ring", "k_linear_decode",
 * "k_gemm_tc", "k_linear_generic", "k_decode_grouped", or for the W8A8 calls
 * "k_linear8_decode", "k_linear8_generic", "k_gemm_tc"), not counting the activation
 * pass; "" if none, or if that call had nothing to do. A static string that
 * the caller must not free. */
W4A8_API const char *w4a8_last_kernel(void);

/*
 * w4a8_selftest_timeout - exercises the library's failure path without
 * faulting the GPU. Every wait inside the kernels is bounded: after about a
 * second of SM cycles it gives up, records W4A8_ERR_TIMEOUT in the device
 * status word (the first recorded fault is kept) and the kernel returns, so
 * the context stays usable. This call enqueues one tiny kernel whose single
 * wait can never be satisfied, with a limit of `cycles` SM cycles
 * (1000 <= cycles <= 2e9, else W4A8_ERR_INVALID_ARG); read the outcome with
 * w4a8_get_device_status. For tests of the error path; the pages have no
 * counterpart.
 */
W4A8_API w4a8_status w4a8_selftest_timeout(long long cycles, void *stream);

/* Read (and with clear != 0, reset) the current device's status word, which
 * kernels set on an internal fault. Synchronizes `stream` first. */
W4A8_API w4a8_status w4a8_get_device_status(int clear, void *stream);

/* A static, human-readable name for a status code. */
W4A8_API const char *w4a8_status_string(w4a8_status s);

#ifdef __cplusplus
}
#endif

#endif /* W4A8_H */
