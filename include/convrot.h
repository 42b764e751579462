/*
 * convrot.h -- C ABI of the B200 (sm_100a) W8A8 ConvRot expert-choice MoE library.
 *
 * What the calls compute (web pages, cited by title and section):
 *  - "Nucleus-Image INT8 Convrot Experts + FP8 Text Encoder", section
 *    "Quantization": every routed-expert matrix is rotated (ConvRot), then
 *    quantised to symmetric INT8 with nearest rounding and one FP32 scale per
 *    output row; rotation groups are 256 for gate/up and 64 for down;
 *    inference uses W8A8 ConvRot linears with BF16 outputs.
 *  - "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How they were
 *    made": int8 ConvRot = block Hadamard rotation, one scale per row, 8-bit
 *    activations.
 *  - "MLX Nucleus-Image", opening paragraph: 64 routed experts with
 *    expert-choice routing; table "Conversion notes": each expert picks its
 *    top-C tokens, outputs are scattered back; experts compute
 *    silu(gate) * up with gate in the first half.
 *
 * Readings fixed by this library where the pages are silent:
 *  - rotation: Sylvester Hadamard in natural order, normalised by 1/sqrt(g),
 *    applied to contiguous groups of g along K; g in {1, 4, 16, 64, 256};
 *  - quantiser (the definition): v' = v . blockdiag(H_g / sqrt(g)),
 *    s = fp32(max|v'| / 127), q = clamp(rne(v' / s), -127, 127), ties to
 *    even; all-zero codes when s is 0. The offline weight quantisers compute
 *    exactly this (fp64 rotation and quotients). The run-time activation and
 *    h quantisers rotate in fp32 and take q = rint(v'_32 * fp32(127 / a_32))
 *    (rows with absmax below 2^-100 divide by their scale instead): their
 *    codes can differ from the definition's by one where v'/s lies within the
 *    fp32 rounding error of a half-integer;
 *  - activations (and the SwiGLU output h) use per-row dynamic scales;
 *  - router score: per-token softmax over the experts (fp64, rounded to
 *    fp32); top-C ties go to the lower token index; each expert's tokens are
 *    listed in ascending order;
 *  - dequant y = fp32(acc) * (s_w * s_x); h = silu(g) * u in fp32; the down
 *    projection's output z is bf16 (a W8A8 linear with BF16 outputs); combine
 *    out32[t] += fp32(w * z) in fp32, one bf16 rounding at the end.
 *
 * Conventions for every call:
 *  - All buffers are owned by the caller; the library allocates nothing.
 *    Pointers marked "device" must be device memory of the current CUDA
 *    device and 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream). They return a status code and never throw or abort.
 *  - Arguments are checked before anything is launched; on any error nothing
 *    is launched. A kernel that gives up on a bounded device-side wait sets a
 *    flag that convrot_check_device_error() reports (CONVROT_ERR_TIMEOUT).
 *  - Layouts are row-major; "K-contiguous" means the last index is K.
 */
#ifndef CONVROT_H_
#define CONVROT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  CONVROT_OK = 0,
  CONVROT_ERR_INVALID_ARG = 1,        /* a size, group or pointer is not acceptable */
  CONVROT_ERR_UNSUPPORTED_DEVICE = 2, /* current device is not sm_100 / no device */
  CONVROT_ERR_WORKSPACE_TOO_SMALL = 3,
  CONVROT_ERR_MISALIGNED = 4,         /* a pointer is not 16-byte aligned */
  CONVROT_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
  CONVROT_ERR_TIMEOUT = 6             /* a device-side wait ran out (see check call) */
};

enum { CONVROT_DTYPE_BF16 = 0, CONVROT_DTYPE_F32 = 1 };

/* Storage of an int8 weight operand B:
 *  CONVROT_LAYOUT_ROWS   row-major [G, N, K] (K-contiguous);
 *  CONVROT_LAYOUT_TILES  the tiled weight format written by
 *      convrot_quantize_weights_tiled: every matrix is cut into 128-row blocks
 *      (the last one zero-padded), every block into 128-byte K tiles (the last
 *      one zero-padded); tile (block rb, k-tile kb) is 16 KB at byte offset
 *      (rb * ceil(K/128) + kb) * 16384 and holds 128 rows of 128 bytes. Blocks
 *      of consecutive matrices follow each other. Each GEMM K-step then reads
 *      whole 16 KB runs of DRAM. For a SwiGLU operand each group holds two
 *      matrices of F rows (gate, then up). */
enum { CONVROT_LAYOUT_ROWS = 0, CONVROT_LAYOUT_TILES = 1 };

/* Version of this ABI (incremented on incompatible changes). */
int convrot_abi_version(void);

/* Static description of a status code. Never NULL. */
const char* convrot_status_string(int status);

/* Name of the last CUDA error (cudaGetErrorName) an entry point saw on the
 * calling host thread, for a CONVROT_ERR_CUDA status; "none" before any. */
const char* convrot_last_cuda_error(void);

/* Checks that the current device is an sm_100 part the kernels were built for.
 * Returns CONVROT_OK or CONVROT_ERR_UNSUPPORTED_DEVICE. */
int convrot_device_check(void);

/* Synchronises `stream`, then reads and clears the device error word.
 * *flags (may be NULL) receives the raw bits. Returns CONVROT_ERR_TIMEOUT if a
 * bounded wait ran out since the last check, CONVROT_ERR_CUDA if the
 * synchronisation failed, else CONVROT_OK. */
int convrot_check_device_error(void* stream, unsigned* flags);

/* Diagnostic: launches one CTA that waits `limit_ns` on an mbarrier nothing
 * arrives on, through the same bounded wait the GEMM pipeline uses. It must
 * give up and record a flag; *result_dev (device int) receives 0 when it gave
 * up. Used to test the failure path without faulting the GPU. */
int convrot_wait_selftest(unsigned long long limit_ns, int* result_dev, void* stream);

/* Diagnostic: one thread clears the two ints at words_dev (a counter and an
 * abort word), then waits up to `limit_ns` for the counter to reach 1 through
 * the bounded cross-CTA wait the requantising GEMM uses between tiles;
 * nothing raises it, so the wait gives up, records a flag (reported by
 * convrot_check_device_error) and sets *result_dev (device int) to 0. */
int convrot_count_wait_selftest(unsigned long long limit_ns, int* words_dev, int* result_dev,
                                void* stream);

/* Host rule of the requantising SwiGLU GEMM (convrot_i8_gemm_swiglu_rq, and
 * the MoE call's gate/up step): how many co-resident CTAs (or CTA pairs) it
 * runs `tiles` tiles on, n_blocks tiles per row block, when `capacity` of
 * them fit on the device at once. The tiles of a row block wait for one
 * another, so the answer is `tiles` when they all fit, else a whole number
 * of row blocks, and 0 when not even one row block's tiles fit together: the
 * library then takes the two-step path (fp32 h, rotation kernel) instead of
 * launching a kernel whose waits could not end. Pure host arithmetic;
 * returns -1 for negative arguments. */
int64_t convrot_swiglu_rq_units(int64_t tiles, int64_t n_blocks, int64_t capacity);

/* ---------------------------------------------------------------------------
 * Rotate + quantise rows at run time (activations per token, and the SwiGLU
 * output h before the down projection). "Nucleus-Image INT8 Convrot Experts +
 * FP8 Text Encoder", section "Quantization". fp32 arithmetic (see the
 * quantiser note at the top): within one code of the definition.
 *   x      device, [rows, K] bf16 (x_dtype = CONVROT_DTYPE_BF16) or fp32
 *   rows   >= 0;  K: multiple of 16 and of `group`, 16 <= K <= 16384
 *   group  rotation group g in {1, 4, 16, 64, 256}
 *   q      device, [rows, K] int8 codes (K-contiguous)
 *   scale  device, [rows] fp32 per-row scales
 * rows == 0 launches nothing and returns CONVROT_OK.
 * ------------------------------------------------------------------------- */
int convrot_rotquant(const void* x, int x_dtype, int64_t rows, int64_t K, int group, int8_t* q,
                     float* scale, void* stream);

/* Offline weight quantisation of bf16 weight rows, exactly the definition:
 * fp64 rotation (exact sums of bf16 values while a group's exponent spread
 * stays under ~37 bits), s = fp32 of the fp64 quotient absmax / 127, codes
 * rne of correctly rounded fp64 quotients. Same sizes and arguments as
 * convrot_rotquant with bf16 input. A stack of expert matrices [E, N, K] is
 * passed as rows = E * N (the rotation is per row, so the 3-D packed layout
 * needs no other entry point). */
int convrot_quantize_weights(const void* w_bf16, int64_t rows, int64_t K, int group,
                             int8_t* w_q, float* row_scale, void* stream);

/* Offline weight quantisation into the tiled weight format (see
 * CONVROT_LAYOUT_TILES): n_mats matrices of `rows` x K bf16 rows, stored
 * back to back in w_bf16 ([n_mats * rows, K]). The codes and per-row scales
 * equal those of convrot_quantize_weights; only their placement differs.
 *   w_tiled    device, convrot_tiled_weight_bytes(n_mats, rows, K) bytes
 *              (padding is written as zero codes)
 *   row_scale  device, [n_mats * rows] fp32
 * A MoE gate/up stack [E, 2f, d] is n_mats = 2E matrices of f rows; a down
 * stack [E, d, f] is n_mats = E matrices of d rows. */
int64_t convrot_tiled_weight_bytes(int64_t n_mats, int64_t rows, int64_t K);
int convrot_quantize_weights_tiled(const void* w_bf16, int64_t n_mats, int64_t rows, int64_t K,
                                   int group, int8_t* w_tiled, float* row_scale, void* stream);

/* ---------------------------------------------------------------------------
 * Router softmax. "MLX Nucleus-Image", opening paragraph (expert-choice).
 *   logits  device, [T, E] bf16;  1 <= E <= 256
 *   s_t     device, [E, T] fp32: s_t[e, t] = softmax_e(logits[t, :]) (transposed)
 * ------------------------------------------------------------------------- */
int convrot_router_softmax(const void* logits_bf16, int64_t T, int E, float* s_t, void* stream);

/* ---------------------------------------------------------------------------
 * Expert-choice top-C. "MLX Nucleus-Image", table "Conversion notes".
 *   s_t   device, [E, T] fp32 scores (no NaN)
 *   C     0 <= C <= T
 *   idx   device, [E, C] int32: the C tokens with the largest score, ties to
 *         the lower token index, in ascending token order
 *   w     device, [E, C] fp32: w[e, c] = s_t[e, idx[e, c]] (a -0 score
 *         compares equal to +0 and comes back as +0)
 *   slot  device, [E, T] int32 or NULL: slot[e, t] = c where idx[e, c] = t,
 *         or -1 if expert e did not pick token t (the inverse of idx)
 * ------------------------------------------------------------------------- */
int convrot_topc(const float* s_t, int64_t T, int E, int64_t C, int32_t* idx, float* w,
                 int32_t* slot, void* stream);

/* Router-weighted combine. "MLX Nucleus-Image", table "Conversion notes" (the
 * experts' outputs are scattered back to their tokens), weighted by the
 * router scores of the choices:
 *   y[t, :] = bf16(sum over e = 0, 1, ..., E-1 with c = slot[e, t] >= 0 of
 *             fp32(s_t[e, t] * z[e * C + c, :])), every product rounded to
 *             fp32 and added in fp32 in that order; a token no expert picked
 *             gets 0.
 *   z     device, [E * C, d] bf16 expert outputs (down projection)
 *   s_t   device, [E, T] fp32 router scores, transposed (the weight of a pick
 *         is its score: convrot_router_softmax)
 *   slot  device, [E, T] int32 from convrot_topc;  y device, [T, d] bf16
 *   1 <= E <= 256, d % 8 == 0, d <= 8192. */
int convrot_combine_rows(const void* z_bf16, const float* s_t, const int32_t* slot, int E,
                         int64_t T, int64_t C, int64_t d, void* y_bf16, void* stream);

/* Gather rows: dst[r, :] = src[idx[r], :], s_dst[r] = s_src[idx[r]].
 *   src [n_src, K] int8, s_src [n_src] fp32, idx [n_rows] int32 (each in
 *   [0, n_src)), dst [n_rows, K] int8, s_dst [n_rows] fp32; K % 16 == 0. */
int convrot_gather_rows(const int8_t* src, const float* s_src, int64_t n_src, const int32_t* idx,
                        int64_t n_rows, int64_t K, int8_t* dst, float* s_dst, void* stream);

/* ---------------------------------------------------------------------------
 * Grouped INT8 GEMMs on the tcgen05 tensor cores (exact int32 accumulation).
 * For every group g: acc[g, m, n] = sum_k a[g, m, k] * b[g, n, k].
 *   a         device, [G, M, K] int8 (K-contiguous)
 *   b         device, int8 weights of G matrices of N rows, stored as
 *             b_layout says (CONVROT_LAYOUT_ROWS: [G, N, K]; TILES: the tiled
 *             weight format, G matrices, or 2G for the SwiGLU call)
 *   K % 16 == 0, 16 <= K;  N % 16 == 0;  G, M, N < 2^31
 * ------------------------------------------------------------------------- */

/* acc stored as int32 d [G, M, N]. */
int convrot_i8_gemm_i32(const int8_t* a, const int8_t* b, int b_layout, int64_t G, int64_t M,
                        int64_t N, int64_t K, int32_t* d, void* stream);

/* y[g, m, n] = bf16(fp32(acc) * (s_b[g, n] * s_a[g, m])); s_a [G, M], s_b [G, N]. */
int convrot_i8_gemm_bf16(const int8_t* a, const float* s_a, const int8_t* b, const float* s_b,
                         int b_layout, int64_t G, int64_t M, int64_t N, int64_t K, void* y_bf16,
                         void* stream);

/* SwiGLU epilogue: b = [G, 2F, K] with gate rows 0..F-1 and up rows F..2F-1,
 * s_b [G, 2F]. h[g, m, f] = silu(y[g, m, f]) * y[g, m, F + f] in fp32 with
 * y = fp32(acc) * (s_b * s_a); h device [G, M, F] fp32; F % 16 == 0. */
int convrot_i8_gemm_swiglu(const int8_t* a, const float* s_a, const int8_t* b, const float* s_b,
                           int b_layout, int64_t G, int64_t M, int64_t F, int64_t K, float* h,
                           void* stream);

/* SwiGLU followed by the rotation and requantisation of h, all in the GEMM's
 * epilogue, so h is never stored ("Nucleus-Image INT8 Convrot Experts + FP8
 * Text Encoder", section "Quantization": the down projection's input is
 * rotated in groups of 64 and quantised per row):
 *   h[g, m, :] as convrot_i8_gemm_swiglu computes it, then per row the same
 *   rotation (group g_h in {1, 4, 16, 64}, F % g_h == 0) and quantiser as
 *   convrot_rotquant: h_q device [G, M, F] int8 codes, s_h device [G, M] fp32.
 *   The results equal convrot_i8_gemm_swiglu followed by convrot_rotquant
 *   (CONVROT_DTYPE_F32, group g_h) bit for bit.
 *   sync    device scratch of at least convrot_swiglu_rq_sync_bytes(G, M)
 *           bytes (the rows' running maxima, the tiles' arrival counters, an
 *           abort word and a count of published tiles per group);
 *           the call clears it on `stream` before the GEMM, so calls sharing
 *           one scratch must be ordered on one stream.
 * The tiles of a row wait for one another (bounded; a wait that runs out sets
 * the device error flag and the call's results are invalid). Returns
 * CONVROT_ERR_INVALID_ARG when the device cannot keep enough of the GEMM's
 * CTAs resident at once for that (ceil(F / 128) of them, or CTA pairs for
 * M > 128); convrot_i8_gemm_swiglu + convrot_rotquant then do the same work. */
size_t convrot_swiglu_rq_sync_bytes(int64_t G, int64_t M);
int convrot_i8_gemm_swiglu_rq(const int8_t* a, const float* s_a, const int8_t* b,
                              const float* s_b, int b_layout, int64_t G, int64_t M, int64_t F,
                              int64_t K, int g_h, int8_t* h_q, float* s_h, void* sync,
                              size_t sync_bytes, void* stream);

/* Router-weighted scatter epilogue:
 * out32[idx[g, m], n] += w[g, m] * (fp32(acc) * (s_b[g, n] * s_a[g, m])).
 * out32 device [T, N] fp32 (accumulated with fp32 atomics, order not fixed);
 * idx [G, M] int32 in [0, T); w [G, M] fp32. */
int convrot_i8_gemm_scatter(const int8_t* a, const float* s_a, const int8_t* b, const float* s_b,
                            int b_layout, const int32_t* idx, const float* w, int64_t G, int64_t M,
                            int64_t N, int64_t K, float* out32, int64_t T, void* stream);

/* y = bf16(x) (nearest even), n elements, n % 4 == 0. */
int convrot_f32_to_bf16(const float* x, int64_t n, void* y_bf16, void* stream);

/* ---------------------------------------------------------------------------
 * W8A8 ConvRot linear. "Nucleus-Image INT8 Convrot Experts + FP8 Text
 * Encoder", section "Quantization" (W8A8 with BF16 outputs).
 *   x       device, [M, K] bf16 activations (rotated and quantised per token)
 *   w_q     device, [N, K] int8 rotated weight codes (convrot_quantize_weights)
 *   w_scale device, [N] fp32
 *   y       device, [M, N] bf16: bf16(fp32(acc) * (w_scale[n] * s_x[m]))
 *   workspace device, >= convrot_linear_workspace_size(M, K) bytes
 * ------------------------------------------------------------------------- */
size_t convrot_linear_workspace_size(int64_t M, int64_t K);
int w8a8_convrot_linear(const void* x_bf16, int64_t M, int64_t K, const int8_t* w_q,
                        const float* w_scale, int64_t N, int group, void* y_bf16, void* workspace,
                        size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * W8A8 ConvRot linear that allocates nothing and takes no workspace.
 * The pages have no counterpart to this call; it exists for callers that
 * cannot hand the library device memory for scratch: a host program that owns
 * only its input and output buffers and no device allocator, a serving loop
 * where cudaMalloc/cudaFree would synchronise the device and stall the other
 * streams, or a process whose device-memory budget is fixed at start-up.
 * Same arguments and result as w8a8_convrot_linear minus the workspace. The
 * activation codes and token scales go to one static device array of this
 * library (CONVROT_NOALLOC_MAX_CODES code bytes + CONVROT_NOALLOC_MAX_ROWS
 * fp32 scales, about 8.1 MiB), which every GPU that loads the library keeps
 * until the process exits.
 *  - Invalid sizes, groups or pointers are reported as by w8a8_convrot_linear
 *    first; then M * K > CONVROT_NOALLOC_MAX_CODES or
 *    M > CONVROT_NOALLOC_MAX_ROWS returns CONVROT_ERR_WORKSPACE_TOO_SMALL and
 *    launches nothing.
 *  - The array belongs to the current device: x and y must be memory of that
 *    device (or managed memory), else CONVROT_ERR_INVALID_ARG.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, no allocation) with that device current; make
 *    that first call before any stream capture.
 *  - All calls share the one array: calls that can overlap on the GPU
 *    (different streams, or host threads without ordering) race on it; order
 *    them on one stream. Nothing in the array needs to start at zero (every
 *    code and scale the GEMM reads is written by the same call first).
 * ------------------------------------------------------------------------- */
#define CONVROT_NOALLOC_MAX_CODES 8388608
#define CONVROT_NOALLOC_MAX_ROWS 16384
int w8a8_convrot_linear_noalloc(const void* x_bf16, int64_t M, int64_t K, const int8_t* w_q,
                                const float* w_scale, int64_t N, int group, void* y_bf16,
                                void* stream);

/* ---------------------------------------------------------------------------
 * Expert-choice W8A8 ConvRot MoE block (one call = the whole hot path).
 * "MLX Nucleus-Image", opening paragraph and table "Conversion notes";
 * "Nucleus-Image INT8 Convrot Experts + FP8 Text Encoder", "Quantization".
 *   x       device, [T, d] bf16;  logits device, [T, E] bf16
 *   w_gu    device, gate/up codes rotated with g_gu in the tiled weight format:
 *           2E matrices of f rows x d (expert e: gate = matrix 2e, up = 2e+1),
 *           convrot_tiled_weight_bytes(2E, f, d) bytes
 *   s_gu    device, [E, 2f] fp32 (gate rows then up rows per expert)
 *   w_d     device, down codes rotated with g_d in the tiled weight format:
 *           E matrices of d rows x f;  s_d device, [E, d] fp32
 *   C       tokens per expert, 0 <= C <= T
 *   y       device, [T, d] bf16 = bf16(sum over the experts that chose t, in
 *           ascending expert order, of w[e, c] * z_e), the sum in fp32, where
 *           z_e = bf16(down_e(requant(silu(gate_e) * up_e))) is the expert's
 *           BF16 output
 *   Sizes: d % 16 == 0, d % g_gu == 0, 16 <= d <= 8192; f % 16 == 0,
 *   f % g_d == 0, 16 <= f <= 8192; 1 <= E <= 256.
 * The workspace holds every intermediate; its layout is reported by
 * moe_workspace_layout so a caller can inspect each stage after the call.
 * With g_d <= 64 (and a device that keeps enough of the gate/up GEMM's CTAs
 * resident, as convrot_i8_gemm_swiglu_rq needs) h is rotated and requantised
 * in the gate/up GEMM's epilogue and the fp32 h region is left untouched;
 * with g_d = 256 h is stored in fp32 and rotated by a separate kernel.
 * Every kernel of the call runs on `stream` (so the call can be captured in a
 * CUDA graph on it); they are chained with programmatic dependent launch, and
 * the activation rotation runs beside the routing kernels. After the fused
 * requantisation the down projection is streamed per expert: its tiles for
 * expert e start once every gate/up tile of e has published its h codes (a
 * count in the hsync scratch), not after the whole gate/up GEMM.
 * Failure of a device-side wait: the call is asynchronous, so a kernel that
 * gives up on a bounded wait (the gate/up GEMM's cross-tile wait gives up
 * after 100 ms, e.g. when another workload holds some of the SMs and the
 * GEMM's CTAs cannot all be resident; the pipeline waits after 2 s) cannot
 * change the returned status. The kernels then stop early and y is invalid;
 * a caller that may share the device checks convrot_check_device_error(stream)
 * after the call (it synchronises) and treats CONVROT_ERR_TIMEOUT as a
 * failed call.
 * ------------------------------------------------------------------------- */
typedef struct {
  size_t x_q;      /* [T, d] int8     rotated activation codes      */
  size_t s_x;      /* [T] fp32        token scales                  */
  size_t s_t;      /* [E, T] fp32     router scores, transposed     */
  size_t idx;      /* [E, C] int32    chosen tokens                 */
  size_t w;        /* [E, C] fp32     router weights of the choices */
  size_t x_g;      /* [E, C, d] int8  gathered codes                */
  size_t s_g;      /* [E, C] fp32     gathered scales               */
  size_t h;        /* [E, C, f] fp32  silu(gate) * up (g_d = 256, and the
                      low-bit block)                                */
  size_t h_q;      /* [E, C, f] int8  rotated, requantised h        */
  size_t s_h;      /* [E, C] fp32     scales of h                   */
  size_t hsync;    /* convrot_swiglu_rq_sync_bytes(E, C) bytes: scratch of
                      the fused requantisation                      */
  size_t slot;     /* [E, T] int32    slot of each token per expert */
  size_t z;        /* [E, C, d] bf16  expert outputs (down projection) */
  size_t total;    /* bytes required                                */
} convrot_moe_layout_t;

int moe_workspace_layout(int64_t T, int64_t d, int64_t f, int E, int64_t C,
                         convrot_moe_layout_t* layout);
size_t moe_workspace_size(int64_t T, int64_t d, int64_t f, int E, int64_t C);
int moe_expert_choice_forward(const void* x_bf16, const void* logits_bf16, const int8_t* w_gu,
                              const float* s_gu, const int8_t* w_d, const float* s_d, int64_t T,
                              int64_t d, int64_t f, int E, int64_t C, int g_gu, int g_d,
                              void* y_bf16, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * W4A8 / W6A8 in the rotated basis.
 * "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How they were made":
 * 6-bit or 4-bit weights in the rotated basis with an FP8 scale per group of
 * 16, 8-bit activations. Readings fixed by this library:
 *  - the rotation is the int8 format's (same groups);
 *  - codes q in [-qmax, qmax], qmax = 7 (bits = 4) or 31 (bits = 6), nearest
 *    rounding, ties to even;
 *  - FP8 = E4M3 (bias 7, 3 mantissa bits, subnormals, largest value 448);
 *  - two scale levels per weight row v' (rotated, fp64): s_r = fp32(a /
 *    (qmax * 448)) with a = max|v'|; for each group j of 16 consecutive
 *    elements sigma_j = e4m3(a_j / (qmax * s_r)) (nearest, ties to the even
 *    code, saturating at 448); q = clamp(rne(v' / (s_r * sigma_j))); a zero
 *    row or a group with sigma 0 has zero codes. A weight decodes to
 *    s_r * sigma_j * q;
 *  - activations: per-token INT8 as in the int8 format; the linear is
 *    y = fp32(acc) * (s_x * s_r), acc = sum_k x_q * sigma * q.
 * The quantiser computes the definition exactly (fp64 rotation and
 * quotients). The GEMM accumulates acc in fp32 on the tensor cores (kind::f16
 * over exact fp16 operands), so acc differs from the exact sum by fp32
 * rounding only: |error| <= K * 2^-23 * sum_k |x_q * sigma * q|.
 *
 * Packed format of `rows` x K weights (rows % 128 == 0, K % 64 == 0),
 * convrot_lowbit_weight_bytes(rows, K, bits) bytes: tiles of 128 rows x 64
 * codes, tile (row block rb, k-block kb) at (rb * K/64 + kb) * T bytes with
 * T = 4608 (bits = 4) or 6656 (bits = 6), holding bits/2 planes of
 * [128 rows][16 bytes] (plane c = bytes 16c .. 16c+15 of each row's packed
 * codes) and then [128 rows][4 bytes] of E4M3 scales (the row's four groups
 * of the k-block, lowest group in the lowest byte). A row's packed codes
 * store u = q + 2^(bits-1): 32-bit words w_0 .. w_7 hold the low four bits,
 * code 8i+2j in bits 4j..4j+3 of w_i and code 8i+2j+1 in bits 16+4j..19+4j
 * (j = 0..3); for bits = 6 words w_8 .. w_11 hold the top two bits, code
 * 16i+2j in bits 2j..2j+1 of w_{8+i} and code 16i+2j+1 in bits 16+2j..17+2j
 * (j = 0..7). Row blocks of consecutive matrices follow each other.
 * ------------------------------------------------------------------------- */
/* Bytes of the packed format; -1 for bits not 4 / 6, rows % 128 or K % 64. */
int64_t convrot_lowbit_weight_bytes(int64_t rows, int64_t K, int bits);

/* Offline: rotate bf16 weight rows [rows, K] (device) with `group` and
 * quantise them to the b-bit format: w_packed (device) as above, row_scale
 * (device) [rows] fp32. 64 <= K <= 16384, K % group == 0. */
int convrot_quantize_weights_lowbit(const void* w_bf16, int64_t rows, int64_t K, int group,
                                    int bits, void* w_packed, float* row_scale, void* stream);

/* Grouped low-bit GEMM stage: for every group g,
 *   acc[g, m, n] = sum_k x_q[g, m, k] * sigma[g, n, k/16] * q[g, n, k]
 * with x_q (device) [G, M, K] int8, s_x (device) [G*M] fp32, w_packed
 * (device) G matrices of N rows in the packed format, row_scale (device)
 * [G*N] fp32. epilogue:
 *   CONVROT_LOWBIT_F32     out fp32 [G, M, N] = acc (s_x unused)
 *   CONVROT_LOWBIT_BF16    out bf16 [G, M, N] = bf16(acc * (s_x * s_r))
 *   CONVROT_LOWBIT_SWIGLU  out fp32 [G, M, N/2] = silu(y[:, f]) * y[:, N/2 + f]
 *                          with y = acc * (s_x * s_r) (gate rows first)
 * N % 256 == 0; 64 <= K <= 16384, K % 64 == 0. tile_tokens = tokens per
 * tile (a multiple of 16, at most 128), 0 = chosen by the library (for
 * M > 128 CTA pairs of 2 x 128 tokens that share each decoded weight). The
 * result does not depend on the choice beyond fp32 summation order. */
enum { CONVROT_LOWBIT_F32 = 0, CONVROT_LOWBIT_BF16 = 1, CONVROT_LOWBIT_SWIGLU = 2 };
int convrot_lowbit_gemm(const int8_t* x_q, const float* s_x, const void* w_packed,
                        const float* row_scale, int64_t G, int64_t M, int64_t N, int64_t K,
                        int bits, int epilogue, int tile_tokens, void* out, void* stream);

/* WbA8 ConvRot linear: x (device) [M, K] bf16 rotated with `group` and
 * quantised per token to INT8, then y (device) [M, N] bf16 =
 * bf16(acc * (s_x * s_r)) against b-bit weights. Workspace (device):
 * convrot_linear_workspace_size(M, K) bytes. N % 256 == 0, K % 64 == 0. */
int lowbit_convrot_linear(const void* x_bf16, int64_t M, int64_t K, const void* w_packed,
                          const float* row_scale, int64_t N, int group, int bits, void* y_bf16,
                          void* workspace, size_t ws_bytes, void* stream);

/* The expert-choice MoE block of moe_expert_choice_forward with b-bit expert
 * weights: w_gu (device) E matrices of 2f rows x d in the packed format (gate
 * rows then up rows per expert), s_gu [E, 2f]; w_d (device) E matrices of d
 * rows x f, s_d [E, d]. Routing, the activation and h quantisation and the
 * combine are the int8 block's; h goes through the workspace's fp32 region.
 * The workspace and its layout are moe_workspace_layout's. d % 256 == 0,
 * f % 128 == 0 (besides d % g_gu == 0, f % g_d == 0). Failure of a
 * device-side wait as for moe_expert_choice_forward. */
int moe_expert_choice_forward_lowbit(const void* x_bf16, const void* logits_bf16,
                                     const void* w_gu, const float* s_gu, const void* w_d,
                                     const float* s_d, int64_t T, int64_t d, int64_t f, int E,
                                     int64_t C, int g_gu, int g_d, int bits, void* y_bf16,
                                     void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H_ */
