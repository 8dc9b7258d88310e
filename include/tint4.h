/*
 * tint4.h -- C ABI of the packed-INT4 ConvRot quantized linear layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (page titles and sections it restates):
 *   "ComfyUI-INT-Crush", "Forward Pass": rotate the activations (Hadamard,
 *   rot_size), quantize weights and activations, run the GEMM;
 *   "Inference > INT4 > CUDA backend": INT4 -> INT8 unpack, INT8 GEMM with
 *   fused dequant, and for rot_size 256 a fused rotate + quantize + GEMM;
 *   "Inference > INT4 > Triton backend": dynamic activation quantization
 *   (W4A8) and the W4A16 path for rot_size 0; "Weight Format": INT4 weights
 *   are uint8 with two values per byte.
 *   "feat: packed int4 convrot model loading and dispatch" (stable-diffusion.cpp
 *   #2010), "Summary": packed nibbles stream to the backend unconverted with
 *   row scales beside them; the activation rotate+quantize is shared by every
 *   linear that reads the same input (convrot_w4a4 and W4A8 kinds).
 *   "TINT4 v1.2 -- torchao INT4 for ComfyUI", "v1.1 新特性 > 5": the W4A16
 *   layer keeps _qdata/_scale/_zp.
 *
 * Formats (readings of the pages, which do not fix them):
 *   bf16          raw bfloat16 bits (uint16_t), round-to-nearest-even.
 *   rotation      block Hadamard along K: each length-g block v of a row is
 *                 replaced by H_g v, H_g the Sylvester (natural-order)
 *                 Hadamard matrix / sqrt(g); g in {16, 64, 256}; 0 = none.
 *   packed int4   uint8 [rows, K/2] row-major; byte j of a row holds element
 *                 2j in its low nibble and 2j+1 in its high nibble, each a
 *                 4-bit two's complement code.  Symmetric codes use [-7, 7].
 *   scales        fp32, one per row of W (row_scale [N]) and one per token
 *                 (tok_scale [M]); scale = absmax / 7 (int4) or / 127 (int8),
 *                 code = clamp(round_half_even(v / scale)); an all-zero row
 *                 has scale 0 and codes 0.  The group-wise entry points
 *                 (below) take one weight scale per row and 128-wide K
 *                 group instead, optionally with zero points.
 *   output        y[m, n] = bf16( acc[m, n] * tok_scale[m] * row_scale[n]
 *                 (+ bias[n]) ), acc the exact int32 sum of code products.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers of the current CUDA device unless stated.
 *     The caller owns and allocates every buffer; the library never allocates
 *     device memory and keeps no pointer after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; outputs are valid once the
 *     stream reaches that point.
 *   - Argument and shape errors are returned synchronously, before anything
 *     is launched.  Nothing throws across the ABI.  Calls on different
 *     streams do not share mutable state except the device error word.
 *   - Shape rules: M >= 0, N >= 16 and N % 16 == 0, K >= 32 and K % 32 == 0,
 *     K % g == 0; K <= 16384 for the rotate/quantize calls.  Pointers must
 *     be 16-byte aligned.  Padding K up to the weight's width is the
 *     caller's job ("ComfyUI-INT-Crush", "Forward Pass" step 3).
 *   - Device-side waits are bounded (default 4 s, see
 *     tint4_set_wait_limit_ns); a wait that gives up records a code in the
 *     device error word, read by tint4_get_device_error.
 */
#ifndef TINT4_H
#define TINT4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TINT4_OK = 0,
    TINT4_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum value */
    TINT4_ERR_UNSUPPORTED_SHAPE = 2, /* a shape rule above is broken */
    TINT4_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
    TINT4_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed */
    TINT4_ERR_TIMEOUT = 5,           /* a bounded device-side wait gave up */
    TINT4_ERR_WORKSPACE = 6,         /* workspace missing or too small */
    TINT4_ERR_NO_DEVICE = 7          /* the current device is not sm_100 */
} tint4_status;

typedef uint16_t tint4_bf16;
/* IEEE binary16 bit patterns: the stored weight-scale format of
 * "ComfyUI-INT-Crush", "Weight Format". */
typedef uint16_t tint4_f16;

/* ABI version, bumped on any signature change. */
int tint4_abi_version(void);

/* Static description of a status code (never NULL). */
const char* tint4_status_string(tint4_status status);

/*
 * Offline weight preparation ("ComfyUI-INT-Crush", "Workflow" converter with
 * --rot-size / --int-bits 4 and "Weight Format"; TINT4, "量化方案" step 2).
 * W fp32 [N, K] -> each g-block along K rotated -> per-row symmetric int4
 * codes in [-7, 7], row_scale[n] = absmax_n / 7 -> w_packed uint8 [N, K/2].
 * group: 0 (no rotation), 16, 64 or 256.  Rotating W with the same block
 * rotation as the activations leaves x W^T unchanged.
 */
tint4_status tint4_pack_weights(const float* W, int N, int K, int group, uint8_t* w_packed,
                                float* row_scale, void* stream);

/*
 * Dynamic per-token activation rotate + quantize ("ComfyUI-INT-Crush",
 * "Forward Pass" steps 2 and 5; "Inference > INT4 > Triton backend").
 * x bf16 [M, K] -> rotate each g-block (fp32) -> tok_scale[m] = absmax_m / Q
 * -> codes.  bits 8: codes is int8 [M, K], Q = 127 (W4A8).  bits 4: codes is
 * packed uint8 [M, K/2], Q = 7 (W4A4).  One call can feed every linear that
 * reads the same input and group ("feat: packed int4 convrot ...", "Summary").
 */
tint4_status convrot_quantize_act(const tint4_bf16* x, int M, int K, int group, int bits,
                                  void* codes, float* tok_scale, void* stream);

/*
 * W4A8 GEMM with fused dequant ("ComfyUI-INT-Crush", "Inference > INT4 >
 * CUDA backend").  a int8 [M, K] activation codes, tok_scale fp32 [M],
 * w_packed uint8 [N, K/2], row_scale fp32 [N], bias bf16 [N] or NULL,
 * y bf16 [M, N].  int32 accumulation on the tensor cores.
 */
tint4_status w4a8_gemm(const int8_t* a, const float* tok_scale, const uint8_t* w_packed,
                       const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                       int N, int K, void* stream);

/*
 * W4A4 GEMM ("Load Diffusion Model INT4 (W4A4)", enable_convrot; stable-
 * diffusion.cpp "feat: packed int4 convrot ...", convrot_w4a4).  a_packed
 * uint8 [M, K/2] packed int4 activation codes; otherwise as w4a8_gemm.
 */
tint4_status w4a4_gemm(const uint8_t* a_packed, const float* tok_scale, const uint8_t* w_packed,
                       const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                       int N, int K, void* stream);

/*
 * w4a4_gemm with a caller workspace (at least convrot_linear_workspace_size(M,
 * K, 4) bytes, 256-byte aligned; its contents are scratch): above 16 tokens
 * the packed activation codes are widened once, to one int8 per code in the
 * workspace, and the int8 tensor-core GEMM runs on them, instead of being
 * widened in shared memory for every weight-row tile.  Same int32 sums and
 * the same output bits as w4a4_gemm; at most 16 tokens it is w4a4_gemm (the
 * workspace is unused and may be NULL).  Errors as w4a4_gemm, plus
 * TINT4_ERR_WORKSPACE.
 */
tint4_status w4a4_gemm_widened(const uint8_t* a_packed, const float* tok_scale,
                               const uint8_t* w_packed, const float* row_scale,
                               const tint4_bf16* bias, tint4_bf16* y, int M, int N, int K,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace the fused linears need (convrot_w4a8_linear: bits 8,
 * convrot_w4a4_linear: bits 4; the grouped, group-wise and W8A8 linears: bits
 * 8): the activation codes, one byte per code for both widths (M * K), plus
 * the token scales (4 * M), each rounded up to 256.  0 for invalid
 * arguments. */
size_t convrot_linear_workspace_size(int M, int K, int bits);

/* The W4A8 workspace size under the name of the boundary's specification:
 * convrot_linear_workspace_size(M, K, 8). */
size_t convrot_w4a8_linear_workspace(int M, int K);

/*
 * Fused ConvRot linear ("ComfyUI-INT-Crush", "Inference > INT4 > CUDA
 * backend": Hadamard rotation + activation quantization + INT8 GEMM as one
 * call; "Forward Pass" last note).  x bf16 [M, K] -> y bf16 [M, N].  The
 * codes pass through `workspace` (device memory of at least
 * convrot_linear_workspace_size(M, K, 8) bytes, 256-byte aligned, owned by
 * the caller; its contents are scratch).
 *   - M = 1 (K <= 4096): one launch that rotates and quantizes x inside the
 *     GEMM's CTAs.
 *   - otherwise: the rotate + quantize grid, then the GEMM grid (the
 *     streaming kernel up to 16 tokens, the tensor-core kernel above), back to
 *     back on `stream` with programmatic dependent launch.
 */
tint4_status convrot_w4a8_linear(const tint4_bf16* x, const uint8_t* w_packed,
                                 const float* row_scale, const tint4_bf16* bias, tint4_bf16* y,
                                 int M, int N, int K, int group, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* As convrot_w4a8_linear with int4 activation codes (W4A4): codes in
 * [-7, 7], scale absmax / 7.  Inside the call the codes are kept one per byte
 * and run through the W4A8 tensor-core kernel, whose int32 sums are the same
 * integers; the packed int4 format is the one convrot_quantize_act(bits 4)
 * and w4a4_gemm exchange. */
tint4_status convrot_w4a4_linear(const tint4_bf16* x, const uint8_t* w_packed,
                                 const float* row_scale, const tint4_bf16* bias, tint4_bf16* y,
                                 int M, int N, int K, int group, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * convrot_w4a8_linear without a caller-provided workspace, for callers that
 * cannot allocate device memory at the point of the call: code that runs
 * inside a fixed memory budget, a host program without a device allocator
 * of its own, or a plug-in whose host application owns every allocation.
 * (The pages have no counterpart: it is a packaging of the same layer.)
 * The workspace (activation codes and token scales) is one fixed 16 MiB
 * device array inside this library.  A GPU
 * reserves it when the library's device code is first loaded there (its
 * first kernel launch or its first call of this entry), whether or not this
 * entry is used, and holds it until the process exits.  Inputs and outputs
 * are as convrot_w4a8_linear; the caller still owns x, w_packed, row_scale,
 * bias and y.
 *   - Sizes: convrot_linear_workspace_size(M, K, 8) must fit in 16 MiB, else
 *     TINT4_ERR_WORKSPACE is returned and nothing is launched.
 *   - The first call on a device (and the first after the device's context
 *     has been rebuilt, e.g. by cudaDeviceReset) looks up the array's device
 *     address (cudaGetSymbolAddress); make that call before any stream
 *     capture.
 *   - No allocation: the call makes no cudaMalloc / cudaFree and calls no
 *     allocating routine.
 *   - Every call on a device shares the one array, and it keeps whatever the
 *     last call left in it (nothing in it needs to start at zero).  Calls
 *     whose work overlaps on the GPU (two streams, or two host threads) race
 *     on it and corrupt each other's results: serialize them.
 */
tint4_status convrot_w4a8_linear_noalloc(const tint4_bf16* x, const uint8_t* w_packed,
                                         const float* row_scale, const tint4_bf16* bias,
                                         tint4_bf16* y, int M, int N, int K, int group,
                                         void* stream);

/*
 * W8A8 ("ComfyUI-INT-Crush", "Inference > INT8": int8 weights times int8
 * activations with int32 accumulation; the rotation and per-row scales are
 * those of the int4 path).
 *   - tint4_quantize_weights_int8: W fp32 [N, K] -> rotated (group 0 / 16 /
 *     64 / 256 along K) -> w_int8 [N, K] codes in [-127, 127], row_scale fp32
 *     [N] = absmax / 127 (offline, like tint4_pack_weights; same rules).
 *   - w8a8_gemm: codes int8 [M, K] (convrot_quantize_act, bits 8), tok_scale
 *     fp32 [M], w_int8 [N, K], row_scale [N], bias bf16 [N] or NULL ->
 *     y bf16 [M, N] = bf16(acc * s_tok * s_row (+ bias)), acc exact int32.
 *     One tensor-core launch at every M (no streaming kernel for small M).
 *   - convrot_w8a8_linear: rotate + quantize x bf16 [M, K] into the workspace
 *     (convrot_linear_workspace_size(M, K, 8) bytes, 256-byte aligned), then
 *     w8a8_gemm.
 * Shape rules as w4a8_gemm / convrot_w4a8_linear (N % 16 == 0, K % 32 == 0,
 * K % group == 0); errors as there.
 */
tint4_status tint4_quantize_weights_int8(const float* W, int N, int K, int group,
                                         int8_t* w_int8, float* row_scale, void* stream);
tint4_status w8a8_gemm(const int8_t* codes, const float* tok_scale, const int8_t* w_int8,
                       const float* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                       int N, int K, void* stream);
tint4_status convrot_w8a8_linear(const tint4_bf16* x, const int8_t* w_int8,
                                 const float* row_scale, const tint4_bf16* bias, tint4_bf16* y,
                                 int M, int N, int K, int group, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * W8A8 with the row scales in the pages' stored INT8 format, fp16 [out, 1]
 * ("ComfyUI-INT-Crush", "Weight Format"): tint4_quantize_weights_int8_f16
 * rounds each row scale absmax / 127 to the nearest fp16 (ties to even) and
 * takes the codes against that stored value (a scale that rounds to 0 or to
 * infinity gives codes 0); the GEMM and the fused linear widen it exactly.
 * Otherwise as the fp32 forms above.
 */
tint4_status tint4_quantize_weights_int8_f16(const float* W, int N, int K, int group,
                                             int8_t* w_int8, tint4_f16* row_scale, void* stream);
tint4_status w8a8_gemm_f16(const int8_t* codes, const float* tok_scale, const int8_t* w_int8,
                           const tint4_f16* row_scale, const tint4_bf16* bias, tint4_bf16* y, int M,
                           int N, int K, void* stream);
tint4_status convrot_w8a8_linear_f16(const tint4_bf16* x, const int8_t* w_int8,
                                     const tint4_f16* row_scale, const tint4_bf16* bias,
                                     tint4_bf16* y, int M, int N, int K, int group, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * Group-wise W4A8 ("ComfyUI-INT-Crush", "Weight Format": INT4 weight scales
 * of shape [out, num_groups]; stable-diffusion.cpp "feat: packed int4
 * convrot model loading and dispatch", "Summary": the asymmetric W4A8 format
 * asym_w4a8_int8).  Weight groups are TINT4_WEIGHT_GROUP consecutive K
 * values of a row; ng = K / TINT4_WEIGHT_GROUP.
 *   - tint4_pack_weights_groupwise: W fp32 [N, K] -> rotated along K (group 0
 *     / 16 / 64 / 256, as tint4_pack_weights) -> per weight group
 *       asym == 0: w_scale = absmax / 7, codes clamp(rne(v / s), -7, 7) as
 *                  two's complement nibbles; w_zero unused (may be NULL);
 *       asym == 1: lo = min(0, min v), hi = max(0, max v), w_scale =
 *                  (hi - lo) / 15, w_zero = clamp(rne(-lo / s), 0, 15),
 *                  codes clamp(rne(v / s) + zero, 0, 15) as plain nibbles;
 *       an all-zero group: scale 0, zero 0, codes 0 (fp32, IEEE division).
 *     w_packed uint8 [N, K/2] (byte j: code 2j low nibble, 2j+1 high),
 *     w_scale fp32 [N, ng], w_zero uint8 [N, ng].
 *   - w4a8_gemm_groupwise: codes int8 [M, K] (convrot_quantize_act, bits 8),
 *     tok_scale fp32 [M], w_packed, w_scale, w_zero (NULL: symmetric codes;
 *     else asymmetric codes with these zero points), bias bf16 [N] or NULL ->
 *     y bf16 [M, N] = bf16(s_tok[m] * sum_j s[n, j] * p_j (+ bias[n])), p_j the
 *     exact integer sum over group j of a * (q - z); the sum over groups is
 *     evaluated in fp32 in group order (at M <= 16 with K <= 8192, one
 *     partial sum per warp of a streaming kernel, added in a fixed order).
 *     One launch: the streaming kernel at M <= 16 and K <= 8192, else the
 *     tensor-core GEMM.
 *   - convrot_w4a8_linear_groupwise: rotate + quantize x bf16 [M, K] into the
 *     workspace (convrot_linear_workspace_size(M, K, 8) bytes, 256-byte
 *     aligned; the codes there are in a private K order), then the GEMM.
 * Shape rules: those of w4a8_gemm (N % 16 == 0, 32 <= K <= 65536) plus
 * K % TINT4_WEIGHT_GROUP == 0 (and, for the packing and the fused linear,
 * K % group == 0, K <= 16384); all pointers 16-byte aligned.  Errors as
 * w4a8_gemm / convrot_w4a8_linear; asym outside {0, 1} is
 * TINT4_ERR_INVALID_ARG.  The caller owns every buffer.
 */
#define TINT4_WEIGHT_GROUP 128
tint4_status tint4_pack_weights_groupwise(const float* W, int N, int K, int group, int asym,
                                          uint8_t* w_packed, float* w_scale, uint8_t* w_zero,
                                          void* stream);
tint4_status w4a8_gemm_groupwise(const int8_t* a, const float* tok_scale,
                                 const uint8_t* w_packed, const float* w_scale,
                                 const uint8_t* w_zero, const tint4_bf16* bias, tint4_bf16* y,
                                 int M, int N, int K, void* stream);
tint4_status convrot_w4a8_linear_groupwise(const tint4_bf16* x, const uint8_t* w_packed,
                                           const float* w_scale, const uint8_t* w_zero,
                                           const tint4_bf16* bias, tint4_bf16* y, int M, int N,
                                           int K, int group, void* workspace,
                                           size_t workspace_bytes, void* stream);

/*
 * The same three calls with the scales in the pages' stored format: fp16
 * [out, num_groups] ("ComfyUI-INT-Crush", "Weight Format").  The packing
 * computes each group scale as above in fp32, rounds it to the nearest fp16
 * (ties to even; 65520 and above becomes infinity), and takes the zero point
 * and the codes against that stored value; a scale that rounds to 0 (or to
 * infinity) gives codes 0 (and zero point 0).  The GEMM and the fused linear
 * widen each fp16 scale exactly and otherwise compute as the fp32 forms.
 * Arguments, rules and errors as above.
 */
tint4_status tint4_pack_weights_groupwise_f16(const float* W, int N, int K, int group, int asym,
                                              uint8_t* w_packed, tint4_f16* w_scale,
                                              uint8_t* w_zero, void* stream);
tint4_status w4a8_gemm_groupwise_f16(const int8_t* a, const float* tok_scale,
                                     const uint8_t* w_packed, const tint4_f16* w_scale,
                                     const uint8_t* w_zero, const tint4_bf16* bias, tint4_bf16* y,
                                     int M, int N, int K, void* stream);
tint4_status convrot_w4a8_linear_groupwise_f16(const tint4_bf16* x, const uint8_t* w_packed,
                                               const tint4_f16* w_scale, const uint8_t* w_zero,
                                               const tint4_bf16* bias, tint4_bf16* y, int M, int N,
                                               int K, int group, void* workspace,
                                               size_t workspace_bytes, void* stream);

/*
 * Grouped GEMM: the same activation codes times up to TINT4_MAX_GROUPS
 * weight matrices in one launch ("feat: packed int4 convrot model loading
 * and dispatch", "Summary": the activation rotate + quantize is shared by the
 * linears of one input; separate Q, K and V projections, say).  For each
 * group g: y_g [M, N_g] = bf16(acc_g * s_tok * s_row_g (+ bias_g)), exactly
 * what w4a8_gemm gives for that group alone.
 *   - codes int8 [M, K], tok_scale fp32 [M] as for w4a8_gemm.
 *   - groups: a HOST array of num_groups entries, read during the call only;
 *     each entry holds device pointers (w_packed [N_g, K/2], row_scale [N_g],
 *     bias [N_g] or NULL, y [M, N_g]) and N_g.
 *   - 1 <= num_groups <= TINT4_MAX_GROUPS; every N_g obeys the w4a8_gemm
 *     rules (N_g % 16 == 0), K too; all pointers 16-byte aligned.
 *   - M <= 16 runs one small-M launch per group; above, one launch for all.
 * Errors: TINT4_ERR_INVALID_ARG (null groups or pointers, num_groups < 1),
 * TINT4_ERR_UNSUPPORTED_SHAPE (num_groups > TINT4_MAX_GROUPS, a bad N_g, M
 * or K), TINT4_ERR_MISALIGNED; nothing is launched then.
 */
#define TINT4_MAX_GROUPS 4
typedef struct {
    const uint8_t* w_packed;
    const float* row_scale;
    const tint4_bf16* bias;
    tint4_bf16* y;
    int N;
} tint4_weight_group;

tint4_status w4a8_gemm_grouped(const int8_t* codes, const float* tok_scale,
                               const tint4_weight_group* groups, int num_groups, int M, int K,
                               void* stream);

/*
 * convrot_w4a8_linear over a group of weight matrices: x bf16 [M, K] is
 * rotated (group `group`) and quantized to int8 once, into the workspace
 * (convrot_linear_workspace_size(M, K, 8) bytes, 256-byte aligned), then
 * w4a8_gemm_grouped runs.  Same rules and errors as convrot_w4a8_linear and
 * w4a8_gemm_grouped.
 */
tint4_status convrot_w4a8_linear_grouped(const tint4_bf16* x, const tint4_weight_group* groups,
                                         int num_groups, int M, int K, int group,
                                         void* workspace, size_t workspace_bytes,
                                         void* stream);

/*
 * W4A16 group-wise asymmetric linear ("TINT4 v1.2", "v1.1 新特性 > 5"
 * _qdata/_scale/_zp, "参数选择指南" group 128; "ComfyUI-INT-Crush",
 * "Inference > INT4 > Triton backend" W4A16).  x bf16 [M, K]; w_q uint8
 * [N, K/2] unsigned codes 0..15 packed low nibble first; scale bf16
 * [N, K/group]; zero uint8 [N, K/group] holding 0..15; y bf16 [M, N] with
 * y[m, n] = sum_k x[m, k] * (q[n, k] - zero[n, k/group]) * scale[n, k/group]
 * accumulated in fp32.
 *   - M <= 32 (decode): the weights are streamed once per 16 tokens (a batch
 *     of 17..32 tokens reads them twice) and each product uses
 *     (q - z) * s exactly; K <= 16384.
 *   - M > 32 (prefill): one tensor-core GEMM launch; every weight is first
 *     rounded to the bf16 number nearest to (q - z) * s (what a bf16
 *     dequantize-then-matmul uses), products accumulate in fp32; K <= 65536.
 * group must be 128; 1 <= M <= 65535 * 128; N % 16 == 0; K % 128 == 0; all
 * pointers 16-byte aligned.  Errors: TINT4_ERR_UNSUPPORTED_SHAPE for sizes
 * outside these limits, TINT4_ERR_MISALIGNED, TINT4_ERR_INVALID_ARG for null
 * pointers; nothing is launched then.
 */
tint4_status w4a16_gemv_gemm(const tint4_bf16* x, const uint8_t* w_q, const tint4_bf16* scale,
                             const uint8_t* zero, int group, tint4_bf16* y, int M, int N, int K,
                             void* stream);

/*
 * Test entry: the raw int32 accumulators acc[m, n] = sum_k qa[m, k] qw[n, k]
 * of the same tensor-core GEMM (act_bits 8: a is int8 [M, K]; act_bits 4: a
 * is packed uint8 [M, K/2]).  acc int32 [M, N].
 */
tint4_status tint4_debug_int32_gemm(const void* a, int act_bits, const uint8_t* w_packed,
                                    int32_t* acc, int M, int N, int K, void* stream);

/*
 * Test and timing entry: the GEMM launch the fused linears make for M > 16
 * ("ComfyUI-INT-Crush", "Inference > INT4 > CUDA backend": INT8 GEMM with
 * fused dequant), on int8 codes stored in the even/odd K order: within every
 * block of 8 codes along K, the codes of positions 0, 2, 4, 6, 1, 3, 5, 7.
 * Same arguments, rules and result as w4a8_gemm on the natural-order codes;
 * M must be > 16 (TINT4_ERR_UNSUPPORTED_SHAPE otherwise, nothing launched).
 */
tint4_status tint4_debug_w4a8_gemm_even_odd(const int8_t* a_even_odd, const float* tok_scale,
                                            const uint8_t* w_packed, const float* row_scale,
                                            const tint4_bf16* bias, tint4_bf16* y, int M, int N,
                                            int K, void* stream);

/*
 * Test entry for the bounded waits: launches one CTA that waits on a barrier
 * nobody arrives at, for at most limit_ns nanoseconds, then records
 * TINT4_ERR_TIMEOUT in the device error word and returns.  The context stays
 * usable.  limit_ns must be in [1e3, 1e10].
 */
tint4_status tint4_debug_bounded_wait(uint64_t limit_ns, void* stream);

/*
 * Synchronizes `stream`, then reads and clears the device error word of the
 * current device.  Returns TINT4_OK, TINT4_ERR_TIMEOUT (a bounded wait gave
 * up since the last read) or TINT4_ERR_CUDA.
 */
tint4_status tint4_get_device_error(void* stream);

/* Limit of every device-side wait for later launches, in nanoseconds
 * (default 4e9).  Values outside [1e3, 6e10] return TINT4_ERR_INVALID_ARG. */
tint4_status tint4_set_wait_limit_ns(uint64_t limit_ns);

/*
 * Decode-chain weight streaming (default off).  The small-M kernels
 * (w4a16_gemv_gemm; w4a8_gemm, w4a4_gemm and the fused linears at M <= 16)
 * are launched with programmatic dependent launch, so they may start while
 * the previous kernel of the stream is still running; they always wait for
 * it before reading the activations, and, with this switch off, before
 * reading anything.  With enable = 1 they start streaming their weight
 * operands (w_q / w_packed, scale, zero, row_scale) at once: in a chain of
 * layers the next layer's weights then flow from HBM while the current layer
 * finishes.  Turn it on only when no weight buffer of a call is written by
 * the kernel launched just before that call on the same stream (weights that
 * are set up once and then only read meet this).  Process-wide, affects later
 * launches; enable must be 0 or 1, else TINT4_ERR_INVALID_ARG.
 */
tint4_status tint4_set_decode_weight_prefetch(int enable);

#ifdef __cplusplus
}
#endif

#endif /* TINT4_H */
