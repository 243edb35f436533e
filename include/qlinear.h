/*
 * qlinear.h - C ABI of the B200 (sm_100a) NVFP4 / FP8-rowwise quantized linear.
 *
 * The operation (Diffusers documentation "BFL (fp8r / nvfp4)"):
 *   - scheme list, `nvfp4` entry: a quantized linear stores a packed E2M1
 *     `weight` (two values per byte), one E4M3 block scale per 16 elements
 *     (`weight_scale`), a global fp32 `weight_scale_2` and a calibrated fp32
 *     activation scale `input_scale`;
 *   - scheme list, `fp8r` entry: an E4M3 `weight` with one fp32 `weight_scale`
 *     per row; activations are quantized per row to E4M3 at run time;
 *   - section "Kernels", table: nvfp4 quantizes the activations at run time and
 *     runs a block-scaled FP4 GEMM; fp8r runs a GEMM with row-wise scales.
 * Element formats are the OCP ones: E4M3 "FN" (bias 7, max 448, no inf) and
 * E2M1 (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6).
 *
 * Arithmetic (the stated reading; the pages print no formula):
 *   NVFP4 quantize of a bf16 row with global scale g, per 16-element block:
 *     c = RN32(1 / RN32(6 g)) (once per tensor); s = E4M3(RN32(amax * c));
 *     d = RN32(decode(s) * g); codes = E2M1(RN32(x * RN32(1/d))), or 0 if d == 0.
 *     Element 2j in bits 3..0 of byte j, element 2j+1 in bits 7..4.
 *   NVFP4 linear: Y = bf16( input_scale * weight_scale_2 *
 *                          sum_k (E2M1(xq) E4M3(xs)) (E2M1(wq) E4M3(ws)) + bias ).
 *   fp8r quantize of a row: scale = RN32(amax / 448); codes = E4M3(RN32(x * RN32(1/scale))),
 *     or 0 if scale == 0.
 *   fp8r linear: Y = bf16( x_scale[m] * w_scale[n] * sum_k E4M3(xq) E4M3(wq) + bias ).
 *   E4M3 / E2M1 encoding: round to nearest, ties to even, saturating to the
 *   largest finite value, sign kept.
 *
 * Conventions for every entry point:
 *   - Tensors are row-major and densely packed (leading dimension = row length).
 *   - All tensor and scale pointers are DEVICE pointers (current device), except
 *     where a function says otherwise. Scalar scales are device pointers so that
 *     no host synchronisation is needed and calls can be captured in graphs.
 *   - Base pointers must be 16-byte aligned (QL_ERR_ALIGN otherwise).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls are
 *     asynchronous on it; nothing synchronises the host.
 *   - The caller owns every buffer, including workspaces. The library never
 *     allocates or frees device memory and keeps no per-call state.
 *   - Return value: QL_OK (0) or an error code below; errors found on the host
 *     leave all outputs untouched. QL_ERR_LAUNCH keeps the CUDA error text,
 *     readable through ql_last_error_message().
 *   - Only sm_100 devices (B200 class) are accepted (QL_ERR_DEVICE otherwise).
 *   - NaN or infinite inputs give unspecified codes (never a fault).
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ql_stream_t; /* a cudaStream_t */

enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1, /* null pointer, non-positive size */
  QL_ERR_SHAPE = 2,       /* size constraint violated (see each function) */
  QL_ERR_ALIGN = 3,       /* a base pointer is not 16-byte aligned */
  QL_ERR_DEVICE = 4,      /* current device is not sm_100 */
  QL_ERR_WORKSPACE = 5,   /* workspace missing or smaller than required */
  QL_ERR_LAUNCH = 6,      /* a CUDA call failed; see ql_last_error_message() */
  QL_ERR_TIMEOUT = 7      /* a kernel's bounded wait expired (device status word) */
};

/* ------------------------------------------------------------------------ */
/* NVFP4                                                                     */
/* ------------------------------------------------------------------------ */

/* Run-time NVFP4 quantization of activations ("BFL (fp8r / nvfp4)", "Kernels"
 * table: nvfp4_quantize for activations). The same routine quantizes a weight
 * offline when given weight_scale_2 as the global scale.
 *   x           bf16 [M, K]
 *   input_scale fp32 scalar (device): the calibrated global scale g
 *   xq          uint8 [M, K/2]  packed E2M1 codes (output)
 *   xs          uint8 [M, K/16] E4M3 block-scale codes (output)
 * Requires M >= 1, K >= 16, K % 16 == 0. */
int nvfp4_quantize_act(const void* x, int64_t M, int64_t K, const float* input_scale,
                       uint8_t* xq, uint8_t* xs, ql_stream_t stream);

/* nvfp4_linear_gemm plus a 16-bit low-rank branch (SVDQuant, "Background: SVDQuant
 * and Nunchaku": the low-rank up projection fused with the 4-bit compute kernel):
 *   Y = bf16( alpha * (sum_k NVFP4(x) NVFP4(w) + sum_j lr_act[m,j] * lr_up[n,j]) + bias )
 * with alpha = input_scale * weight_scale_2, i.e. lr_act is the low-rank branch's
 * activations D divided by alpha (so that alpha * lr_act = D), bf16 [M, rank]
 * row-major; lr_up bf16 [N, rank] row-major. The branch runs on the tensor cores
 * as one more K step (bf16 x bf16, fp32 accumulation) into the FP4 accumulator.
 * Requires 8 <= rank <= 64, rank % 8 == 0, 16-byte aligned lr_act / lr_up; the
 * workspace is the one nvfp4_linear_prologue filled. */
int nvfp4_linear_gemm_lowrank(int64_t M, int64_t K, const uint8_t* w, int64_t N,
                              const float* weight_scale_2, const float* input_scale,
                              const float* bias, const void* lr_act, const void* lr_up,
                              int64_t rank, void* y, const void* workspace,
                              size_t workspace_bytes, ql_stream_t stream);

/* SVDQuant-style NVFP4 linear (svdq_w4a4, NVFP4 variant, of the Diffusers page
 * "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers": activation outliers
 * moved into the weights, a 16-bit low-rank branch, the residual in 4 bits):
 *   xs = bf16(RN32(x * smooth))                 (per input column; smooth may be NULL)
 *   Y  = bf16( input_scale * weight_scale_2 * NVFP4(xs) NVFP4(w)^T
 *              + (xs lora_down^T) lora_up^T + bias )
 *   x          bf16 [M, K]
 *   smooth     fp32 [K] multipliers, or NULL (xs = x)
 *   lora_down  bf16 [rank, K]; lora_up bf16 [N, rank]; 8 <= rank <= 64, rank % 8 == 0
 *   w, w_scale, weight_scale_2, bias, y  as nvfp4_linear (w: the 4-bit residual)
 *   input_scale  the calibrated global scale of xs
 *   workspace  >= svdq_nvfp4_linear_workspace_size(M, K, N, rank) bytes
 * Two launches: a prologue that reads x once (smoothing, quantization of xs, the
 * low-rank down projection on warp-level bf16 tensor-core MMAs into the workspace,
 * weight-scale layout: the fusion the page describes for the down projection); the
 * 4-bit GEMM with the low-rank up projection as one more bf16 K step into the same
 * accumulator (the fusion the page describes for the up projection).
 * Requires the nvfp4_linear shapes and 16-byte aligned pointers. */
size_t svdq_nvfp4_linear_workspace_size(int64_t M, int64_t K, int64_t N, int64_t rank);
int svdq_nvfp4_linear(const void* x, int64_t M, int64_t K, const float* smooth,
                      const void* lora_down, const void* lora_up, int64_t rank, const uint8_t* w,
                      const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                      const float* input_scale, const float* bias, void* y, void* workspace,
                      size_t workspace_bytes, ql_stream_t stream);

/* W4A16 linear: 4-bit weights, 16-bit activations (the awq_w4a16 kernel family of
 * the Diffusers page "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers",
 * section "Introducing Nunchaku Lite", used there for the memory-bound adaptive
 * normalization and modulation projections), with the nvfp4 weight of this
 * library. The weight is dequantized to the compute dtype and the activations are
 * not quantized (the unfused path of "BFL (fp8r / nvfp4)", section "Kernels"):
 *   what[n, k] = bf16( RN32( E2M1(w[n, k]) * E4M3(w_scale[n, k/16]) * weight_scale_2 ) )
 *   Y[m, n]    = bf16( sum_k x[m, k] * what[n, k] + bias[n] )   (fp32 accumulation)
 *   x               bf16 [M, K] (a few rows: one per conditioning vector)
 *   w, w_scale      as nvfp4_linear: uint8 [N, K/2] packed E2M1, uint8 [N, K/16] E4M3
 *   weight_scale_2  device fp32 scalar
 *   bias            fp32 [N] or NULL
 *   y               bf16 [M, N] (output)
 * One launch, no workspace: the weight streams once from HBM for up to 8 rows of x
 * (made for M <= 8); larger M runs passes of 16 rows, each reading the weight again.
 * Requires K >= 32, K % 32 == 0; x, w, y 16-byte aligned, w_scale 2-byte aligned. */
int w4a16_linear(const void* x, int64_t M, int64_t K, const uint8_t* w,
                 const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                 const float* bias, void* y, ql_stream_t stream);

/* The MLP up projection with its GELU and the down projection's quantization
 * fused into the GEMM epilogue (the "fused GELU/MLP" kernels of the Diffusers
 * page "Nunchaku" section, for the nvfp4 scheme): instead of Y it writes
 *   H = NVFP4( bf16( GELU( bf16(input_scale * weight_scale_2 * X W^T + bias) ) ) )
 * with GELU(v) = v * Phi(v) (exact, erfc form, fp32) and the same 16-element block
 * rule as nvfp4_quantize_act, under the given global scale next_input_scale (the
 * down projection's calibrated input_scale). H goes straight into the activation
 * part of the down projection's workspace (a buffer of at least
 * nvfp4_linear_workspace_size(M, N, N_down) bytes): the next call is
 * nvfp4_linear_quantized_input on that workspace. X, W, scales and bias as
 * nvfp4_linear; `workspace` is this layer's own nvfp4_linear workspace.
 * Requires N % 256 == 0 (the next layer's K). Two launches (prologue, GEMM). */
int nvfp4_linear_gelu_quantize(const void* x, int64_t M, int64_t K, const uint8_t* w,
                               const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                               const float* input_scale, const float* bias,
                               const float* next_input_scale, void* next_workspace,
                               size_t next_workspace_bytes, void* workspace,
                               size_t workspace_bytes, ql_stream_t stream);

/* nvfp4_linear whose activations are already quantized in `workspace` (by
 * nvfp4_linear_gelu_quantize of the previous layer, with input_scale as its
 * next_input_scale): lays out this layer's weight scales, then runs the GEMM.
 * Arguments as nvfp4_linear_gemm plus w_scale (row-major [N, K/16]). */
int nvfp4_linear_quantized_input(int64_t M, int64_t K, const uint8_t* w, const uint8_t* w_scale,
                                 int64_t N, const float* weight_scale_2,
                                 const float* input_scale, const float* bias, void* y,
                                 void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* Bytes of workspace nvfp4_linear needs for this problem size (0 on bad sizes). */
size_t nvfp4_linear_workspace_size(int64_t M, int64_t K, int64_t N);

/* Weight block scales laid out once, for weights that do not change between calls
 * (a load-time step, like the weight's own quantization; FlashInfer's mm_fp4, the
 * kernel the pages name, is likewise handed its weight block scales already in its
 * own layout). The tensor-core layout of
 * the scales depends on the GEMM's tile width bn (tiles of 224 rows do not align
 * with the 128-row scale atoms), so the atoms are made for one bn:
 *   nvfp4_weight_scale_atoms_size(N, K, bn)  bytes of the atoms (0 on bad sizes or
 *                                           a bn outside {128, 192, 224, 256})
 *   nvfp4_layout_weight_scales(w_scale, N, K, bn, atoms, atoms_bytes, stream)
 *     w_scale uint8 [N, K/16] E4M3 row-major (as for nvfp4_linear); atoms: the caller's
 *     device buffer (16-byte aligned), written on `stream`.
 * ql_tile_config(1, M, N, K, ...) gives the bn nvfp4_linear itself would use for M. */
size_t nvfp4_weight_scale_atoms_size(int64_t N, int64_t K, int bn);
int nvfp4_layout_weight_scales(const uint8_t* w_scale, int64_t N, int64_t K, int bn,
                               uint8_t* atoms, size_t atoms_bytes, ql_stream_t stream);

/* nvfp4_linear on weight scales laid out by nvfp4_layout_weight_scales for tiles of
 * bn rows: the prologue quantizes only the activations, and the GEMM runs at tile
 * width bn (CTA pairs from M >= 512) reading the given atoms. Arguments as
 * nvfp4_linear, with w_scale_atoms / bn instead of w_scale; the same workspace size.
 * The result is bit for bit that of nvfp4_linear at the same tile width.
 * Errors as nvfp4_linear; QL_ERR_SHAPE for a bn outside {128, 192, 224, 256}. */
int nvfp4_linear_laid_out(const void* x, int64_t M, int64_t K, const uint8_t* w,
                          const uint8_t* w_scale_atoms, int bn, int64_t N,
                          const float* weight_scale_2, const float* input_scale,
                          const float* bias, void* y, void* workspace, size_t workspace_bytes,
                          ql_stream_t stream);

/* NVFP4 W4A4 linear forward: quantizes x at run time with input_scale and
 * contracts it on the tensor cores against the pre-quantized weight.
 * Two launches on `stream`: nvfp4_linear_prologue, then nvfp4_linear_gemm
 * (started early through programmatic dependent launch). The prologue is itself
 * launched as a programmatic dependent of whatever precedes it on `stream`, and
 * waits for that kernel to complete before it reads or writes memory. For M <= 64
 * (the skinny kernels) the GEMM lets the next kernel on `stream` start early: a
 * kernel the caller launches next with the programmatic-stream-serialization
 * attribute must wait for its prerequisite grid (griddepcontrol.wait /
 * cudaGridDependencySynchronize) before it reads y. Kernels launched without that
 * attribute are ordered as usual.
 *   x              bf16 [M, K]
 *   w              uint8 [N, K/2]  packed E2M1 weight codes
 *   w_scale        uint8 [N, K/16] E4M3 weight block scales (row-major, as stored
 *                  in the checkpoint; any hardware layout is produced internally)
 *   weight_scale_2 fp32 scalar (device)
 *   input_scale    fp32 scalar (device)
 *   bias           fp32 [N] or NULL
 *   y              bf16 [M, N] (output)
 *   workspace      device buffer of >= nvfp4_linear_workspace_size(M, K, N) bytes;
 *                  holds the quantized activations and the scale layouts between
 *                  the two kernels of one call (its contents are internal)
 *                  Calls that overlap on the GPU must not share a workspace.
 * Requires M, N >= 1, K >= 32, K % 32 == 0 (16-byte aligned packed rows). */
int nvfp4_linear(const void* x, int64_t M, int64_t K,
                 const uint8_t* w, const uint8_t* w_scale, int64_t N,
                 const float* weight_scale_2, const float* input_scale,
                 const float* bias, void* y,
                 void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* The same NVFP4 linear as ONE kernel launch (the "GEMM-prologue fusion" of the
 * activation quantization): every warp of the GEMM's persistent grid first
 * quantizes its share of x (codes and scales into the workspace, which stays in
 * L2) and lays out the weight scales, the CTAs meet at a grid-wide barrier, then
 * the same GEMM as nvfp4_linear_gemm runs. Gives the same bits as nvfp4_linear.
 * Measured slower than nvfp4_linear on B200 for the diffusion-transformer layers:
 * the quantization gets the GEMM's one CTA of 8 warps per SM instead of a full
 * grid of its own.
 *   arguments as nvfp4_linear; workspace of nvfp4_linear_workspace_size bytes,
 *   which need not be cleared: the barrier's words in it carry a per-call tag,
 *   and every call leaves them zero. Calls that overlap on the GPU must not share
 *   a workspace.
 * Requires K % 256 == 0 (QL_ERR_SHAPE otherwise) and a 16-byte aligned w_scale.
 * The barrier's wait is bounded: if some CTA of the grid cannot start (e.g. on a
 * partitioned GPU) the call ends with QL_ERR_TIMEOUT in the device status word. */
int nvfp4_linear_single_launch(const void* x, int64_t M, int64_t K, const uint8_t* w,
                               const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                               const float* input_scale, const float* bias, void* y,
                               void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* The two halves of nvfp4_linear, for callers that time or schedule them apart.
 * nvfp4_linear == nvfp4_linear_prologue followed by nvfp4_linear_gemm on the same
 * stream and workspace. The prologue quantizes x into the workspace and lays out
 * both scale tensors for the tensor cores; the GEMM reads only the workspace,
 * w, the scalars and bias. Same argument meaning and requirements as above. */
int nvfp4_linear_prologue(const void* x, int64_t M, int64_t K,
                          const uint8_t* w_scale, int64_t N, const float* input_scale,
                          void* workspace, size_t workspace_bytes, ql_stream_t stream);
int nvfp4_linear_gemm(int64_t M, int64_t K, const uint8_t* w, int64_t N,
                      const float* weight_scale_2, const float* input_scale,
                      const float* bias, void* y,
                      const void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* Offsets (bytes from the workspace base) of the quantized activations inside an
 * nvfp4_linear workspace, for diagnostics: codes are row-major uint8 [M, K/2] at
 * *codes_offset. Returns QL_OK or QL_ERR_SHAPE. */
int nvfp4_linear_workspace_layout(int64_t M, int64_t K, int64_t N, size_t* codes_offset,
                                  size_t* act_scales_offset, size_t* weight_scales_offset);

/* Calibration rule used by the workloads: out = RN32(amax(|x|) / (6 * 448)),
 * the global scale that maps the largest magnitude onto E2M1 6 times E4M3 448.
 *   x bf16 [n]; out fp32 scalar (device, overwritten). Requires n >= 1. */
int nvfp4_global_scale(const void* x, int64_t n, float* out, ql_stream_t stream);

/* nvfp4_linear without a caller workspace. No counterpart in the BFL page; it is
 * for callers that cannot allocate device memory themselves: a plugin whose host
 * application owns all device memory and forbids allocations on its hot path, a
 * serving loop that must never enter the allocator (an allocation can synchronise
 * the device or fail under memory pressure), or a C caller with no memory manager.
 * Same arguments and results as nvfp4_linear, minus the workspace: the scratch
 * lives in one fixed 32 MiB array in device memory inside this library, held by
 * every GPU that loads it until the process exits. Problems that need more
 * scratch than that (nvfp4_linear_workspace_size(M, K, N) > 32 MiB) are rejected
 * with QL_ERR_WORKSPACE and a message in ql_last_error_message(). The call
 * allocates and frees nothing. The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) and keeps it; make that first
 * call before any stream capture. All calls on a device share the array and each
 * rewrites what it reads, so nothing needs clearing between calls, but calls whose
 * kernels overlap on the GPU (unordered streams) race on it. */
int nvfp4_linear_noalloc(const void* x, int64_t M, int64_t K,
                         const uint8_t* w, const uint8_t* w_scale, int64_t N,
                         const float* weight_scale_2, const float* input_scale,
                         const float* bias, void* y, ql_stream_t stream);

/* ------------------------------------------------------------------------ */
/* INT4 W4A4                                                                 */
/* ------------------------------------------------------------------------ */

/* INT4 quantization of rows: the INT4 variant of the 4-bit layer of the Diffusers
 * page "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers" (section
 * "Introducing Nunchaku Lite": svdq_w4a4, "available in INT4 and NVFP4 variants").
 * The page gives no format; this library's reading, per 64-element group along K:
 *   scale = RN32(amax / 7); codes = clamp(round-half-even(RN32(x * RN32(1/scale))),
 *   -8, 7); all codes 0 when scale == 0.
 *   x      bf16 [M, K]
 *   q      uint8 [M, K/2] signed 4-bit codes, element 2j in bits 3..0 of byte j
 *   scale  fp32 [M, K/64] row-major group scales
 * Used for activations (rows = tokens) and weights (rows = output channels).
 * Requires K >= 64, K % 64 == 0; x and q 16-byte aligned. */
int int4_quantize_rows(const void* x, int64_t M, int64_t K, uint8_t* q, float* scale,
                       ql_stream_t stream);

/* Bytes of workspace int4_linear needs (0 on bad sizes): the quantized rows of x
 * (codes, then scales, each part 1 KB aligned) followed by the workspace of
 * int4_linear_gemm. */
size_t int4_linear_workspace_size(int64_t M, int64_t K, int64_t N);

/* INT4 W4A4 linear forward (no low-rank branch):
 *   Y[m, n] = bf16( sum_g x_scale[m,g] w_scale[n,g] sum_{k in g} qx[m,k] qw[n,k] + bias[n] )
 * quantizing x at run time (int4_quantize_rows into the workspace), then
 * int4_linear_gemm. Per-group fp32 scales have no block-scaled tcgen05 form, so the
 * GEMM moves them into the operands: both INT4 operands are dequantized to f16 with
 * one power-of-two factor per row, RN16(RN32(q * s * 2^-e)), and one f16 tensor-core
 * GEMM (fp32 accumulation) applies the factors in its epilogue. Each product is
 * within 2^-10 of its exact value, so |Y - exact| <= 2^-10 * sum |x w| plus the fp32
 * accumulation's rounding (the INT4 codes and scales themselves are exact).
 *   x        bf16 [M, K]
 *   w        uint8 [N, K/2] INT4 weight codes (as int4_quantize_rows writes them)
 *   w_scale  fp32 [N, K/64] group scales
 *   bias     fp32 [N] or NULL;  y  bf16 [M, N] (output)
 *   workspace >= int4_linear_workspace_size(M, K, N) bytes, 16-byte aligned
 * Requires K >= 64, K % 64 == 0; x, w 16-byte aligned. Four launches (quantize,
 * two dequantizations, GEMM). */
int int4_linear(const void* x, int64_t M, int64_t K, const uint8_t* w, const float* w_scale,
                int64_t N, const float* bias, void* y, void* workspace, size_t workspace_bytes,
                ql_stream_t stream);

/* Bytes of workspace int4_linear_gemm needs (0 on bad sizes): f16 copies of both
 * operands and their row factors, 2 * (M + N) * K + 4 * (M + N) bytes plus alignment. */
size_t int4_linear_gemm_workspace_size(int64_t M, int64_t K, int64_t N);

/* The GEMM half of int4_linear, from activations quantized by int4_quantize_rows:
 * xq uint8 [M, K/2], x_scale fp32 [M, K/64]; w, w_scale, bias and y as for int4_linear;
 * workspace >= int4_linear_gemm_workspace_size(M, K, N) bytes, 16-byte aligned, for
 * the f16 operands (owned by the caller, overwritten).
 * Requires K >= 64, K % 64 == 0; xq and w 16-byte aligned, the scales and bias 4-byte,
 * y 2-byte aligned (a 16-byte-aligned y with N % 8 == 0 takes TMA stores).
 * Errors: QL_ERR_INVALID_ARG (null pointer, size <= 0), QL_ERR_SHAPE, QL_ERR_ALIGN,
 * QL_ERR_WORKSPACE, QL_ERR_DEVICE, QL_ERR_LAUNCH. Every wait inside the GEMM is
 * bounded; one that runs out sets the device status word (read with
 * ql_read_device_status) to QL_ERR_TIMEOUT. */
int int4_linear_gemm(const uint8_t* xq, const float* x_scale, int64_t M, int64_t K,
                     const uint8_t* w, const float* w_scale, int64_t N, const float* bias,
                     void* y, void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* ------------------------------------------------------------------------ */
/* fp8r (FP8 row-wise)                                                       */
/* ------------------------------------------------------------------------ */

/* Per-row E4M3 quantization ("BFL (fp8r / nvfp4)", scheme list, fp8r entry).
 * Quantizes weights (rows = output channels) and activations (rows = tokens).
 *   x       bf16 [M, K]
 *   xq      uint8 [M, K] E4M3 codes (output)
 *   x_scale fp32 [M] row scales (output)
 * Requires M >= 1, K >= 8, K % 8 == 0. */
int fp8r_quantize_rows(const void* x, int64_t M, int64_t K, uint8_t* xq, float* x_scale,
                       ql_stream_t stream);

/* Bytes of workspace fp8r_linear needs (0 on bad sizes). */
size_t fp8r_linear_workspace_size(int64_t M, int64_t K, int64_t N);

/* fp8r linear forward: quantizes x per row at run time and runs the E4M3 GEMM with
 * the row-wise scales ("Kernels" table: a scaled GEMM with row-wise scales).
 *   x       bf16 [M, K]
 *   w       uint8 [N, K] E4M3 weight codes
 *   w_scale fp32 [N] per-row weight scales
 *   bias    fp32 [N] or NULL
 *   y       bf16 [M, N] (output)
 *   workspace >= fp8r_linear_workspace_size(M, K, N) bytes
 * Requires M, N >= 1, K >= 16, K % 16 == 0. */
int fp8r_linear(const void* x, int64_t M, int64_t K,
                const uint8_t* w, const float* w_scale, int64_t N,
                const float* bias, void* y,
                void* workspace, size_t workspace_bytes, ql_stream_t stream);

/* The GEMM half of fp8r_linear, from activations already quantized by
 * fp8r_quantize_rows: xq uint8 [M, K], x_scale fp32 [M]. */
int fp8r_linear_gemm(const uint8_t* xq, const float* x_scale, int64_t M, int64_t K,
                     const uint8_t* w, const float* w_scale, int64_t N,
                     const float* bias, void* y, ql_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics and status                                                    */
/* ------------------------------------------------------------------------ */

/* The hardware element encoders used by the kernels, on an fp32 array:
 * out[i] = E4M3 code of in[i] (one byte each), or the E2M1 code (low nibble of
 * each byte). in and out are device pointers; n >= 1. */
int ql_encode_e4m3(const float* in, uint8_t* out, int64_t n, ql_stream_t stream);
int ql_encode_e2m1(const float* in, uint8_t* out, int64_t n, ql_stream_t stream);

/* Device status word of the current device: kernels whose bounded waits expire
 * write QL_ERR_TIMEOUT there (they never hang). Reading synchronises the device.
 * ql_read_device_status stores the word in *status (host pointer) and clears it. */
int ql_read_device_status(int* status);

/* The SM clock a GEMM launch ran at: elapsed SM cycles (*cycles) and nanoseconds
 * (*ns) of the first CTA of the most recent NVFP4 or fp8r GEMM launch on the
 * current device (the INT4 GEMM does not record it), from its set-up to its
 * teardown; cycles / ns is that CTA's mean SM clock in GHz. Host pointers;
 * synchronises the device; both 0 before the first launch. No counterpart on the
 * pages: a measurement aid (the part lowers its clock under a heavy tensor-core
 * load, so the dense peak at that clock is the relevant one). QL_ERR_INVALID_ARG
 * for null pointers. */
int ql_read_gemm_clock(int64_t* cycles, int64_t* ns);

/* Test hook: while set (nonzero), the next GEMM launches start with one wait on a
 * barrier that nothing completes, so the bounded-wait path runs and reports
 * QL_ERR_TIMEOUT through the status word. `timeout_ms` bounds every wait of the
 * GEMM kernels (default 2000 ms; 0 restores the default). Host-side settings. */
void ql_set_fault_injection(int enable, int timeout_ms);

/* Tuning override of the GEMM tile shape for later calls (both schemes): output
 * tiles of (128 * cg) rows x bn columns, cg = 2 running each MMA across a pair of
 * SMs. bn in {128, 192, 224, 256}, cg in {1, 2}; bn = 0 restores the automatic choice.
 * Returns QL_OK or QL_ERR_INVALID_ARG. Workspace sizes already cover every tile. */
int ql_set_tile_override(int bn, int cg);

/* The GEMM tile shape a call of this size would use now (the automatic choice, or
 * the override): bn columns, cg = 1 (one SM per 128-row tile) or 2 (a CTA pair per
 * 256-row tile). fp4 = 1 for the NVFP4 GEMM, 0 for fp8r. Host only; bn and cg
 * are written only on QL_OK. QL_ERR_INVALID_ARG for null outputs or sizes < 1. */
int ql_tile_config(int fp4, int64_t M, int64_t N, int64_t K, int* bn, int* cg);

/* Text of a status code, and of the last CUDA error recorded by this thread. */
const char* ql_status_string(int status);
const char* ql_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_H */
