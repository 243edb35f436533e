// Host-side declarations shared by the translation units of the library.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace ql {

constexpr int QL_ERR_TIMEOUT_CODE = 7;  // same value as QL_ERR_TIMEOUT in qlinear.h

// One GEMM launch (both schemes). a, b: row-major codes [M, K*] and [N, K*]
// (K* = K/2 bytes for FP4, K bytes for FP8).
// Tile choice: output tiles of (128 * cg) x bn; cg = 2 runs one MMA over a CTA pair.
struct GemmConfig {
  int bn;
  int cg;
  int arows;  // rows of A per pipeline stage of a skinny kernel (16, 32, 64), or 0
};

struct GemmProblem {
  bool fp4;
  int bn;
  int cg;
  int arows;  // GemmConfig::arows: 0, or the skinny kernel's rows of A per stage
  int64_t M, N, K;
  const void* a;
  const void* b;
  const uint8_t* sfa;    // FP4 only: activation scale atoms
  const uint8_t* sfb;    // FP4 only: weight scale atoms for tile width bn
  const float* scale_a;  // FP4: input_scale scalar; FP8: x_scale [M]
  const float* scale_b;  // FP4: weight_scale_2 scalar; FP8: w_scale [N]
  const float* bias;     // [N] or null
  void* y;               // bf16 [M, N]
  int* status;           // device status word
  uint64_t timeout_ns;
  int inject_fault;
  bool pdl;              // launched right after its producer kernel (programmatic dependency)
  bool b_ready;          // with pdl: B (the weight codes) is not written by that kernel, so the
                         // GEMM may start loading it before the wait (plain mode)
  // fused (FP4, K % 256 == 0): the launch first quantizes x into a (codes) and
  // sfa (scale atoms) and lays out the row-major weight scales into sfb (atoms for
  // tile width bn), then runs the GEMM on them
  bool fused;
  const void* x;             // bf16 [M, K]
  const uint8_t* w_scale;    // E4M3 [N, K/16] row-major (also: a skinny plain GEMM given it
                             // lays out the weight scales itself, per stage)
  uint64_t* sync;            // 8 words (64 bytes) in the workspace
  uint32_t tag;              // odd, different from the previous launch on this workspace
  // GELU-quantize epilogue (FP4, N % 256 == 0): instead of y, NVFP4 of GELU(Y) with
  // global scale *gq_scale into gq_codes [M, N/2] and the activation scale atoms
  // gq_atoms of a layer with K' = N (rows padded to 128)
  bool gelu_quant;
  uint8_t* gq_codes;
  uint8_t* gq_atoms;
  const float* gq_scale;
  // low-rank branch (FP4, plain mode, 8 <= lr_rank <= 64, lr_rank % 8 == 0):
  // Y += alpha * lr_act x lr_up^T with lr_act bf16 [M, r] (the low-rank activations
  // divided by alpha) and lr_up bf16 [N, r]
  const void* lr_act;
  const void* lr_up;
  int lr_rank;
  // FP8 path only: a and b hold f16 [rows, K] instead of E4M3 (kind::f16 MMAs, K
  // tiles of 64 elements); scale_a [M] and scale_b [N] scale the rows and columns
  bool f16_operands;
};

// whole_buffers: only tile widths whose two TMEM accumulator buffers do not share
// a slab (the GELU-quantize epilogue). allow_skinny: M <= 64 may use the skinny
// kernels (plain GEMM without the low-rank branch; the prologue that lays out the
// weight scales must make the same choice).
GemmConfig choose_config(bool fp4, int64_t M, int64_t N, int64_t K, bool whole_buffers = false,
                         bool allow_skinny = true);
bool set_tile_override(int bn, int cg);  // bn == 0 restores the automatic choice
// Elapsed SM cycles and nanoseconds of CTA 0 of the last GEMM launch on the current
// device (synchronous copy from the device).
cudaError_t read_gemm_clock(unsigned long long* cycles, unsigned long long* ns);
cudaError_t launch_gemm(const GemmProblem& p, cudaStream_t stream);

cudaError_t launch_nvfp4_quantize_rowmajor(const void* x, int64_t M, int64_t K, const float* g,
                                           uint8_t* xq, uint8_t* xs, cudaStream_t s);
// The prologue of nvfp4_linear: activations into codes + scale atoms, and (when
// weight_layout) the weight scales into atoms for tiles of bn rows. Without the
// weight layout and with early, it lets the next (skinny) GEMM launch at its start.
cudaError_t launch_nvfp4_prologue(const void* x, int64_t M, int64_t K, const uint8_t* w_scale,
                                  int64_t N, int bn, const float* input_scale, uint8_t* workspace,
                                  cudaStream_t s, bool weight_layout = true, bool early = true);
// The weight scales [N, K/16] into the atoms for tiles of bn rows, at `atoms`
// (the layout of the workspace's weight part).
cudaError_t launch_nvfp4_weight_atoms(const uint8_t* w_scale, int64_t K, int64_t N, int bn,
                                      uint8_t* atoms, cudaStream_t s);
// Weight-scale layout only (the activation part of the workspace is left as is).
cudaError_t launch_nvfp4_weight_layout(const uint8_t* w_scale, int64_t M, int64_t K, int64_t N,
                                       int bn, const float* input_scale, uint8_t* workspace,
                                       cudaStream_t s);
// Prologue of the SVDQuant-style linear in one launch: NVFP4 codes and scale atoms
// of xs = bf16(RN32(x * smooth)) (smooth may be null) into the nvfp4_linear
// workspace, lr_act bf16 [M, rank] = bf16((xs down^T) / alpha) with alpha =
// *input_scale * *weight_scale_2 (rank % 8 == 0, rank <= 64; rank 0 skips it), and
// the weight scales in atom layout for tiles of bn rows. x 16-byte aligned, K % 32 == 0.
cudaError_t launch_svdq_prologue(const void* x, int64_t M, int64_t K, const float* smooth,
                                 const void* down, int rank, const uint8_t* w_scale, int64_t N,
                                 int bn, const float* input_scale, const float* weight_scale_2,
                                 uint8_t* workspace, void* lr_act, int* status,
                                 uint64_t timeout_ns, cudaStream_t s);
// W4A16 linear (w4a16.cu): K % 32 == 0, x / w 16-byte aligned, w_scale 2-byte aligned.
cudaError_t launch_w4a16_linear(const void* x, int64_t M, int64_t K, const uint8_t* w,
                                const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                                const float* bias, void* y, cudaStream_t s);
// INT4 W4A4 (int4.cu): K % 64 == 0; x, q, w 16-byte aligned.
cudaError_t launch_int4_quantize(const void* x, int64_t M, int64_t K, uint8_t* q, float* scale,
                                 cudaStream_t s);
// INT4 rows [rows, K/2] + group scales [rows, K/64] -> f16 [rows, K] (16-byte aligned)
// and the row factors [rows] (out = RN16(RN32(q * s * 2^-e)), factor = 2^e).
cudaError_t launch_int4_dequant_f16(const uint8_t* q, const float* scale, int64_t rows, int64_t K,
                                    void* out, float* factor, cudaStream_t s);
cudaError_t launch_fp8r_quantize_rows(const void* x, int64_t M, int64_t K, uint8_t* xq,
                                      float* x_scale, cudaStream_t s);
cudaError_t launch_global_scale(const void* x, int64_t n, float* out, cudaStream_t s);
cudaError_t launch_encode(const float* in, uint8_t* out, int64_t n, bool fp4, cudaStream_t s);

// 2-D tiled tensor map over a row-major matrix (rows x inner elements, rows
// `row_bytes` apart) with boxes of box_rows x box_inner; false when the driver
// entry point is missing or rejects the arguments. Out-of-range elements load as 0.
bool encode_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
               uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
               CUtensorMapSwizzle swz, CUtensorMapL2promotion promo);

// Sets the text ql_last_error_message() returns on this thread.
void set_error_text(const char* text);

// QL_OK when the current device is an sm_100 part (its ordinal in *dev), else
// QL_ERR_DEVICE or QL_ERR_LAUNCH with the error text set.
int check_current_device(int* dev);

}  // namespace ql
