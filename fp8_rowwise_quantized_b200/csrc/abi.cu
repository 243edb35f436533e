// C ABI of the quantized linear (declared in include/qlinear.h): argument
// validation, workspace carving, device checks, the device status word and the
// error text. Every step of the computation runs in the kernels of quantize.cu
// and gemm.cu; this file only checks arguments and launches them.
#include <cuda_runtime.h>
#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/qlinear.h"
#include "internal.h"
#include "layout.cuh"

namespace {

// Status word written by kernels whose bounded waits expire (one per device).
__device__ int g_device_status;

thread_local char g_last_error[256] = "";
std::atomic<int> g_inject_fault{0};
std::atomic<int> g_timeout_ms{2000};

int record(cudaError_t e, const char* where) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e),
                cudaGetErrorString(e));
  return QL_ERR_LAUNCH;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device must be an sm_100 part; returns QL_OK or an error code.
int check_device(int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record(e, "cudaGetDevice");
  static std::atomic<int> cc_cache[64] = {};  // 0 = unknown, else major*10+minor
  int cc = dev < 64 ? cc_cache[dev].load(std::memory_order_relaxed) : 0;
  if (cc == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return record(e, "cudaDeviceGetAttribute");
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return record(e, "cudaDeviceGetAttribute");
    cc = major * 10 + minor;
    if (dev < 64) cc_cache[dev].store(cc, std::memory_order_relaxed);
  }
  if (cc != 100) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "device %d has compute capability %d.%d; this library runs on sm_100 only", dev,
                  cc / 10, cc % 10);
    return QL_ERR_DEVICE;
  }
  if (dev_out) *dev_out = dev;
  return QL_OK;
}

int* status_ptr(int dev) {
  static int* cache[64] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cache[dev]) return cache[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
  if (dev < 64) cache[dev] = static_cast<int*>(p);
  return static_cast<int*>(p);
}

int fail_shape(const char* what) {
  std::snprintf(g_last_error, sizeof(g_last_error), "shape: %s", what);
  return QL_ERR_SHAPE;
}

uint64_t timeout_ns() { return static_cast<uint64_t>(g_timeout_ms.load()) * 1000000ull; }

// Tag of one single-launch nvfp4_linear call: odd, and different for consecutive
// calls (a per-process counter, mixed, from a time-dependent start), so the sync
// words of the workspace never look finished from an earlier call.
uint32_t next_launch_tag() {
  static const uint32_t start = static_cast<uint32_t>(
      std::chrono::steady_clock::now().time_since_epoch().count() * 0x9E3779B97F4A7C15ull >> 32);
  static std::atomic<uint32_t> seq{0};
  uint32_t t = start + seq.fetch_add(1) * 0x9E3779B9u;
  t ^= t >> 16;
  t *= 0x85EBCA6Bu;
  t ^= t >> 13;
  return t | 1u;
}

bool nvfp4_shape_ok(int64_t M, int64_t K, int64_t N) {
  return M >= 1 && N >= 1 && K >= 32 && K % 32 == 0 && M <= (1ll << 30) && N <= (1ll << 30) &&
         K <= (1ll << 30);
}

bool fp8r_shape_ok(int64_t M, int64_t K, int64_t N) {
  return M >= 1 && N >= 1 && K >= 16 && K % 16 == 0 && M <= (1ll << 30) && N <= (1ll << 30) &&
         K <= (1ll << 30);
}

}  // namespace

int ql::check_current_device(int* dev) { return check_device(dev); }

void ql::set_error_text(const char* text) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", text);
}

extern "C" {

const char* ql_status_string(int status) {
  switch (status) {
    case QL_OK: return "ok";
    case QL_ERR_INVALID_ARG: return "invalid argument (null pointer or non-positive size)";
    case QL_ERR_SHAPE: return "unsupported shape";
    case QL_ERR_ALIGN: return "base pointer not 16-byte aligned";
    case QL_ERR_DEVICE: return "device is not sm_100";
    case QL_ERR_WORKSPACE: return "workspace missing or too small";
    case QL_ERR_LAUNCH: return "CUDA launch or runtime error";
    case QL_ERR_TIMEOUT: return "a kernel's bounded wait expired";
  }
  return "unknown status";
}

const char* ql_last_error_message(void) { return g_last_error; }

void ql_set_fault_injection(int enable, int timeout_ms) {
  g_inject_fault.store(enable ? 1 : 0);
  g_timeout_ms.store(timeout_ms > 0 ? timeout_ms : 2000);
}

int ql_read_gemm_clock(int64_t* cycles, int64_t* ns) {
  if (!cycles || !ns) return QL_ERR_INVALID_ARG;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  unsigned long long c = 0, t = 0;
  cudaError_t e = ql::read_gemm_clock(&c, &t);
  if (e != cudaSuccess) return record(e, "ql_read_gemm_clock");
  *cycles = static_cast<int64_t>(c);
  *ns = static_cast<int64_t>(t);
  return QL_OK;
}

int ql_read_device_status(int* status) {
  if (!status) return QL_ERR_INVALID_ARG;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != QL_OK) return rc;
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e != cudaSuccess) return record(e, "cudaMemcpyFromSymbol");
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return record(e, "cudaMemcpyToSymbol");
  *status = v;
  return QL_OK;
}

// ------------------------------------------------------------------ NVFP4

int nvfp4_quantize_act(const void* x, int64_t M, int64_t K, const float* input_scale,
                       uint8_t* xq, uint8_t* xs, ql_stream_t stream) {
  if (!x || !input_scale || !xq || !xs || M <= 0 || K <= 0) return QL_ERR_INVALID_ARG;
  if (K % 16 != 0) return fail_shape("K must be a multiple of 16");
  if (!aligned16(x) || !aligned16(xq)) return QL_ERR_ALIGN;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_nvfp4_quantize_rowmajor(x, M, K, input_scale, xq, xs,
                                                     reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "nvfp4_quantize_act");
}

size_t nvfp4_linear_workspace_size(int64_t M, int64_t K, int64_t N) {
  if (!nvfp4_shape_ok(M, K, N)) return 0;
  // large enough for the weight-scale layout of every tile width the call may use
  // (the narrow widths of the skinny kernels only when M <= 64)
  size_t need = 0;
  for (int bn : {64, 96, 128, 192, 224, 256}) {
    if (bn < 128 && M > 64) continue;
    const size_t t = ql::nvfp4_workspace(M, K, N, bn).total;
    need = t > need ? t : need;
  }
  return need;
}

int ql_tile_config(int fp4, int64_t M, int64_t N, int64_t K, int* bn, int* cg) {
  if (!bn || !cg || M < 1 || N < 1 || K < 1) return QL_ERR_INVALID_ARG;
  const ql::GemmConfig c = ql::choose_config(fp4 != 0, M, N, K);
  *bn = c.bn;
  *cg = c.cg;
  return QL_OK;
}

int ql_set_tile_override(int bn, int cg) {
  return ql::set_tile_override(bn, cg) ? QL_OK : QL_ERR_INVALID_ARG;
}

int nvfp4_linear_workspace_layout(int64_t M, int64_t K, int64_t N, size_t* codes_offset,
                                  size_t* act_scales_offset, size_t* weight_scales_offset) {
  if (!nvfp4_shape_ok(M, K, N)) return QL_ERR_SHAPE;
  const ql::Nvfp4Workspace L = ql::nvfp4_workspace(M, K, N, ql::choose_config(true, M, N, K).bn);
  if (codes_offset) *codes_offset = L.codes_off;
  if (act_scales_offset) *act_scales_offset = L.act_sf_off;
  if (weight_scales_offset) *weight_scales_offset = L.wgt_sf_off;
  return QL_OK;
}

int nvfp4_linear_prologue(const void* x, int64_t M, int64_t K, const uint8_t* w_scale, int64_t N,
                          const float* input_scale, void* workspace, size_t workspace_bytes,
                          ql_stream_t stream) {
  if (!x || !w_scale || !input_scale || M <= 0 || N <= 0 || K <= 0) return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N)) return fail_shape("nvfp4: needs K >= 32 and K % 32 == 0");
  if (!aligned16(x)) return QL_ERR_ALIGN;
  const int bn = ql::choose_config(true, M, N, K).bn;
  const ql::Nvfp4Workspace L = ql::nvfp4_workspace(M, K, N, bn);
  if (!workspace || workspace_bytes < nvfp4_linear_workspace_size(M, K, N)) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_nvfp4_prologue(x, M, K, w_scale, N, bn, input_scale,
                                            static_cast<uint8_t*>(workspace),
                                            reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "nvfp4_linear_prologue");
}

static int nvfp4_gemm_impl(int64_t M, int64_t K, const uint8_t* w, int64_t N,
                           const float* weight_scale_2, const float* input_scale,
                           const float* bias, void* y, const void* workspace,
                           size_t workspace_bytes, ql_stream_t stream, bool pdl,
                           const void* lr_act = nullptr, const void* lr_up = nullptr,
                           int lr_rank = 0, const uint8_t* w_scale_rowmajor = nullptr) {
  if (!w || !weight_scale_2 || !input_scale || !y || M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N)) return fail_shape("nvfp4: needs K >= 32 and K % 32 == 0");
  if (!aligned16(w) || !aligned16(y) || (bias && !aligned16(bias))) return QL_ERR_ALIGN;
  const ql::GemmConfig cfg = ql::choose_config(true, M, N, K);
  const int bn = cfg.bn;
  const ql::Nvfp4Workspace L = ql::nvfp4_workspace(M, K, N, bn);
  if (!workspace || workspace_bytes < nvfp4_linear_workspace_size(M, K, N)) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != QL_OK) return rc;
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  ql::GemmProblem p{};
  p.fp4 = true;
  p.bn = bn;
  p.cg = cfg.cg;
  p.arows = cfg.arows;
  p.M = M;
  p.N = N;
  p.K = K;
  p.a = ws + L.codes_off;
  p.b = w;
  p.sfa = ws + L.act_sf_off;
  p.sfb = ws + L.wgt_sf_off;
  p.scale_a = input_scale;
  p.scale_b = weight_scale_2;
  p.bias = bias;
  p.y = y;
  p.status = status_ptr(dev);
  p.timeout_ns = timeout_ns();
  p.inject_fault = g_inject_fault.load();
  p.pdl = pdl;
  p.b_ready = true;  // the kernel before is this library's prologue: it does not write w
  p.lr_act = lr_act;
  p.lr_up = lr_up;
  p.lr_rank = lr_rank;
  if (cfg.arows > 0) p.w_scale = w_scale_rowmajor;  // skinny: scales laid out in the GEMM
  cudaError_t e = ql::launch_gemm(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "nvfp4 gemm launch");
}

int nvfp4_linear_gemm(int64_t M, int64_t K, const uint8_t* w, int64_t N,
                      const float* weight_scale_2, const float* input_scale, const float* bias,
                      void* y, const void* workspace, size_t workspace_bytes, ql_stream_t stream) {
  return nvfp4_gemm_impl(M, K, w, N, weight_scale_2, input_scale, bias, y, workspace,
                         workspace_bytes, stream, false);
}

int nvfp4_linear_gemm_lowrank(int64_t M, int64_t K, const uint8_t* w, int64_t N,
                              const float* weight_scale_2, const float* input_scale,
                              const float* bias, const void* lr_act, const void* lr_up,
                              int64_t rank, void* y, const void* workspace,
                              size_t workspace_bytes, ql_stream_t stream) {
  if (!lr_act || !lr_up) return QL_ERR_INVALID_ARG;
  if (rank < 8 || rank > 64 || rank % 8 != 0)
    return fail_shape("low-rank branch: needs rank in 8..64, rank % 8 == 0");
  if (!aligned16(lr_act) || !aligned16(lr_up)) return QL_ERR_ALIGN;
  return nvfp4_gemm_impl(M, K, w, N, weight_scale_2, input_scale, bias, y, workspace,
                         workspace_bytes, stream, false, lr_act, lr_up, static_cast<int>(rank));
}

size_t svdq_nvfp4_linear_workspace_size(int64_t M, int64_t K, int64_t N, int64_t rank) {
  const size_t base = nvfp4_linear_workspace_size(M, K, N);
  if (base == 0 || rank < 8 || rank > 64 || rank % 8 != 0) return 0;
  return base + ql::align_up(static_cast<size_t>(M) * static_cast<size_t>(rank) * 2, 1024);
}

int svdq_nvfp4_linear(const void* x, int64_t M, int64_t K, const float* smooth,
                      const void* lora_down, const void* lora_up, int64_t rank, const uint8_t* w,
                      const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                      const float* input_scale, const float* bias, void* y, void* workspace,
                      size_t workspace_bytes, ql_stream_t stream) {
  if (!x || !lora_down || !lora_up || !w || !w_scale || !weight_scale_2 || !input_scale || !y ||
      M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N)) return fail_shape("nvfp4: needs K >= 32 and K % 32 == 0");
  if (rank < 8 || rank > 64 || rank % 8 != 0)
    return fail_shape("low-rank branch: needs rank in 8..64, rank % 8 == 0");
  if (!aligned16(x) || (smooth && !aligned16(smooth)) || !aligned16(lora_down) ||
      !aligned16(lora_up) || !aligned16(w) || !aligned16(y) || (bias && !aligned16(bias)))
    return QL_ERR_ALIGN;
  const size_t base = nvfp4_linear_workspace_size(M, K, N);
  if (!workspace || workspace_bytes < svdq_nvfp4_linear_workspace_size(M, K, N, rank))
    return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != QL_OK) return rc;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int bn = ql::choose_config(true, M, N, K).bn;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* lr_act = ws + base;
  // 1. one pass over x: smoothing, NVFP4 of the smoothed activations, the low-rank
  //    down projection (divided by alpha), weight-scale layout
  const cudaError_t e = ql::launch_svdq_prologue(
      x, M, K, smooth, lora_down, static_cast<int>(rank), w_scale, N, bn, input_scale,
      weight_scale_2, ws, lr_act, status_ptr(dev), timeout_ns(), s);
  if (e != cudaSuccess) return record(e, "svdq_nvfp4_linear prologue");
  // 2. the 4-bit GEMM with the low-rank up projection as one more K step
  return nvfp4_gemm_impl(M, K, w, N, weight_scale_2, input_scale, bias, y, workspace,
                         workspace_bytes, stream, true, lr_act, lora_up, static_cast<int>(rank));
}

int nvfp4_linear(const void* x, int64_t M, int64_t K, const uint8_t* w, const uint8_t* w_scale,
                 int64_t N, const float* weight_scale_2, const float* input_scale,
                 const float* bias, void* y, void* workspace, size_t workspace_bytes,
                 ql_stream_t stream) {
  if (!x || !w || !w_scale || !weight_scale_2 || !input_scale || !y || M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N)) return fail_shape("nvfp4: needs K >= 32 and K % 32 == 0");
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || (bias && !aligned16(bias)))
    return QL_ERR_ALIGN;
  if (!workspace || workspace_bytes < nvfp4_linear_workspace_size(M, K, N)) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  if (ql::choose_config(true, M, N, K).arows > 0) {
    // skinny layer: the prologue quantizes the activations only and lets the GEMM
    // launch at once; the GEMM streams the weights meanwhile and lays out their
    // scales itself, then waits for the activations
    int rc = check_device(nullptr);
    if (rc != QL_OK) return rc;
    const cudaError_t e = ql::launch_nvfp4_prologue(
        x, M, K, w_scale, N, ql::choose_config(true, M, N, K).bn, input_scale,
        static_cast<uint8_t*>(workspace), reinterpret_cast<cudaStream_t>(stream), false);
    if (e != cudaSuccess) return record(e, "nvfp4_linear prologue");
    return nvfp4_gemm_impl(M, K, w, N, weight_scale_2, input_scale, bias, y, workspace,
                           workspace_bytes, stream, true, nullptr, nullptr, 0, w_scale);
  }
  int rc = nvfp4_linear_prologue(x, M, K, w_scale, N, input_scale, workspace, workspace_bytes,
                                 stream);
  if (rc != QL_OK) return rc;
  return nvfp4_gemm_impl(M, K, w, N, weight_scale_2, input_scale, bias, y, workspace,
                         workspace_bytes, stream, true);
}

static bool laid_out_width_ok(int bn) { return bn == 128 || bn == 192 || bn == 224 || bn == 256; }

size_t nvfp4_weight_scale_atoms_size(int64_t N, int64_t K, int bn) {
  if (!nvfp4_shape_ok(1, K, N) || !laid_out_width_ok(bn)) return 0;
  const int64_t na = (bn + 127) / 128;
  return static_cast<size_t>(ql::ceil_div64(N, bn) * ql::sf_kgroups(K) * na) * ql::kSfAtomBytes;
}

int nvfp4_layout_weight_scales(const uint8_t* w_scale, int64_t N, int64_t K, int bn,
                               uint8_t* atoms, size_t atoms_bytes, ql_stream_t stream) {
  if (!w_scale || !atoms || N <= 0 || K <= 0) return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(1, K, N)) return fail_shape("nvfp4: needs K >= 32 and K % 32 == 0");
  if (!laid_out_width_ok(bn)) return fail_shape("weight-scale layout: bn must be 128, 192, 224 or 256");
  if (atoms_bytes < nvfp4_weight_scale_atoms_size(N, K, bn)) return QL_ERR_WORKSPACE;
  if (!aligned16(atoms)) return QL_ERR_ALIGN;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_nvfp4_weight_atoms(w_scale, K, N, bn, atoms,
                                                reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "nvfp4_layout_weight_scales");
}

int nvfp4_linear_laid_out(const void* x, int64_t M, int64_t K, const uint8_t* w,
                          const uint8_t* w_scale_atoms, int bn, int64_t N,
                          const float* weight_scale_2, const float* input_scale,
                          const float* bias, void* y, void* workspace, size_t workspace_bytes,
                          ql_stream_t stream) {
  if (!x || !w || !w_scale_atoms || !weight_scale_2 || !input_scale || !y || M <= 0 || N <= 0 ||
      K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N)) return fail_shape("nvfp4: needs K >= 32 and K % 32 == 0");
  if (!laid_out_width_ok(bn)) return fail_shape("weight-scale layout: bn must be 128, 192, 224 or 256");
  if (!aligned16(x) || !aligned16(w) || !aligned16(w_scale_atoms) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return QL_ERR_ALIGN;
  if (!workspace || workspace_bytes < nvfp4_linear_workspace_size(M, K, N)) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != QL_OK) return rc;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the activations only (the ordinary prologue kernel, its weight jobs empty)
  cudaError_t e = ql::launch_nvfp4_prologue(x, M, K, nullptr, N, bn, input_scale,
                                            static_cast<uint8_t*>(workspace), s, false, false);
  if (e != cudaSuccess) return record(e, "nvfp4_linear_laid_out prologue");
  const ql::Nvfp4Workspace L = ql::nvfp4_workspace(M, K, N, bn);
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  ql::GemmProblem p{};
  p.fp4 = true;
  p.bn = bn;
  p.cg = M >= 512 ? 2 : 1;  // the automatic choice's rule for pairs
  p.arows = 0;
  p.M = M;
  p.N = N;
  p.K = K;
  p.a = ws + L.codes_off;
  p.b = w;
  p.sfa = ws + L.act_sf_off;
  p.sfb = w_scale_atoms;
  p.scale_a = input_scale;
  p.scale_b = weight_scale_2;
  p.bias = bias;
  p.y = y;
  p.status = status_ptr(dev);
  p.timeout_ns = timeout_ns();
  p.inject_fault = g_inject_fault.load();
  p.pdl = true;
  p.b_ready = true;  // the kernel before is the activation prologue: it does not write w
  e = ql::launch_gemm(p, s);
  return e == cudaSuccess ? QL_OK : record(e, "nvfp4_linear_laid_out gemm");
}

int nvfp4_linear_single_launch(const void* x, int64_t M, int64_t K, const uint8_t* w,
                               const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                               const float* input_scale, const float* bias, void* y,
                               void* workspace, size_t workspace_bytes, ql_stream_t stream) {
  if (!x || !w || !w_scale || !weight_scale_2 || !input_scale || !y || M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N) || K % 256 != 0)
    return fail_shape("nvfp4_linear_single_launch: needs K % 256 == 0");
  if (!aligned16(x) || !aligned16(w) || !aligned16(w_scale) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return QL_ERR_ALIGN;
  if (!workspace || workspace_bytes < nvfp4_linear_workspace_size(M, K, N)) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  // one launch: the GEMM kernel first quantizes the activations and lays out
  // the weight scales into the workspace (which stays in L2), then multiplies
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != QL_OK) return rc;
  const ql::GemmConfig cfg = ql::choose_config(true, M, N, K, false, false);
  const ql::Nvfp4Workspace L = ql::nvfp4_workspace(M, K, N, cfg.bn);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  ql::GemmProblem p{};
  p.fp4 = true;
  p.bn = cfg.bn;
  p.cg = cfg.cg;
  p.M = M;
  p.N = N;
  p.K = K;
  p.a = ws + L.codes_off;
  p.b = w;
  p.sfa = ws + L.act_sf_off;
  p.sfb = ws + L.wgt_sf_off;
  p.scale_a = input_scale;
  p.scale_b = weight_scale_2;
  p.bias = bias;
  p.y = y;
  p.status = status_ptr(dev);
  p.timeout_ns = timeout_ns();
  p.inject_fault = g_inject_fault.load();
  p.pdl = false;
  p.fused = true;
  p.x = x;
  p.w_scale = w_scale;
  p.sync = reinterpret_cast<uint64_t*>(ws + L.sync_off);
  p.tag = next_launch_tag();
  cudaError_t e = ql::launch_gemm(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "nvfp4_linear_single_launch");
}

int nvfp4_linear_gelu_quantize(const void* x, int64_t M, int64_t K, const uint8_t* w,
                               const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                               const float* input_scale, const float* bias,
                               const float* next_input_scale, void* next_workspace,
                               size_t next_workspace_bytes, void* workspace,
                               size_t workspace_bytes, ql_stream_t stream) {
  if (!x || !w || !w_scale || !weight_scale_2 || !input_scale || !next_input_scale ||
      !next_workspace || M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N)) return fail_shape("nvfp4: needs K >= 32 and K % 32 == 0");
  if (N % 256 != 0) return fail_shape("nvfp4_linear_gelu_quantize: needs N % 256 == 0");
  if (!aligned16(x) || !aligned16(w) || (bias && !aligned16(bias)) || !aligned16(next_workspace))
    return QL_ERR_ALIGN;
  // the next layer's activations: K' = N; their part of its workspace does not
  // depend on its N' or tile width
  const ql::Nvfp4Workspace next = ql::nvfp4_workspace(M, N, 1, 128);
  const size_t next_need = next.act_sf_off + static_cast<size_t>((M + 127) / 128) *
                                                 static_cast<size_t>(N / 64) * ql::kSfAtomBytes;
  if (next_workspace_bytes < next_need) return QL_ERR_WORKSPACE;
  if (!workspace || workspace_bytes < nvfp4_linear_workspace_size(M, K, N)) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != QL_OK) return rc;
  // tiles whose accumulator buffers are whole (this epilogue's 8 warps split them)
  const ql::GemmConfig cfg = ql::choose_config(true, M, N, K, true);
  cudaError_t pe = ql::launch_nvfp4_prologue(x, M, K, w_scale, N, cfg.bn, input_scale,
                                             static_cast<uint8_t*>(workspace),
                                             reinterpret_cast<cudaStream_t>(stream));
  if (pe != cudaSuccess) return record(pe, "nvfp4_linear_gelu_quantize prologue");
  const ql::Nvfp4Workspace L = ql::nvfp4_workspace(M, K, N, cfg.bn);
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  uint8_t* nws = static_cast<uint8_t*>(next_workspace);
  ql::GemmProblem p{};
  p.fp4 = true;
  p.bn = cfg.bn;
  p.cg = cfg.cg;
  p.M = M;
  p.N = N;
  p.K = K;
  p.a = ws + L.codes_off;
  p.b = w;
  p.sfa = ws + L.act_sf_off;
  p.sfb = ws + L.wgt_sf_off;
  p.scale_a = input_scale;
  p.scale_b = weight_scale_2;
  p.bias = bias;
  p.y = nullptr;
  p.status = status_ptr(dev);
  p.timeout_ns = timeout_ns();
  p.inject_fault = g_inject_fault.load();
  p.pdl = true;
  p.gelu_quant = true;
  p.gq_codes = nws + next.codes_off;
  p.gq_atoms = nws + next.act_sf_off;
  p.gq_scale = next_input_scale;
  cudaError_t e = ql::launch_gemm(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "nvfp4_linear_gelu_quantize");
}

int nvfp4_linear_quantized_input(int64_t M, int64_t K, const uint8_t* w, const uint8_t* w_scale,
                                 int64_t N, const float* weight_scale_2,
                                 const float* input_scale, const float* bias, void* y,
                                 void* workspace, size_t workspace_bytes, ql_stream_t stream) {
  if (!w || !w_scale || !weight_scale_2 || !input_scale || !y || !workspace || M <= 0 ||
      N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N)) return fail_shape("nvfp4: needs K >= 32 and K % 32 == 0");
  if (workspace_bytes < nvfp4_linear_workspace_size(M, K, N)) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  const int bn = ql::choose_config(true, M, N, K).bn;
  cudaError_t e = ql::launch_nvfp4_weight_layout(w_scale, M, K, N, bn, input_scale,
                                                 static_cast<uint8_t*>(workspace),
                                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return record(e, "nvfp4_linear_quantized_input");
  return nvfp4_gemm_impl(M, K, w, N, weight_scale_2, input_scale, bias, y, workspace,
                         workspace_bytes, stream, true);
}

int w4a16_linear(const void* x, int64_t M, int64_t K, const uint8_t* w, const uint8_t* w_scale,
                 int64_t N, const float* weight_scale_2, const float* bias, void* y,
                 ql_stream_t stream) {
  if (!x || !w || !w_scale || !weight_scale_2 || !y || M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!nvfp4_shape_ok(M, K, N)) return fail_shape("w4a16: needs K >= 32 and K % 32 == 0");
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(w_scale) & 1u) != 0 ||
      (reinterpret_cast<uintptr_t>(bias) & 3u) != 0)
    return QL_ERR_ALIGN;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_w4a16_linear(x, M, K, w, w_scale, N, weight_scale_2, bias, y,
                                          reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "w4a16_linear");
}

int nvfp4_global_scale(const void* x, int64_t n, float* out, ql_stream_t stream) {
  if (!x || !out || n <= 0) return QL_ERR_INVALID_ARG;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_global_scale(x, n, out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "nvfp4_global_scale");
}

// ------------------------------------------------------------------ fp8r

int fp8r_quantize_rows(const void* x, int64_t M, int64_t K, uint8_t* xq, float* x_scale,
                       ql_stream_t stream) {
  if (!x || !xq || !x_scale || M <= 0 || K <= 0) return QL_ERR_INVALID_ARG;
  if (K % 8 != 0) return fail_shape("fp8r: K must be a multiple of 8");
  if (!aligned16(x) || !aligned16(xq)) return QL_ERR_ALIGN;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_fp8r_quantize_rows(x, M, K, xq, x_scale,
                                                reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "fp8r_quantize_rows");
}

size_t fp8r_linear_workspace_size(int64_t M, int64_t K, int64_t N) {
  if (!fp8r_shape_ok(M, K, N)) return 0;
  return ql::align_up(static_cast<size_t>(M) * static_cast<size_t>(K), 1024) +
         ql::align_up(static_cast<size_t>(M) * 4, 1024);
}

static int fp8r_gemm_impl(const uint8_t* xq, const float* x_scale, int64_t M, int64_t K,
                          const uint8_t* w, const float* w_scale, int64_t N, const float* bias,
                          void* y, ql_stream_t stream, bool pdl) {
  if (!xq || !x_scale || !w || !w_scale || !y || M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!fp8r_shape_ok(M, K, N)) return fail_shape("fp8r: needs K >= 16 and K % 16 == 0");
  if (!aligned16(xq) || !aligned16(w) || !aligned16(y) || !aligned16(w_scale) ||
      (bias && !aligned16(bias)))
    return QL_ERR_ALIGN;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != QL_OK) return rc;
  ql::GemmProblem p{};
  p.fp4 = false;
  const ql::GemmConfig cfg = ql::choose_config(false, M, N, K);
  p.bn = cfg.bn;
  p.cg = cfg.cg;
  p.M = M;
  p.N = N;
  p.K = K;
  p.a = xq;
  p.b = w;
  p.scale_a = x_scale;
  p.scale_b = w_scale;
  p.bias = bias;
  p.y = y;
  p.status = status_ptr(dev);
  p.timeout_ns = timeout_ns();
  p.inject_fault = g_inject_fault.load();
  p.pdl = pdl;
  p.b_ready = true;  // the kernel before is fp8r_quantize_rows: it does not write w
  cudaError_t e = ql::launch_gemm(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "fp8r gemm launch");
}

int fp8r_linear_gemm(const uint8_t* xq, const float* x_scale, int64_t M, int64_t K,
                     const uint8_t* w, const float* w_scale, int64_t N, const float* bias, void* y,
                     ql_stream_t stream) {
  return fp8r_gemm_impl(xq, x_scale, M, K, w, w_scale, N, bias, y, stream, false);
}

int fp8r_linear(const void* x, int64_t M, int64_t K, const uint8_t* w, const float* w_scale,
                int64_t N, const float* bias, void* y, void* workspace, size_t workspace_bytes,
                ql_stream_t stream) {
  if (!x || !w || !w_scale || !y || M <= 0 || N <= 0 || K <= 0) return QL_ERR_INVALID_ARG;
  if (!fp8r_shape_ok(M, K, N)) return fail_shape("fp8r: needs K >= 16 and K % 16 == 0");
  const size_t need = fp8r_linear_workspace_size(M, K, N);
  if (!workspace || workspace_bytes < need) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  uint8_t* xq = static_cast<uint8_t*>(workspace);
  float* xs = reinterpret_cast<float*>(xq + ql::align_up(static_cast<size_t>(M) * K, 1024));
  int rc = fp8r_quantize_rows(x, M, K, xq, xs, stream);
  if (rc != QL_OK) return rc;
  return fp8r_gemm_impl(xq, xs, M, K, w, w_scale, N, bias, y, stream, true);
}

// ------------------------------------------------------------------ INT4 W4A4

static bool int4_shape_ok(int64_t M, int64_t K, int64_t N) {
  return M >= 1 && N >= 1 && K >= 64 && K % 64 == 0 && M <= (1ll << 30) && N <= (1ll << 30) &&
         K <= (1ll << 30);
}

int int4_quantize_rows(const void* x, int64_t M, int64_t K, uint8_t* q, float* scale,
                       ql_stream_t stream) {
  if (!x || !q || !scale || M <= 0 || K <= 0) return QL_ERR_INVALID_ARG;
  if (!int4_shape_ok(M, K, 1)) return fail_shape("int4: needs K >= 64 and K % 64 == 0");
  if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
    return QL_ERR_ALIGN;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_int4_quantize(x, M, K, q, scale, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "int4_quantize_rows");
}

size_t int4_linear_gemm_workspace_size(int64_t M, int64_t K, int64_t N) {
  if (!int4_shape_ok(M, K, N)) return 0;
  return ql::align_up(static_cast<size_t>(M) * static_cast<size_t>(K) * 2, 1024) +
         ql::align_up(static_cast<size_t>(M) * 4, 1024) +
         ql::align_up(static_cast<size_t>(N) * static_cast<size_t>(K) * 2, 1024) +
         ql::align_up(static_cast<size_t>(N) * 4, 1024);
}

int int4_linear_gemm(const uint8_t* xq, const float* x_scale, int64_t M, int64_t K,
                     const uint8_t* w, const float* w_scale, int64_t N, const float* bias,
                     void* y, void* workspace, size_t workspace_bytes, ql_stream_t stream) {
  if (!xq || !x_scale || !w || !w_scale || !y || M <= 0 || N <= 0 || K <= 0)
    return QL_ERR_INVALID_ARG;
  if (!int4_shape_ok(M, K, N)) return fail_shape("int4: needs K >= 64 and K % 64 == 0");
  if (!workspace || workspace_bytes < int4_linear_gemm_workspace_size(M, K, N))
    return QL_ERR_WORKSPACE;
  if (!aligned16(xq) || !aligned16(w) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(x_scale) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(w_scale) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(bias) & 3u) != 0 || (reinterpret_cast<uintptr_t>(y) & 1u) != 0)
    return QL_ERR_ALIGN;
  int dev = 0;
  int rc = check_device(&dev);
  if (rc != QL_OK) return rc;
  // workspace: f16 x [M, K] | x row factors [M] | f16 w [N, K] | w row factors [N]
  uint8_t* base = static_cast<uint8_t*>(workspace);
  void* xh = base;
  base += ql::align_up(static_cast<size_t>(M) * static_cast<size_t>(K) * 2, 1024);
  float* xf = reinterpret_cast<float*>(base);
  base += ql::align_up(static_cast<size_t>(M) * 4, 1024);
  void* wh = base;
  base += ql::align_up(static_cast<size_t>(N) * static_cast<size_t>(K) * 2, 1024);
  float* wf = reinterpret_cast<float*>(base);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = ql::launch_int4_dequant_f16(xq, x_scale, M, K, xh, xf, s);
  if (e != cudaSuccess) return record(e, "int4 dequantize x");
  e = ql::launch_int4_dequant_f16(w, w_scale, N, K, wh, wf, s);
  if (e != cudaSuccess) return record(e, "int4 dequantize w");
  ql::GemmProblem p{};
  p.fp4 = false;
  p.f16_operands = true;
  const ql::GemmConfig cfg = ql::choose_config(false, M, N, K);
  p.bn = cfg.bn;
  p.cg = cfg.cg;
  p.M = M;
  p.N = N;
  p.K = K;
  p.a = xh;
  p.b = wh;
  p.scale_a = xf;
  p.scale_b = wf;
  p.bias = bias;
  p.y = y;
  p.status = status_ptr(dev);
  p.timeout_ns = timeout_ns();
  p.inject_fault = g_inject_fault.load();
  p.pdl = true;
  e = ql::launch_gemm(p, s);
  return e == cudaSuccess ? QL_OK : record(e, "int4 f16 gemm launch");
}

size_t int4_linear_workspace_size(int64_t M, int64_t K, int64_t N) {
  if (!int4_shape_ok(M, K, N)) return 0;
  return ql::align_up(static_cast<size_t>(M) * static_cast<size_t>(K / 2), 1024) +
         ql::align_up(static_cast<size_t>(M) * static_cast<size_t>(K / 64) * 4, 1024) +
         int4_linear_gemm_workspace_size(M, K, N);
}

int int4_linear(const void* x, int64_t M, int64_t K, const uint8_t* w, const float* w_scale,
                int64_t N, const float* bias, void* y, void* workspace, size_t workspace_bytes,
                ql_stream_t stream) {
  if (!x || !w || !w_scale || !y || M <= 0 || N <= 0 || K <= 0) return QL_ERR_INVALID_ARG;
  if (!int4_shape_ok(M, K, N)) return fail_shape("int4: needs K >= 64 and K % 64 == 0");
  if (!workspace || workspace_bytes < int4_linear_workspace_size(M, K, N)) return QL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QL_ERR_ALIGN;
  uint8_t* xq = static_cast<uint8_t*>(workspace);
  const size_t q_bytes = ql::align_up(static_cast<size_t>(M) * static_cast<size_t>(K / 2), 1024);
  const size_t s_bytes = ql::align_up(static_cast<size_t>(M) * static_cast<size_t>(K / 64) * 4, 1024);
  float* xs = reinterpret_cast<float*>(xq + q_bytes);
  int rc = int4_quantize_rows(x, M, K, xq, xs, stream);
  if (rc != QL_OK) return rc;
  return int4_linear_gemm(xq, xs, M, K, w, w_scale, N, bias, y, xq + q_bytes + s_bytes,
                          workspace_bytes - q_bytes - s_bytes, stream);
}

// ------------------------------------------------------------------ diagnostics

int ql_encode_e4m3(const float* in, uint8_t* out, int64_t n, ql_stream_t stream) {
  if (!in || !out || n <= 0) return QL_ERR_INVALID_ARG;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_encode(in, out, n, false, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "ql_encode_e4m3");
}

int ql_encode_e2m1(const float* in, uint8_t* out, int64_t n, ql_stream_t stream) {
  if (!in || !out || n <= 0) return QL_ERR_INVALID_ARG;
  int rc = check_device(nullptr);
  if (rc != QL_OK) return rc;
  cudaError_t e = ql::launch_encode(in, out, n, true, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QL_OK : record(e, "ql_encode_e2m1");
}

}  // extern "C"
