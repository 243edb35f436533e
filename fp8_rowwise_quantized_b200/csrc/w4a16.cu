// W4A16 linear: 4-bit NVFP4 weights, bf16 activations, bf16 output.
//
// The layer family of "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers"
// (section "Introducing Nunchaku Lite", kernel families: awq_w4a16) for the adaptive
// normalization / modulation projections, with the weight format of the nvfp4
// scheme of the Diffusers page "BFL (fp8r / nvfp4)" (scheme list). The weight is
// dequantized to the compute dtype (the unfused path of that page, section
// "Kernels", last paragraph):
//   what[n, k] = bf16(RN32(E2M1(w[n, k]) * E4M3(w_scale[n, k/16]) * weight_scale_2))
//   y[m, n]    = bf16(sum_k x[m, k] * what[n, k] + bias[n])
// and the activations stay in bf16.
//
// These layers run on a few token rows (a batch of conditioning vectors), so the
// kernel is a GEMV that streams the weight once from HBM: per byte of weight codes
// it does a fixed amount of decode work and a few fp32 FMAs on the CUDA cores. A
// tensor-core GEMM would waste the MMA on padding and add a shared-memory round
// trip without moving the HBM bound.
//
// Work split: one warp owns kRows consecutive weight rows at a time; lane l reads
// the 32-element chunks l, l + 32, ... of each of those rows (16 bytes of codes and
// two scale bytes per chunk and row, the next chunk prefetched while the current
// one is decoded), multiplies them with the same chunk of up to MR activation rows
// (read through L1; every warp of the SM reads the same few KB), and accumulates
// in fp32 (even and odd elements in the two halves of packed f32x2 FMAs). A warp
// butterfly sums the lanes, and lane i writes one (row, column) output.
// Grid: one wave of persistent CTAs (SM count x resident CTAs per SM) striding
// over the row groups; grid.y walks the activation rows MR at a time.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace ql {
namespace {

constexpr int kW4Threads = 256;
constexpr int kW4Warps = kW4Threads / 32;
constexpr int kRows = 4;  // weight rows per warp task

// Packed fp32 pair (element 2i in the low word).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack_f32x2(uint64_t p, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}

// acc += a * b, both lanes of the packed pairs, each an fp32 fma (RN).
__device__ __forceinline__ void fma_f32x2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// Block scale code s -> (E4M3(s), E4M3(s)) as an f16x2 word (exact: every E4M3
// value is an f16 value).
__device__ __forceinline__ uint32_t scale_f16x2(uint32_t s) {
  uint32_t r;
  asm("{\n\t.reg .b16 c;\n\t"
      "cvt.u16.u32 c, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, c;\n\t}"
      : "=r"(r)
      : "r"(s | (s << 8)));
  return r;
}

// Two E2M1 codes (one byte of the packed weight: element 2j in the low nibble) ->
// the two dequantized weights as bf16 bits in the high halves of two fp32 words:
//   p = E2M1 * E4M3(s) in f16 (exact: at most 6 significant bits, 2^-10 <= |p| <=
//       2688 or 0),
//   RN32(p * g) (two fp32 lanes), then RN to bf16 (one cvt for the pair).
// Returns the packed pair of fp32 values (element 2j in the low word).
__device__ __forceinline__ uint64_t w4_decode2(uint32_t byte, uint32_t ss, uint64_t gg) {
  uint64_t r;
  asm("{\n\t"
      ".reg .b8 c;\n\t"
      ".reg .b16 lo16, hi16;\n\t"
      ".reg .b32 h, f0, f1, b, w0, w1;\n\t"
      ".reg .b64 p;\n\t"
      "cvt.u8.u32 c, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 h, c;\n\t"
      "mul.rn.f16x2 h, h, %2;\n\t"
      "mov.b32 {lo16, hi16}, h;\n\t"
      "cvt.f32.f16 f0, lo16;\n\t"
      "cvt.f32.f16 f1, hi16;\n\t"
      "mov.b64 p, {f0, f1};\n\t"
      "mul.rn.f32x2 p, p, %3;\n\t"
      "mov.b64 {f0, f1}, p;\n\t"
      "cvt.rn.bf16x2.f32 b, f1, f0;\n\t"
      "shl.b32 w0, b, 16;\n\t"
      "and.b32 w1, b, -65536;\n\t"
      "mov.b64 %0, {w0, w1};\n\t}"
      : "=l"(r)
      : "r"(byte), "r"(ss), "l"(gg));
  return r;
}

// bf16 pair (one word, element 2i in the low half) -> packed fp32 pair.
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  return pack_f32x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

template <int MR>
__global__ void __launch_bounds__(kW4Threads)
    w4a16_gemv_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                      const uint8_t* __restrict__ w, const uint8_t* __restrict__ ws, int64_t N,
                      const float* __restrict__ g_ptr, const float* __restrict__ bias,
                      uint16_t* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = static_cast<int64_t>(blockIdx.x) * kW4Warps + (threadIdx.x >> 5);
  const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * kW4Warps;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * MR;
  const int64_t chunks = K / 32;        // 32 elements: 16 code bytes, 2 scale bytes
  const int64_t row_code_bytes = K / 2;
  const int64_t row_scale_bytes = K / 16;
  const int64_t tasks = (N + kRows - 1) / kRows;
  const float g = __ldg(g_ptr);
  const uint64_t gg = pack_f32x2(g, g);
  int mr_valid = static_cast<int>(M - m0 < MR ? M - m0 : MR);

  for (int64_t task = warp_global; task < tasks; task += warp_stride) {
    const int64_t n0 = task * kRows;
    uint64_t acc[kRows][MR];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int m = 0; m < MR; ++m) acc[r][m] = 0;

    // software pipeline over this lane's chunks: codes and scales of chunk c + 32
    // are in flight while chunk c is decoded
    uint4 code[kRows];
    uint32_t scl[kRows];
    auto load_chunk = [&](int64_t c, uint4 (&cd)[kRows], uint32_t (&sc)[kRows]) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const int64_t n = n0 + r;
        if (c < chunks && n < N) {
          cd[r] = ld_stream16(w + n * row_code_bytes + c * 16);
          sc[r] = __ldg(reinterpret_cast<const uint16_t*>(ws + n * row_scale_bytes + c * 2));
        } else {
          cd[r] = make_uint4(0, 0, 0, 0);
          sc[r] = 0;
        }
      }
    };
    load_chunk(lane, code, scl);
    for (int64_t c = lane; c < chunks; c += 32) {
      uint4 next_code[kRows];
      uint32_t next_scl[kRows];
      load_chunk(c + 32, next_code, next_scl);
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // 8 elements: k = 32 c + 8 i .. + 8
        // activations of this word for every row of the pass, as fp32 pairs
        uint64_t xv[MR][4];
#pragma unroll
        for (int m = 0; m < MR; ++m) {
          uint4 u = make_uint4(0, 0, 0, 0);
          if (m < mr_valid)
            u = __ldg(reinterpret_cast<const uint4*>(x + (m0 + m) * K + c * 32 + i * 8));
          xv[m][0] = bf16x2_to_f32x2(u.x);
          xv[m][1] = bf16x2_to_f32x2(u.y);
          xv[m][2] = bf16x2_to_f32x2(u.z);
          xv[m][3] = bf16x2_to_f32x2(u.w);
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          const uint32_t word = i == 0 ? code[r].x : i == 1 ? code[r].y : i == 2 ? code[r].z
                                                                                 : code[r].w;
          const uint32_t ss = scale_f16x2((scl[r] >> (8 * (i >> 1))) & 0xFFu);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t wv = w4_decode2(word >> (8 * j), ss, gg);
#pragma unroll
            for (int m = 0; m < MR; ++m) fma_f32x2(acc[r][m], wv, xv[m][j]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        code[r] = next_code[r];
        scl[r] = next_scl[r];
      }
    }

    // lanes -> one sum per (row, activation row); lane r * MR + m writes it
    float out = 0.0f;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        float lo, hi;
        unpack_f32x2(acc[r][m], lo, hi);
        float v = lo + hi;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        if (lane == r * MR + m) out = v;
      }
    }
    if (lane < kRows * MR) {
      const int r = lane / MR, m = lane % MR;
      const int64_t n = n0 + r;
      if (n < N && m < mr_valid) {
        const float v = bias ? out + __ldg(bias + n) : out;
        const __nv_bfloat16 b = __float2bfloat16_rn(v);
        y[(m0 + m) * N + n] = *reinterpret_cast<const uint16_t*>(&b);
      }
    }
  }
}

template <int MR>
cudaError_t launch_mr(const void* x, int64_t M, int64_t K, const uint8_t* w, const uint8_t* ws,
                      int64_t N, const float* g, const float* bias, void* y, cudaStream_t s) {
  static int blocks_per_sm[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_sm = dev < 64 ? blocks_per_sm[dev] : 0;
  if (per_sm == 0) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, w4a16_gemv_kernel<MR>, kW4Threads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    if (dev < 64) blocks_per_sm[dev] = per_sm;
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t tasks = (N + kRows - 1) / kRows;
  const int64_t want = (tasks + kW4Warps - 1) / kW4Warps;
  const int64_t wave = static_cast<int64_t>(sms) * per_sm;
  const int64_t row_passes = (M + MR - 1) / MR;
  // one wave in total over the row passes (at least one CTA per pass)
  int64_t bx = wave / row_passes;
  if (bx < 1) bx = 1;
  if (bx > want) bx = want;
  if (row_passes > 65535) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(row_passes));
  w4a16_gemv_kernel<MR><<<grid, kW4Threads, 0, s>>>(
      static_cast<const uint16_t*>(x), M, K, w, ws, N, g, bias, static_cast<uint16_t*>(y));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a16_linear(const void* x, int64_t M, int64_t K, const uint8_t* w,
                                const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                                const float* bias, void* y, cudaStream_t s) {
  if (M == 1) return launch_mr<1>(x, M, K, w, w_scale, N, weight_scale_2, bias, y, s);
  if (M == 2) return launch_mr<2>(x, M, K, w, w_scale, N, weight_scale_2, bias, y, s);
  if (M <= 4) return launch_mr<4>(x, M, K, w, w_scale, N, weight_scale_2, bias, y, s);
  return launch_mr<8>(x, M, K, w, w_scale, N, weight_scale_2, bias, y, s);
}

}  // namespace ql
