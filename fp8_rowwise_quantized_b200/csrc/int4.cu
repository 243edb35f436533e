// INT4 W4A4 linear: the INT4 variant of the 4-bit layer of "Bringing Nunchaku 4-bit
// Diffusion Inference to Diffusers" (section "Introducing Nunchaku Lite": svdq_w4a4,
// "available in INT4 and NVFP4 variants"), without the low-rank branch. The page
// gives no format; the reading is signed 4-bit codes in [-8, 7] with one fp32 scale
// per 64-element group along K for both operands:
//   scale = RN32(amax / 7); codes = clamp(round-half-even(RN32(x * RN32(1 / scale))),
//   -8, 7); zero scale -> zero codes; element 2j in the low nibble of byte j.
//   Y[m, n] = bf16( sum_g xs[m,g] ws[n,g] sum_{k in g} qx[m,k] qw[n,k] + bias[n] )
//
// How the product runs on B200. tcgen05 has no 4-bit integer kind and applies
// per-block scales only in its block formats (power-of-two or E4M3 scales, the
// NVFP4 path of this library); the group scales here are arbitrary fp32 values.
// Summing each group in integers and scaling it on the CUDA cores costs four fp32
// operations per output and group, more than the whole tensor-core work. Instead the
// scales move into the operands: each INT4 row is dequantized once to f16,
//   hat[r, k] = RN16(RN32(q[r, k] * (s[r, k/64] * 2^-e_r)))   with a row factor 2^e_r,
// e_r = E - 12 for the row's largest group scale m 2^E (m in [0.5, 1)), so every
// value stays below 2^15 and inside the f16 range; then one f16 GEMM on the tensor
// cores (kind::f16, fp32 accumulation) gives Y = bf16(2^(e_m + e_n) sum_k xhat what
// + bias), the row and column factors applied in the epilogue.
// Error: each operand carries one f16 rounding (relative 2^-11; the RN32 before it
// adds at most 2^-24), so each product is within 2^-10 of its exact value, and
// |Y - exact| <= 2^-10 * sum_k |qx xs qw ws| plus the fp32 accumulation's rounding:
// within the linear's tolerance of 1e-3 * sum |x w| by construction, typically far
// below it (the rounding errors have random signs). Groups whose scale is 2^24 times
// smaller than the row's largest fall into f16 subnormals; their absolute error
// stays below 2^-25 * 2^e_r, negligible against the row's large groups.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace ql {
namespace {

// ------------------------------------------------------------------ quantization
// One thread per 64-element group (128 contiguous bytes of x, 32 bytes of codes).
__global__ void __launch_bounds__(256)
int4_quantize_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                     uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int64_t G = K / 64;
  const int64_t total = M * G;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / G, g = i - r * G;
    const uint16_t* xg = x + r * K + g * 64;
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __ldg(reinterpret_cast<const uint4*>(xg) + j);
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, bf16x8_amax(v[j].x, v[j].y, v[j].z, v[j].w));
    const float sc = __fdiv_rn(amax, 7.0f);
    const float inv = sc == 0.0f ? 0.0f : __frcp_rn(sc);
    uint32_t words[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // 8 elements -> one word of 8 nibbles
      const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xv = (e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]);
        int c = __float2int_rn(__fmul_rn(xv, inv));  // round half to even
        c = c < -8 ? -8 : (c > 7 ? 7 : c);
        word |= (static_cast<uint32_t>(c) & 0xFu) << (4 * e);
      }
      words[j] = word;
    }
    uint4* dst = reinterpret_cast<uint4*>(q + r * (K / 2) + g * 32);
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    scale[i] = sc;
  }
}

// ------------------------------------------------------------------ dequantization to f16
constexpr int kI4DqWarps = 8;

// One warp per row: the row factor from the largest group scale, then the row in
// chunks of 256 elements, lane l taking elements 8l .. 8l + 7 of a chunk (4 code
// bytes in, 16 bytes of f16 out: both coalesced across the warp).
__global__ void __launch_bounds__(kI4DqWarps * 32)
int4_dequant_f16_kernel(const uint8_t* __restrict__ q, const float* __restrict__ scale,
                        int64_t rows, int64_t K, uint16_t* __restrict__ out,
                        float* __restrict__ factor) {
  const int lane = threadIdx.x & 31;
  const int64_t groups = K / 64;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * kI4DqWarps + (threadIdx.x >> 5); r < rows;
       r += static_cast<int64_t>(gridDim.x) * kI4DqWarps) {
    const float* srow = scale + r * groups;
    float mx = 0.0f;
    for (int64_t g = lane; g < groups; g += 32) mx = fmaxf(mx, fabsf(__ldg(srow + g)));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    int e = 0;
    if (mx > 0.0f && mx <= 3.4028234663852886e38f) {
      int E;
      frexpf(mx, &E);  // mx = m 2^E, m in [0.5, 1)
      e = E - 12;
    }
    if (lane == 0) factor[r] = ldexpf(1.0f, e);
    const uint8_t* qrow = q + r * (K / 2);
    uint16_t* orow = out + r * K;
    for (int64_t c = 0; c < K; c += 256) {
      const int64_t k0 = c + 8 * lane;
      if (k0 >= K) continue;
      const float sc = ldexpf(__ldg(srow + k0 / 64), -e);  // exact: a power-of-two step
      const uint32_t codes = __ldg(reinterpret_cast<const uint32_t*>(qrow + k0 / 2));
      uint32_t h[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // byte j: elements 2j (low nibble) and 2j + 1
        const int lo = static_cast<int>(codes << (28 - 8 * j)) >> 28;
        const int hi = static_cast<int>(codes << (24 - 8 * j)) >> 28;
        const __half2 p = __floats2half2_rn(__fmul_rn(static_cast<float>(lo), sc),
                                            __fmul_rn(static_cast<float>(hi), sc));
        h[j] = *reinterpret_cast<const uint32_t*>(&p);
      }
      *reinterpret_cast<uint4*>(orow + k0) = make_uint4(h[0], h[1], h[2], h[3]);
    }
  }
}

}  // namespace

cudaError_t launch_int4_quantize(const void* x, int64_t M, int64_t K, uint8_t* q, float* scale,
                                 cudaStream_t s) {
  const int64_t groups = M * (K / 64);
  int64_t blocks = (groups + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  int4_quantize_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      static_cast<const uint16_t*>(x), M, K, q, scale);
  return cudaGetLastError();
}

cudaError_t launch_int4_dequant_f16(const uint8_t* q, const float* scale, int64_t rows, int64_t K,
                                    void* out, float* factor, cudaStream_t s) {
  if (rows <= 0 || K <= 0 || K % 64 != 0) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (rows + kI4DqWarps - 1) / kI4DqWarps;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  if (blocks > cap) blocks = cap;
  int4_dequant_f16_kernel<<<static_cast<unsigned>(blocks), kI4DqWarps * 32, 0, s>>>(
      q, scale, rows, K, static_cast<uint16_t*>(out), factor);
  return cudaGetLastError();
}

}  // namespace ql
