// Quantization kernels (HBM-bound):
//   * NVFP4 activation / weight quantization (packed E2M1 codes + E4M3 block
//     scales through a global fp32 scale), with the scales written either
//     row-major (public layout) or straight into the tensor-core scale layout;
//   * re-layout of row-major weight block scales into the tensor-core layout;
//   * FP8 row-wise quantization (E4M3 codes + one fp32 scale per row);
//   * calibration reduction amax / (6 * 448);
//   * element encoder diagnostics.
// The scheme is the one of the Diffusers page "BFL (fp8r / nvfp4)" (scheme list:
// nvfp4 and fp8r entries; "Kernels" table: run-time activation quantization).
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "layout.cuh"
#include "ptx.cuh"

namespace ql {

namespace {

constexpr int kQuantThreads = 256;

// 16-byte read-only load of 8 bf16 values.
__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Quantize one 16-element block held as 8 packed bf16 pairs. Returns the E4M3
// scale code in *scale_code and the 8 packed code bytes in (lo, hi).
// Arithmetic (each step one fp32 rounding): sf = amax * c; s = E4M3(sf);
// d = value(s) * g; d == 0 -> zero codes; else codes = E2M1(x * (1/d)).
__device__ __forceinline__ void nvfp4_block(const uint32_t (&w)[8], float c, float g,
                                            uint32_t* scale_code, uint32_t* lo, uint32_t* hi) {
  float v[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_lo(w[i]);
    v[2 * i + 1] = bf16_hi(w[i]);
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float sf = __fmul_rn(amax, c);
  const uint32_t s = cvt_e4m3x4(sf, 0.0f, 0.0f, 0.0f) & 0xFFu;
  const float d = __fmul_rn(e4m3_positive_value(s), g);
  *scale_code = s;
  if (d == 0.0f) {
    *lo = 0u;
    *hi = 0u;
    return;
  }
  const float inv = __frcp_rn(d);
  float a[8], b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    a[i] = __fmul_rn(v[i], inv);
    b[i] = __fmul_rn(v[8 + i], inv);
  }
  *lo = cvt_e2m1x8(a);
  *hi = cvt_e2m1x8(b);
}

// One thread per (row r, 64-element group kg): up to 4 blocks of 16.
//   x  bf16 [M, K]; xq uint8 [M, K/2]
//   SF_MMA == false: xs uint8 [M, K/16] row-major
//   SF_MMA == true:  xs in the atom layout for rows padded to 128 and K groups
//                    padded to whole K tiles (padding written as zero)
template <bool SF_MMA>
__device__ __forceinline__ void nvfp4_quantize_group(int64_t idx, const uint16_t* __restrict__ x,
                                                     int64_t M, int64_t K,
                                                     const float* __restrict__ g_ptr,
                                                     uint8_t* __restrict__ xq,
                                                     uint8_t* __restrict__ xs, int64_t rows_total,
                                                     int64_t kg_total) {
  if (idx >= rows_total * kg_total) return;
  const int64_t r = idx / kg_total;
  const int64_t kg = idx % kg_total;
  const int64_t nblk = K / 16;
  const float g = __ldg(g_ptr);
  const float c = __frcp_rn(__fmul_rn(6.0f, g));

  int nb = 0;  // valid 16-blocks in this group
  if (r < M && 4 * kg < nblk) nb = (nblk - 4 * kg >= 4) ? 4 : static_cast<int>(nblk - 4 * kg);

  uint32_t scales[4] = {0u, 0u, 0u, 0u};
  if (nb > 0) {
    const uint16_t* xr = x + r * K + kg * 64;
    uint8_t* qr = xq + r * (K / 2) + kg * 32;
    uint4 raw[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b < nb) {
        raw[2 * b] = ldg16(xr + b * 16);
        raw[2 * b + 1] = ldg16(xr + b * 16 + 8);
      }
    }
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b < nb) {
        const uint32_t w[8] = {raw[2 * b].x, raw[2 * b].y, raw[2 * b].z, raw[2 * b].w,
                               raw[2 * b + 1].x, raw[2 * b + 1].y, raw[2 * b + 1].z,
                               raw[2 * b + 1].w};
        uint32_t lo, hi;
        nvfp4_block(w, c, g, &scales[b], &lo, &hi);
        *reinterpret_cast<uint2*>(qr + b * 8) = make_uint2(lo, hi);
      }
    }
  }
  const uint32_t word = scales[0] | (scales[1] << 8) | (scales[2] << 16) | (scales[3] << 24);
  if (SF_MMA) {
    *reinterpret_cast<uint32_t*>(xs + sf_act_word_offset(r, kg, kg_total)) = word;
  } else if (nb > 0) {
    uint8_t* sr = xs + r * nblk + kg * 4;
    if (nb == 4 && (reinterpret_cast<uintptr_t>(sr) & 3) == 0) {
      *reinterpret_cast<uint32_t*>(sr) = word;
    } else {
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (b < nb) sr[b] = static_cast<uint8_t>(scales[b]);
    }
  }
}

template <bool SF_MMA>
__global__ void __launch_bounds__(kQuantThreads)
nvfp4_quantize_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                      const float* __restrict__ g_ptr, uint8_t* __restrict__ xq,
                      uint8_t* __restrict__ xs, int64_t rows_total, int64_t kg_total) {
  nvfp4_quantize_group<SF_MMA>(static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x, x, M,
                               K, g_ptr, xq, xs, rows_total, kg_total);
}

// Row-major weight scales [N, K/16] -> atom layout for tiles of `bn` rows.
// One thread per (tile, row slot nn < na*128, group kg).
__device__ __forceinline__ void nvfp4_weight_scale_word(int64_t idx, const uint8_t* __restrict__ ws,
                                                        int64_t N, int64_t K, int bn, int na,
                                                        int64_t n_tiles, int64_t KG,
                                                        uint8_t* __restrict__ out) {
  const int64_t slots = static_cast<int64_t>(na) * 128;
  if (idx >= n_tiles * slots * KG) return;
  const int64_t kg = idx % KG;
  const int64_t nn = (idx / KG) % slots;
  const int64_t t = idx / (KG * slots);
  const int64_t n = t * bn + nn;
  const int64_t nblk = K / 16;
  uint32_t word = 0;
  if (nn < bn && n < N) {
    const uint8_t* src = ws + n * nblk + kg * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (4 * kg + j < nblk) word |= static_cast<uint32_t>(__ldg(src + j)) << (8 * j);
  }
  *reinterpret_cast<uint32_t*>(out + sf_wgt_word_offset(t, nn, kg, KG, na)) = word;
}

// The prologue of nvfp4_linear in one launch: blocks [0, act_blocks) quantize the
// activations into the workspace (codes row-major, scales in atom layout), the
// remaining blocks lay out the weight scales for the GEMM's tile width. It lets
// the dependent GEMM launch start its set-up right away; the GEMM reads the
// workspace only after this grid has completed.
__global__ void __launch_bounds__(kQuantThreads)
nvfp4_prologue_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                      const float* __restrict__ g_ptr, uint8_t* __restrict__ xq,
                      uint8_t* __restrict__ xs, int64_t rows_total, int64_t KG,
                      int64_t act_blocks, const uint8_t* __restrict__ ws, int64_t N, int bn,
                      int na, int64_t n_tiles, uint8_t* __restrict__ wout) {
  grid_dependents_launch();
  if (blockIdx.x < act_blocks) {
    nvfp4_quantize_group<true>(static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x, x, M,
                               K, g_ptr, xq, xs, rows_total, KG);
  } else {
    nvfp4_weight_scale_word((static_cast<int64_t>(blockIdx.x) - act_blocks) * blockDim.x +
                                threadIdx.x,
                            ws, N, K, bn, na, n_tiles, KG, wout);
  }
}

// FP8 row-wise: one warp per row; pass 1 takes the row amax, pass 2 encodes.
//   scale = amax / 448 (fp32 division); scale == 0 -> zero codes;
//   else codes = E4M3(x * (1/scale)).  Requires K % 8 == 0.
__global__ void __launch_bounds__(kQuantThreads)
fp8r_quantize_rows_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                          uint8_t* __restrict__ xq, float* __restrict__ x_scale) {
  grid_dependents_launch();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= M) return;
  const uint16_t* xr = x + row * K;
  const int64_t chunks = K / 8;
  float amax = 0.0f;
  for (int64_t ch = lane; ch < chunks; ch += 32) {
    const uint4 u = ldg16(xr + ch * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = __fdiv_rn(amax, 448.0f);
  if (lane == 0) x_scale[row] = scale;
  uint8_t* qr = xq + row * K;
  if (scale == 0.0f) {
    for (int64_t ch = lane; ch < chunks; ch += 32)
      *reinterpret_cast<uint2*>(qr + ch * 8) = make_uint2(0u, 0u);
    return;
  }
  const float inv = __frcp_rn(scale);
  for (int64_t ch = lane; ch < chunks; ch += 32) {
    const uint4 u = ldg16(xr + ch * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    const uint32_t lo = cvt_e4m3x4(__fmul_rn(bf16_lo(w[0]), inv), __fmul_rn(bf16_hi(w[0]), inv),
                                   __fmul_rn(bf16_lo(w[1]), inv), __fmul_rn(bf16_hi(w[1]), inv));
    const uint32_t hi = cvt_e4m3x4(__fmul_rn(bf16_lo(w[2]), inv), __fmul_rn(bf16_hi(w[2]), inv),
                                   __fmul_rn(bf16_lo(w[3]), inv), __fmul_rn(bf16_hi(w[3]), inv));
    *reinterpret_cast<uint2*>(qr + ch * 8) = make_uint2(lo, hi);
  }
}

// amax(|x|) over n bf16 values into *slot (as the bit pattern of a non-negative
// float, so unsigned max orders it); slot must start at 0.
__global__ void __launch_bounds__(kQuantThreads)
amax_bf16_kernel(const uint16_t* __restrict__ x, int64_t n, unsigned int* slot) {
  float m = 0.0f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    m = fmaxf(m, fabsf(__uint_as_float(static_cast<uint32_t>(x[i]) << 16)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (threadIdx.x % 32 == 0) atomicMax(slot, __float_as_uint(m));
}

__global__ void zero_word_kernel(unsigned int* slot) { *slot = 0u; }

__global__ void global_scale_finish_kernel(float* out) {
  const float amax = __uint_as_float(*reinterpret_cast<unsigned int*>(out));
  *out = __fdiv_rn(amax, 2688.0f);
}

__global__ void encode_kernel(const float* __restrict__ in, uint8_t* __restrict__ out, int64_t n,
                              int fp4) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = in[i];
  if (fp4) {
    const float a[8] = {v, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    out[i] = static_cast<uint8_t>(cvt_e2m1x8(a) & 0xFu);
  } else {
    out[i] = static_cast<uint8_t>(cvt_e4m3x4(v, 0.f, 0.f, 0.f) & 0xFFu);
  }
}

inline unsigned grid_for(int64_t work, int threads) {
  return static_cast<unsigned>((work + threads - 1) / threads);
}

}  // namespace

cudaError_t launch_nvfp4_quantize_rowmajor(const void* x, int64_t M, int64_t K, const float* g,
                                           uint8_t* xq, uint8_t* xs, cudaStream_t s) {
  const int64_t kg_total = ceil_div64(K, 64);
  nvfp4_quantize_kernel<false><<<grid_for(M * kg_total, kQuantThreads), kQuantThreads, 0, s>>>(
      static_cast<const uint16_t*>(x), M, K, g, xq, xs, M, kg_total);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_prologue(const void* x, int64_t M, int64_t K, const uint8_t* w_scale,
                                  int64_t N, int bn, const float* input_scale, uint8_t* workspace,
                                  cudaStream_t s) {
  const Nvfp4Workspace L = nvfp4_workspace(M, K, N, bn);
  const int64_t KG = sf_kgroups(K);
  const int64_t rows = ceil_div64(M, 128) * 128;
  const int na = (bn + 127) / 128;
  const int64_t n_tiles = ceil_div64(N, bn);
  const int64_t act_blocks = grid_for(rows * KG, kQuantThreads);
  const int64_t w_blocks = grid_for(n_tiles * na * 128 * KG, kQuantThreads);
  nvfp4_prologue_kernel<<<static_cast<unsigned>(act_blocks + w_blocks), kQuantThreads, 0, s>>>(
      static_cast<const uint16_t*>(x), M, K, input_scale, workspace + L.codes_off,
      workspace + L.act_sf_off, rows, KG, act_blocks, w_scale, N, bn, na, n_tiles,
      workspace + L.wgt_sf_off);
  return cudaGetLastError();
}

cudaError_t launch_fp8r_quantize_rows(const void* x, int64_t M, int64_t K, uint8_t* xq,
                                      float* x_scale, cudaStream_t s) {
  const int rows_per_block = kQuantThreads / 32;
  fp8r_quantize_rows_kernel<<<grid_for(M, rows_per_block), kQuantThreads, 0, s>>>(
      static_cast<const uint16_t*>(x), M, K, xq, x_scale);
  return cudaGetLastError();
}

cudaError_t launch_global_scale(const void* x, int64_t n, float* out, cudaStream_t s) {
  unsigned int* slot = reinterpret_cast<unsigned int*>(out);
  zero_word_kernel<<<1, 1, 0, s>>>(slot);
  const int64_t want = grid_for(n, kQuantThreads);
  const int64_t blocks = want < 148 * 8 ? want : 148 * 8;
  amax_bf16_kernel<<<static_cast<unsigned>(blocks), kQuantThreads, 0, s>>>(
      static_cast<const uint16_t*>(x), n, slot);
  global_scale_finish_kernel<<<1, 1, 0, s>>>(out);
  return cudaGetLastError();
}

cudaError_t launch_encode(const float* in, uint8_t* out, int64_t n, bool fp4, cudaStream_t s) {
  encode_kernel<<<grid_for(n, kQuantThreads), kQuantThreads, 0, s>>>(in, out, n, fp4 ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace ql
