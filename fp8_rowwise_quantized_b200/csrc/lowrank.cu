// Low-rank down projection of the SVDQuant-style NVFP4 linear ("Bringing Nunchaku
// 4-bit Diffusion Inference to Diffusers", section "Background: SVDQuant and
// Nunchaku": a small 16-bit low-rank branch next to the 4-bit residual):
//   D[m, j] = sum_k xs[m, k] * down[j, k],   xs = bf16(RN32(x * smooth)), j < rank,
// written as lr_act[m, j] = bf16(D[m, j] / alpha), alpha = input_scale *
// weight_scale_2: the form the GEMM's low-rank K step reads (it multiplies the
// whole accumulator by alpha).
//
// A [M, K] x [K, rank] product with rank <= 64: one block of 8 warps per 16 rows,
// each warp a K range, on the warp-level bf16 tensor-core MMA (m16n8k16, fp32
// accumulation); the 8 partial sums are added in a fixed order in shared memory,
// so the result does not depend on scheduling.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"

namespace ql {

namespace {

constexpr int kLrWarps = 8;

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&c)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Columns k .. k+7 of one row (16 bytes), smoothed (bf16(RN32(x * smooth))), as 4
// bf16x2 pairs.
__device__ __forceinline__ uint4 smoothed8(const uint16_t* __restrict__ row,
                                           const float* __restrict__ smooth, int k, bool valid) {
  if (!valid) return make_uint4(0u, 0u, 0u, 0u);
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>(row + k));
  if (!smooth) return raw;
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(smooth + k));
  const float4 s1 = __ldg(reinterpret_cast<const float4*>(smooth + k + 4));
  const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 p =
        __floats2bfloat162_rn(__fmul_rn(__uint_as_float(w[i] << 16), sv[2 * i]),
                              __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), sv[2 * i + 1]));
    o[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// NB blocks of 8 output columns (rank = 8 NB). Fragment layout of m16n8k16 (row.col):
// thread (g = lane / 4, t = lane % 4) holds A[g][2t..], A[g+8][2t..], A[g][2t+8..],
// A[g+8][2t+8..], B[2t..][g], B[2t+8..][g] and C[g][2t..2t+1], C[g+8][2t..2t+1].
// A sum over k may take its terms in any order, so A and B use the same permutation
// of each 32-column chunk: thread t's slots of the first MMA are columns 8t .. 8t+3
// and of the second 8t+4 .. 8t+7, i.e. one 16-byte load per row (and per row of
// down) feeds two MMAs.
template <int NB>
__global__ void __launch_bounds__(32 * kLrWarps)
lowrank_down_kernel(const uint16_t* __restrict__ x, int M, int K, const float* __restrict__ smooth,
                    const uint16_t* __restrict__ down, const float* __restrict__ scale_a,
                    const float* __restrict__ scale_b, uint16_t* __restrict__ out) {
  constexpr int R = 8 * NB;
  __shared__ float part[kLrWarps][16][R + 1];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane / 4, t = lane % 4;
  const int row0 = blockIdx.x * 16;
  const int ksteps = K / 16;                                        // even: K % 32 == 0
  const int per = 2 * ((ksteps + 2 * kLrWarps - 1) / (2 * kLrWarps));  // even
  const int s0 = warp * per;
  const int s1 = min(ksteps, s0 + per);
  const bool va = row0 + g < M, vb = row0 + g + 8 < M;
  const uint16_t* xa = x + static_cast<int64_t>(va ? row0 + g : 0) * K;
  const uint16_t* xb = x + static_cast<int64_t>(vb ? row0 + g + 8 : 0) * K;
  float c[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0.0f;
#pragma unroll 2
  for (int st = s0; st < s1; st += 2) {
    const int k = st * 16 + 8 * t;
    const uint4 ua = smoothed8(xa, smooth, k, va);
    const uint4 ub = smoothed8(xb, smooth, k, vb);
    const uint32_t a0[4] = {ua.x, ub.x, ua.y, ub.y};
    const uint32_t a1[4] = {ua.z, ub.z, ua.w, ub.w};
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const uint4 d = __ldg(reinterpret_cast<const uint4*>(down + static_cast<int64_t>(8 * nb + g) * K + k));
      mma_m16n8k16_bf16(c[nb], a0, d.x, d.y);
      mma_m16n8k16_bf16(c[nb], a1, d.z, d.w);
    }
  }
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    part[warp][g][8 * nb + 2 * t] = c[nb][0];
    part[warp][g][8 * nb + 2 * t + 1] = c[nb][1];
    part[warp][g + 8][8 * nb + 2 * t] = c[nb][2];
    part[warp][g + 8][8 * nb + 2 * t + 1] = c[nb][3];
  }
  __syncthreads();
  const float alpha = __fmul_rn(__ldg(scale_a), __ldg(scale_b));
  for (int i = threadIdx.x; i < 16 * R; i += blockDim.x) {
    const int rr = i / R, j = i - (i / R) * R;
    float d = 0.0f;
#pragma unroll
    for (int w = 0; w < kLrWarps; ++w) d = __fadd_rn(d, part[w][rr][j]);  // fixed order
    if (row0 + rr < M) {
      const __nv_bfloat16 h = __float2bfloat16_rn(__fdiv_rn(d, alpha));
      out[static_cast<int64_t>(row0 + rr) * R + j] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

}  // namespace

cudaError_t launch_lowrank_down(const void* x, int64_t M, int64_t K, const float* smooth,
                                const void* down, int rank, const float* scale_a,
                                const float* scale_b, void* out, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>((M + 15) / 16));
  const dim3 block(32 * kLrWarps);
  const auto* xx = static_cast<const uint16_t*>(x);
  const auto* dd = static_cast<const uint16_t*>(down);
  auto* oo = static_cast<uint16_t*>(out);
  const int m = static_cast<int>(M), k = static_cast<int>(K);
#define QL_LR(NB_)                                                                    \
  case NB_:                                                                           \
    lowrank_down_kernel<NB_><<<grid, block, 0, s>>>(xx, m, k, smooth, dd, scale_a, scale_b, oo); \
    break;
  switch (rank / 8) {
    QL_LR(1)
    QL_LR(2)
    QL_LR(3)
    QL_LR(4)
    QL_LR(5)
    QL_LR(6)
    QL_LR(7)
    QL_LR(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef QL_LR
  return cudaGetLastError();
}

}  // namespace ql
