// INT4 W4A4 linear: the INT4 variant of the 4-bit layer of "Bringing Nunchaku 4-bit
// Diffusion Inference to Diffusers" (section "Introducing Nunchaku Lite": svdq_w4a4,
// "available in INT4 and NVFP4 variants"), without the low-rank branch. The page
// gives no format; the reading is signed 4-bit codes in [-8, 7] with one fp32 scale
// per 64-element group along K for both operands:
//   scale = RN32(amax / 7); codes = clamp(round-half-even(RN32(x * RN32(1 / scale))),
//   -8, 7); zero scale -> zero codes; element 2j in the low nibble of byte j.
//   Y[m, n] = bf16( sum_g xs[m,g] ws[n,g] sum_{k in g} qx[m,k] qw[n,k] + bias[n] )
//
// Why this path looks the way it does on B200: the group scales are arbitrary fp32
// values, so each 64-wide group's integer product sum has to be scaled on its own
// before it joins the accumulator. The tcgen05 tensor cores apply per-block scales
// only in the block formats (E2M1 / E4M3 elements with E4M3 or power-of-two scales:
// the NVFP4 path of this library); their integer MMA accumulates a whole K range
// in TMEM. So the INT4 layer runs on warp-level integer MMAs (int32 results in
// registers), one 16 x 8 output block and group at a time, and the CUDA cores
// scale and add each group's sums in fp32 (one integer add and three fp32
// operations per output and group, two outputs per packed fp32 instruction). That
// scaling, not the tensor work, bounds the kernel. The 4-bit warp MMA of the PTX ISA
// is not native on sm_100 (it runs as unpacking plus int8 MMAs, per MMA), so the
// codes are unpacked to int8 once per fragment (four SIMD byte operations per 8
// codes) and fed to int8 MMAs (m16n8k32), two per group.
//
// GEMM layout: a CTA of 8 warps owns a 128 x 128 output tile (warps 2 x 4, each
// 64 x 32: 4 x 4 MMAs per group). Each pipeline stage holds one group: 128 rows of
// activation codes and of weight codes (32 bytes each, padded to 48-byte rows so
// that the 8-byte fragment loads of a warp hit distinct banks) and the 128 + 128
// group scales, filled by cp.async (zero fill outside M / N). The MMA's k slots
// are permuted the same way in both operands (lane t of a quad owns elements
// 16t .. 16t+15 of the group across the group's two MMAs), which leaves each group's
// sum unchanged and lets a lane read 8 contiguous bytes per row.
// The int32 sums (|sum| <= 4096) become fp32 exactly through the 1.5 * 2^23 magic
// number (an integer add and a float subtract, no conversion instruction).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace ql {
namespace {

constexpr int kI4Threads = 256;
constexpr int kI4Tile = 128;       // output rows and columns per CTA
constexpr int kI4Row = 48;         // shared-memory bytes per operand row (32 + 16 pad)
constexpr int kI4Stages = 6;
constexpr int kI4StageBytes = 2 * kI4Tile * kI4Row + 2 * kI4Tile * 4;  // A, B, sx, sw

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

// ------------------------------------------------------------------ GEMM
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// d = a * b + c on int8 operands (m16n8k32, int32 accumulation).
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1, const int (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%10, %11, %12, %13};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]), "r"(c[2]),
        "r"(c[3]));
}

// Eight signed 4-bit codes (one word, element i in nibble i) -> int8: the even
// elements in the bytes of `even`, the odd ones in `odd` (per byte: (v ^ 8) - 8).
__device__ __forceinline__ void s4x8_to_s8(uint32_t w, uint32_t& even, uint32_t& odd) {
  even = __vsub4((w & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);
  odd = __vsub4(((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);
}

// exact int32 -> fp32 for |v| < 2^22: the bits of 1.5 * 2^23 + v, minus 1.5 * 2^23
__device__ __forceinline__ uint32_t small_int_bits(int v) {
  return static_cast<uint32_t>(v + 0x4B400000);
}

// acc.{x,y} += ((bits.{x,y} - 1.5 * 2^23) * sw.{x,y}) * sx, two lanes per packed op
// (each lane: one subtraction, one multiply, one fma, all RN)
__device__ __forceinline__ void scale_add2(float& a0, float& a1, uint32_t b0, uint32_t b1,
                                           float sw0, float sw1, float sx) {
  asm("{\n\t.reg .b64 f, m, w, x, acc;\n\t"
      "mov.b64 f, {%2, %3};\n\t"
      "mov.b64 m, {0f4B400000, 0f4B400000};\n\t"
      "sub.rn.f32x2 f, f, m;\n\t"
      "mov.b64 w, {%4, %5};\n\t"
      "mul.rn.f32x2 f, f, w;\n\t"
      "mov.b64 x, {%6, %6};\n\t"
      "mov.b64 acc, {%0, %1};\n\t"
      "fma.rn.f32x2 acc, f, x, acc;\n\t"
      "mov.b64 {%0, %1}, acc;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(b0), "r"(b1), "f"(sw0), "f"(sw1), "f"(sx));
}

__global__ void __launch_bounds__(kI4Threads, 1)
int4_gemm_kernel(const uint8_t* __restrict__ xq, const float* __restrict__ xs, int64_t M,
                 int64_t K, const uint8_t* __restrict__ wq, const float* __restrict__ ws,
                 int64_t N, const float* __restrict__ bias, uint16_t* __restrict__ y) {
  extern __shared__ __align__(128) uint8_t i4_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, t = lane & 3;
  const int warp_m = warp >> 2, warp_n = warp & 3;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kI4Tile;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kI4Tile;
  const int64_t G = K / 64;
  const int64_t row_bytes = K / 2;
  const uint32_t smem = smem_u32(i4_smem);

  // this thread's copies: 16 bytes of A and of B (row tid / 2, half tid % 2), one scale
  const int crow = tid >> 1, chalf = tid & 1;
  const bool a_ok = m0 + crow < M, b_ok = n0 + crow < N;
  const uint8_t* a_src = xq + (a_ok ? (m0 + crow) : 0) * row_bytes + chalf * 16;
  const uint8_t* b_src = wq + (b_ok ? (n0 + crow) : 0) * row_bytes + chalf * 16;
  const bool s_is_a = tid < kI4Tile;
  const int srow = tid & (kI4Tile - 1);
  const bool s_ok = s_is_a ? (m0 + srow < M) : (n0 + srow < N);
  const float* s_src = s_is_a ? xs + (s_ok ? (m0 + srow) : 0) * G : ws + (s_ok ? (n0 + srow) : 0) * G;

  auto load_stage = [&](int stage, int64_t g) {
    const uint32_t base = smem + stage * kI4StageBytes;
    const uint32_t a_dst = base + crow * kI4Row + chalf * 16;
    const uint32_t b_dst = base + kI4Tile * kI4Row + crow * kI4Row + chalf * 16;
    const uint32_t s_dst = base + 2 * kI4Tile * kI4Row + (s_is_a ? 0 : kI4Tile * 4) + srow * 4;
    cp_async16(a_dst, a_src + g * 32, a_ok);
    cp_async16(b_dst, b_src + g * 32, b_ok);
    cp_async4(s_dst, s_src + g, s_ok);
  };

  float acc[4][4][4];
#pragma unroll
  for (int mi = 0; mi < 4; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mi][ni][e] = 0.0f;

#pragma unroll
  for (int s = 0; s < kI4Stages - 1; ++s) {
    if (s < G) load_stage(s, s);
    cp_async_commit();
  }
  for (int64_t g = 0; g < G; ++g) {
    cp_async_wait<kI4Stages - 2>();
    __syncthreads();  // stage g landed for every thread; stage g - 1 is free
    {
      const int64_t gn = g + kI4Stages - 1;
      if (gn < G) load_stage(static_cast<int>(gn % kI4Stages), gn);
      cp_async_commit();
    }
    const uint8_t* st = i4_smem + (g % kI4Stages) * kI4StageBytes;
    const uint8_t* a_s = st;
    const uint8_t* b_s = st + kI4Tile * kI4Row;
    const float* sx_s = reinterpret_cast<const float*>(st + 2 * kI4Tile * kI4Row);
    const float* sw_s = sx_s + kI4Tile;
    // operands unpacked once to int8: for each row (A) or column (B) of the warp tile,
    // the lane's 16 codes (elements 16t .. 16t+15 of the group) as [even, odd] bytes
    // of words 0 and 1 of its 8 bytes; MMA 0 takes word 0, MMA 1 word 1, and in both
    // the even bytes fill k slots 4t .. 4t+3 and the odd ones 16+4t .. 16+4t+3, in A
    // and B alike (so each group's sum is unchanged)
    uint32_t af[4][2][4], bf[4][2][2];
    float sx[4][2], sw[4][2];
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) {
      const int r = warp_m * 64 + mi * 16 + gq;
      const uint2 lo = *reinterpret_cast<const uint2*>(a_s + r * kI4Row + 8 * t);
      const uint2 hi = *reinterpret_cast<const uint2*>(a_s + (r + 8) * kI4Row + 8 * t);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        s4x8_to_s8(h == 0 ? lo.x : lo.y, af[mi][h][0], af[mi][h][2]);
        s4x8_to_s8(h == 0 ? hi.x : hi.y, af[mi][h][1], af[mi][h][3]);
      }
      sx[mi][0] = sx_s[r];
      sx[mi][1] = sx_s[r + 8];
    }
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
      const int c = warp_n * 32 + ni * 8 + gq;
      const uint2 bv = *reinterpret_cast<const uint2*>(b_s + c * kI4Row + 8 * t);
      s4x8_to_s8(bv.x, bf[ni][0][0], bf[ni][0][1]);
      s4x8_to_s8(bv.y, bf[ni][1][0], bf[ni][1][1]);
      const int oc = warp_n * 32 + ni * 8 + 2 * t;
      sw[ni][0] = sw_s[oc];
      sw[ni][1] = sw_s[oc + 1];
    }
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) {
#pragma unroll
      for (int ni = 0; ni < 4; ++ni) {
        const int zero[4] = {0, 0, 0, 0};
        int d0[4], d[4];
        mma_s8(d0, af[mi][0][0], af[mi][0][1], af[mi][0][2], af[mi][0][3], bf[ni][0][0],
               bf[ni][0][1], zero);
        mma_s8(d, af[mi][1][0], af[mi][1][1], af[mi][1][2], af[mi][1][3], bf[ni][1][0],
               bf[ni][1][1], d0);
        // outputs (row gq, col 2t), (gq, 2t+1), (gq+8, 2t), (gq+8, 2t+1)
        scale_add2(acc[mi][ni][0], acc[mi][ni][1], small_int_bits(d[0]), small_int_bits(d[1]),
                   sw[ni][0], sw[ni][1], sx[mi][0]);
        scale_add2(acc[mi][ni][2], acc[mi][ni][3], small_int_bits(d[2]), small_int_bits(d[3]),
                   sw[ni][0], sw[ni][1], sx[mi][1]);
      }
    }
  }
  cp_async_wait<0>();

  // epilogue: + bias, RN to bf16
#pragma unroll
  for (int mi = 0; mi < 4; ++mi) {
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t m = m0 + warp_m * 64 + mi * 16 + gq + (e >> 1) * 8;
        const int64_t n = n0 + warp_n * 32 + ni * 8 + 2 * t + (e & 1);
        if (m < M && n < N) {
          const float v = bias ? acc[mi][ni][e] + __ldg(bias + n) : acc[mi][ni][e];
          const __nv_bfloat16 b = __float2bfloat16_rn(v);
          y[m * N + n] = *reinterpret_cast<const uint16_t*>(&b);
        }
      }
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

cudaError_t launch_int4_gemm(const uint8_t* xq, const float* xs, int64_t M, int64_t K,
                             const uint8_t* wq, const float* ws, int64_t N, const float* bias,
                             void* y, cudaStream_t s) {
  static int configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int smem = kI4Stages * kI4StageBytes;
  if (dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(int4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured[dev] = 1;
  }
  const int64_t tm = (M + kI4Tile - 1) / kI4Tile, tn = (N + kI4Tile - 1) / kI4Tile;
  if (tm > 65535) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(tn), static_cast<unsigned>(tm));
  int4_gemm_kernel<<<grid, kI4Threads, smem, s>>>(xq, xs, M, K, wq, ws, N, bias,
                                                  static_cast<uint16_t*>(y));
  return cudaGetLastError();
}

}  // namespace ql
