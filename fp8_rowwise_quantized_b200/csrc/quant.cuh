// Device building blocks shared by the quantization kernels: the NVFP4 rule for one
// 16-element block, the SVDQuant smoothing of 8 values and the re-layout of
// row-major weight block scales into the tensor-core atom layout.
// The scheme is the one of the Diffusers page "BFL (fp8r / nvfp4)" (scheme list:
// nvfp4 entry); the smoothing is the one of "Bringing Nunchaku 4-bit Diffusion
// Inference to Diffusers" (section "Background: SVDQuant and Nunchaku").
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "layout.cuh"
#include "ptx.cuh"

namespace ql {

// SVDQuant smoothing of 8 bf16 values: bf16(RN32(x * smooth)), with s0, s1 the 8
// fp32 multipliers of their columns.
__device__ __forceinline__ uint4 smooth8(const uint4 u, const float4 s0, const float4 s1) {
  const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(__fmul_rn(bf16_lo(w[i]), sv[2 * i]),
                                                   __fmul_rn(bf16_hi(w[i]), sv[2 * i + 1]));
    o[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Eight bf16 values (four packed words, element 2i in the low half of word i) times
// `inv`: each product rounded to fp32 (two lanes per packed multiply), then to E2M1
// (RN, satfinite); element i in bits 4i+3 .. 4i of the result.
__device__ __forceinline__ uint32_t e2m1x8_of_bf16_scaled(uint32_t w0, uint32_t w1, uint32_t w2,
                                                          uint32_t w3, float inv) {
  uint32_t r;
  asm("{\n\t"
      ".reg .b32 l0, l1, l2, l3, h0, h1, h2, h3;\n\t"
      ".reg .b64 p0, p1, p2, p3, q;\n\t"
      ".reg .b8 c0, c1, c2, c3;\n\t"
      "mov.b64 q, {%5, %5};\n\t"
      "shl.b32 l0, %1, 16;\n\t"
      "and.b32 h0, %1, -65536;\n\t"
      "shl.b32 l1, %2, 16;\n\t"
      "and.b32 h1, %2, -65536;\n\t"
      "shl.b32 l2, %3, 16;\n\t"
      "and.b32 h2, %3, -65536;\n\t"
      "shl.b32 l3, %4, 16;\n\t"
      "and.b32 h3, %4, -65536;\n\t"
      "mov.b64 p0, {l0, h0};\n\t"
      "mov.b64 p1, {l1, h1};\n\t"
      "mov.b64 p2, {l2, h2};\n\t"
      "mov.b64 p3, {l3, h3};\n\t"
      "mul.rn.f32x2 p0, p0, q;\n\t"
      "mul.rn.f32x2 p1, p1, q;\n\t"
      "mul.rn.f32x2 p2, p2, q;\n\t"
      "mul.rn.f32x2 p3, p3, q;\n\t"
      "mov.b64 {l0, h0}, p0;\n\t"
      "mov.b64 {l1, h1}, p1;\n\t"
      "mov.b64 {l2, h2}, p2;\n\t"
      "mov.b64 {l3, h3}, p3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, h0, l0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, h1, l1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, h2, l2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, h3, l3;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(r)
      : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "f"(inv));
  return r;
}

// Largest magnitude of 16 bf16 values (8 packed words) as an fp32 value: sign bits
// cleared, unsigned 16-bit maxima (non-negative floats order like their bit
// patterns), then the larger half.
__device__ __forceinline__ float bf16x16_amax(const uint4 u, const uint4 v) {
  constexpr uint32_t kAbs = 0x7FFF7FFFu;
  uint32_t m = __vmaxu2(__vmaxu2(__vmaxu2(u.x & kAbs, u.y & kAbs), __vmaxu2(u.z & kAbs, u.w & kAbs)),
                        __vmaxu2(__vmaxu2(v.x & kAbs, v.y & kAbs), __vmaxu2(v.z & kAbs, v.w & kAbs)));
  m = __vmaxu2(m, m >> 16);  // low half: the larger of the two halves
  return __uint_as_float(m << 16);
}

// NVFP4 of one 16-element block held as two groups of 8 bf16 values (u: elements
// 0..7, v: 8..15), with g the global scale and c = RN(1/RN(6 g)):
//   s = E4M3(RN(amax * c)), d = RN(val(s) * g),
//   codes = E2M1(RN(x * RN(1/d))), all zero when d == 0.
// Returns the 16 codes (element 2j in the low nibble of byte j) and the scale code.
// Branch-free: for d == 0 the codes are computed from an infinite reciprocal and
// then replaced by zeros.
__device__ __forceinline__ uint2 nvfp4_block16(const uint4 u, const uint4 v, float g, float c,
                                               uint32_t& scale_code) {
  const float amax = bf16x16_amax(u, v);
  const uint32_t s = cvt_e4m3x2(0.0f, __fmul_rn(amax, c)) & 0xFFu;
  scale_code = s;
  const float d = __fmul_rn(e4m3_to_float(s), g);
  const float inv = __frcp_rn(d);
  const uint32_t lo = e2m1x8_of_bf16_scaled(u.x, u.y, u.z, u.w, inv);
  const uint32_t hi = e2m1x8_of_bf16_scaled(v.x, v.y, v.z, v.w, inv);
  const bool zero = d == 0.0f;
  return make_uint2(zero ? 0u : lo, zero ? 0u : hi);
}

// The same block rule with the per-block reciprocal read from a table: inv_of[s] =
// RN32(1 / RN32(value(s) * g)) for the 128 non-negative scale codes s (0 where
// value(s) * g == 0), computed once per CTA with the same operations, so the codes
// are the same bits as nvfp4_block16's.
__device__ __forceinline__ uint2 nvfp4_block16_tab(const uint4 u, const uint4 v, float c,
                                                   const float* inv_of, uint32_t& scale_code) {
  const float amax = bf16x16_amax(u, v);
  const uint32_t s = cvt_e4m3x2(0.0f, __fmul_rn(amax, c)) & 0x7Fu;  // amax >= 0: sign bit 0
  scale_code = s;
  const float inv = inv_of[s];
  const uint32_t lo = e2m1x8_of_bf16_scaled(u.x, u.y, u.z, u.w, inv);
  const uint32_t hi = e2m1x8_of_bf16_scaled(v.x, v.y, v.z, v.w, inv);
  const bool zero = inv == 0.0f;
  return make_uint2(zero ? 0u : lo, zero ? 0u : hi);
}

// Fills inv_of[0..127] for global scale g (threads 0..127 of the block, one entry
// each); the caller synchronises the block before use.
__device__ __forceinline__ void fill_block_reciprocals(float* inv_of, float g, int tid) {
  if (tid < 128) {
    const float d = __fmul_rn(e4m3_to_float(static_cast<uint32_t>(tid)), g);
    inv_of[tid] = d != 0.0f ? __frcp_rn(d) : 0.0f;
  }
}

// Row-major weight scales [N, K/16] -> atom layout for tiles of `bn` rows, through
// shared memory so that both the reads (64 contiguous bytes per row) and the
// writes (whole 512-byte atoms) are coalesced. One job = (tile, 128-row atom a,
// kWsGroups consecutive 64-element groups), run by 256 threads (tid 0..255) in two
// halves with a barrier of those threads between them (the caller's):
//   weight_scale_atoms_load(job, ...); <barrier>; weight_scale_atoms_store(job, ...)
constexpr int kWsGroups = 16;
using WsTile = uint32_t[128][kWsGroups + 1];

// The 8 words of weight_scale_atoms_load held in registers (word j of row tid / 2,
// group 8 * (tid % 2) + j), so that the loads can be issued long before the words
// are written to shared memory.
__device__ __forceinline__ void weight_scale_words(int64_t job, int tid,
                                                   const uint8_t* __restrict__ ws, int64_t N,
                                                   int64_t K, int bn, int na, int64_t KG,
                                                   uint32_t (&words)[8]) {
  const int64_t kg_chunks = ceil_div64(KG, kWsGroups);
  const int64_t kc = job % kg_chunks;
  const int a = static_cast<int>((job / kg_chunks) % na);
  const int64_t t = job / (kg_chunks * na);
  const int64_t nblk = K / 16;
  const int rr = tid / 2;
  const int g0 = (tid % 2) * 8;
  const int64_t nn = static_cast<int64_t>(a) * 128 + rr;
  const int64_t n = t * bn + nn;
  const bool row_ok = nn < bn && n < N;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int64_t kg = kc * kWsGroups + g0 + j;
    uint32_t word = 0;
    if (row_ok && 4 * kg < nblk) {
      const uint8_t* src = ws + n * nblk + kg * 4;
      if (4 * kg + 4 <= nblk && (reinterpret_cast<uintptr_t>(src) & 3) == 0) {
        word = __ldg(reinterpret_cast<const uint32_t*>(src));
      } else {
        for (int b = 0; b < 4; ++b)
          if (4 * kg + b < nblk) word |= static_cast<uint32_t>(__ldg(src + b)) << (8 * b);
      }
    }
    words[j] = word;
  }
}

__device__ __forceinline__ void weight_scale_words_to_tile(int tid, const uint32_t (&words)[8],
                                                           WsTile& tile) {
#pragma unroll
  for (int j = 0; j < 8; ++j) tile[tid / 2][(tid % 2) * 8 + j] = words[j];
}

__device__ __forceinline__ void weight_scale_atoms_load(int64_t job, int tid,
                                                        const uint8_t* __restrict__ ws, int64_t N,
                                                        int64_t K, int bn, int na, int64_t KG,
                                                        WsTile& tile) {
  uint32_t words[8];
  weight_scale_words(job, tid, ws, N, K, bn, na, KG, words);
  weight_scale_words_to_tile(tid, words, tile);
}

// One 512-byte atom = 128 words per group; thread tid writes word tid % 128 of the
// groups tid / 128, tid / 128 + 2, ...
__device__ __forceinline__ void weight_scale_atoms_store(int64_t job, int tid, int na, int64_t KG,
                                                         uint8_t* __restrict__ out,
                                                         const WsTile& tile) {
  const int64_t kg_chunks = ceil_div64(KG, kWsGroups);
  const int64_t kc = job % kg_chunks;
  const int a = static_cast<int>((job / kg_chunks) % na);
  const int64_t t = job / (kg_chunks * na);
  for (int j = tid / 128; j < kWsGroups; j += 2) {
    const int64_t kg = kc * kWsGroups + j;
    if (kg >= KG) continue;
    const int w = tid % 128;
    const int rr = (w % 4) * 32 + w / 4;  // word w holds row rr of the atom
    uint8_t* atom = out + static_cast<size_t>(((t * KG) + kg) * na + a) * kSfAtomBytes;
    reinterpret_cast<uint32_t*>(atom)[w] = tile[rr][j];
  }
}

// Number of weight-scale jobs for N rows, tile width bn and KG groups.
__host__ __device__ inline int64_t weight_scale_jobs(int64_t N, int bn, int64_t KG) {
  return ceil_div64(N, bn) * ((bn + 127) / 128) * ceil_div64(KG, kWsGroups);
}

}  // namespace ql
