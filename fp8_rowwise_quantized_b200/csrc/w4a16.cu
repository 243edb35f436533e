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
// These layers run on a few activation rows, so the weight is read once from HBM
// and the time goes to streaming it and to the per-weight decode. Design:
//   * one CTA of 16 warps per SM; a warp owns one item, a tile of 16 weight rows
//     times one of S parts of K (S chosen so that the items fill one wave), and
//     streams its codes and block scales straight into registers with 16-byte
//     loads, four 128-element groups ahead (about 74 KB in flight per SM, what
//     plain loads need to cover HBM latency; bulk copies into shared memory kept
//     too few bytes in flight per SM and were slower);
//   * the decode writes bf16 MMA fragments directly and mma.sync (m16n8k16, fp32
//     accumulation) does the multiply-adds, one instruction per 256 weights, which
//     leaves the issue slots to the decode. The tensor core is not here for FLOPs:
//     the MMA's N = 8 columns hold up to 8 activation rows;
//   * per weight pair: E2M1 pair -> f16 pair (exact), the products with the block
//     scale straight into fp32 by mixed-precision fma (exact: at most 6 significant
//     bits), one fp32 multiply by weight_scale_2 (the single RN32 rounding), and the
//     bf16 pair;
//   * the S partial sums of a tile meet in shared memory; bias, bf16 rounding and
//     the stores follow.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace ql {
namespace {

constexpr int kWTileRows = 16;      // weight rows per tile (the MMA's M)
constexpr int kWWarps = 16;         // warps per CTA, one item each
constexpr int kWThreads = 32 * kWWarps;
constexpr int kWGroup = 128;        // elements of a row per warp step: 4 lanes x 32

// Two block-scale codes (bytes 0 and 1 of s) -> their E4M3 values as an f16 pair
// (exact: every E4M3 value is an f16 value); byte 0 in the low half.
__device__ __forceinline__ uint32_t scale_f16x2(uint32_t s) {
  uint32_t h;
  asm("{\n\t.reg .b16 c;\n\t"
      "cvt.u16.u32 c, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, c;\n\t}"
      : "=r"(h)
      : "r"(s));
  return h;
}

// One 32-bit word of packed codes (element 2i in the low nibble of byte i) and
// the block scale d (f16: the low half of dd when HI == 0, else the high half) ->
// the four bf16 pairs of its eight dequantized weights (byte i -> r[i], element
// 2i in the low half). Per byte: E2M1 pair -> f16 pair (exact); v * d exactly in
// fp32 (mixed-precision fma with -0, so a -0 code stays -0); RN32(v * d * g) by
// one fp32 multiply per element; RN to bf16.
#define QL_W4_BYTE(C, R, D)                      \
  "cvt.rn.f16x2.e2m1x2 h, " C ";\n\t"            \
  "mov.b32 {v0, v1}, h;\n\t"                     \
  "fma.rn.f32.f16 f0, v0, " D ", 0f80000000;\n\t" \
  "fma.rn.f32.f16 f1, v1, " D ", 0f80000000;\n\t" \
  "mov.b64 p, {f0, f1};\n\t"                     \
  "mul.rn.f32x2 p, p, %6;\n\t"                   \
  "mov.b64 {f0, f1}, p;\n\t"                     \
  "cvt.rn.bf16x2.f32 " R ", f1, f0;\n\t"

template <int HI>
__device__ __forceinline__ void w4_word(uint32_t word, uint32_t dd, uint64_t gg, uint32_t (&r)[4]) {
  if (HI == 0) {
    asm("{\n\t"
        ".reg .b8 c0, c1, c2, c3;\n\t"
        ".reg .b16 v0, v1, d0, d1;\n\t"
        ".reg .b32 h, f0, f1;\n\t"
        ".reg .b64 p;\n\t"
        "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
        "mov.b32 {d0, d1}, %5;\n\t"
        QL_W4_BYTE("c0", "%0", "d0") QL_W4_BYTE("c1", "%1", "d0")
        QL_W4_BYTE("c2", "%2", "d0") QL_W4_BYTE("c3", "%3", "d0")
        "}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
        : "r"(word), "r"(dd), "l"(gg));
  } else {
    asm("{\n\t"
        ".reg .b8 c0, c1, c2, c3;\n\t"
        ".reg .b16 v0, v1, d0, d1;\n\t"
        ".reg .b32 h, f0, f1;\n\t"
        ".reg .b64 p;\n\t"
        "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
        "mov.b32 {d0, d1}, %5;\n\t"
        QL_W4_BYTE("c0", "%0", "d1") QL_W4_BYTE("c1", "%1", "d1")
        QL_W4_BYTE("c2", "%2", "d1") QL_W4_BYTE("c3", "%3", "d1")
        "}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
        : "r"(word), "r"(dd), "l"(gg));
  }
}
#undef QL_W4_BYTE

// D (16 x 8, fp32) += A (16 x 16, bf16, row-major) * B (16 x 8, bf16, column-major).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct W4Args {
  const uint16_t* x;
  int64_t M, K, N;
  const uint8_t* w;
  const uint8_t* ws;
  const float* g_ptr;
  const float* bias;
  uint16_t* y;
  int parts;  // S: parts of K per tile, a power of two dividing kWWarps
};


// Decode one group's codes of this lane (16 bytes of rows gid and gid + 8, scale
// pairs sa / sb) into bf16 fragments and run its 8 MMAs (per block of 8
// activation rows), alternating between two accumulators.
template <int MB>
__device__ __forceinline__ void w4_group(float (&acc)[MB][2][4], const uint4& c0, const uint4& c1,
                                         uint32_t sa, uint32_t sb, const uint4 (&xv)[MB][4],
                                         uint64_t gg) {
  const uint32_t da = scale_f16x2(sa), db = scale_f16x2(sb);
  const uint32_t wa[4] = {c0.x, c0.y, c0.z, c0.w};
  const uint32_t wb[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // code bytes 4q .. 4q + 3: MMAs 2q and 2q + 1
    uint32_t ra_[4], rb_[4];
    if (q < 2) {  // elements 0..15 of the chunk: the first scale byte
      w4_word<0>(wa[q], da, gg, ra_);
      w4_word<0>(wb[q], db, gg, rb_);
    } else {      // elements 16..31: the second
      w4_word<1>(wa[q], da, gg, ra_);
      w4_word<1>(wb[q], db, gg, rb_);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t a0 = ra_[2 * h], a2 = ra_[2 * h + 1];
      const uint32_t a1 = rb_[2 * h], a3 = rb_[2 * h + 1];
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        const uint32_t b0 = h == 0 ? xv[mb][q].x : xv[mb][q].z;
        const uint32_t b1 = h == 0 ? xv[mb][q].y : xv[mb][q].w;
        mma_bf16_16816(acc[mb][h], a0, a1, a2, a3, b0, b1);
      }
    }
  }
}

// 16-byte read-only load, not kept in L1; the L2::256B hint has L2 fetch the whole
// aligned 256 bytes around it, so the next groups of the same row (64 bytes each)
// are already on their way when their own loads are issued.
__device__ __forceinline__ uint4 ld_codes16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// One warp item: groups [g_begin, g_end) of the tile whose rows gid / gid + 8 are
// ra / rb. FULL: both rows exist and every group lies inside K, so no load needs a
// guard and the pointers advance by constants. The codes and scales of the next
// P groups wait in registers while one is decoded. Activation rows past M are
// read as row M - 1: they only feed MMA columns that are never stored.
template <int MB, int P, bool FULL>
__device__ __forceinline__ void w4_item(const W4Args& a, float (&acc)[MB][2][4], int64_t ra,
                                        int64_t rb, int64_t g_begin, int64_t g_end, int64_t m0,
                                        int gid, int tid, uint64_t gg) {
  const int64_t code_row = a.K / 2, scale_row = a.K / 16;
  const bool va = FULL || ra < a.N, vb = FULL || rb < a.N;
  const int64_t e_first = g_begin * kWGroup + 32 * tid;
  const uint8_t* pa = a.w + (va ? ra : 0) * code_row + e_first / 2;
  const uint8_t* pb = a.w + (vb ? rb : 0) * code_row + e_first / 2;
  const uint16_t* qa = reinterpret_cast<const uint16_t*>(a.ws + (va ? ra : 0) * scale_row) + e_first / 32;
  const uint16_t* qb = reinterpret_cast<const uint16_t*>(a.ws + (vb ? rb : 0) * scale_row) + e_first / 32;
  const uint4* px[MB];
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
    int64_t m = m0 + 8 * mb + gid;
    if (m > a.M - 1) m = a.M - 1;
    px[mb] = reinterpret_cast<const uint4*>(a.x + m * a.K + e_first);
  }
  // group g_begin + j sits j * 64 code bytes, 4 scale words and 16 activation
  // vectors further on
  auto load = [&](int64_t j, uint4& c0, uint4& c1, uint32_t& s0, uint32_t& s1) {
    const int64_t gi = g_begin + j;
    if (FULL) {
      if (gi < g_end) {
        c0 = ld_codes16(pa + 64 * j);
        c1 = ld_codes16(pb + 64 * j);
        s0 = __ldg(qa + 4 * j);
        s1 = __ldg(qb + 4 * j);
      }
    } else {
      c0 = c1 = make_uint4(0, 0, 0, 0);
      s0 = s1 = 0;
      const bool in_k = gi < g_end && gi * kWGroup + 32 * tid < a.K;
      if (in_k && va) {
        c0 = ld_codes16(pa + 64 * j);
        s0 = __ldg(qa + 4 * j);
      }
      if (in_k && vb) {
        c1 = ld_codes16(pb + 64 * j);
        s1 = __ldg(qb + 4 * j);
      }
    }
  };
  uint4 ca[P], cb[P];
  uint32_t sa[P], sb[P];
#pragma unroll
  for (int i = 0; i < P; ++i) load(i, ca[i], cb[i], sa[i], sb[i]);
  const int64_t n_groups = g_end - g_begin;
  for (int64_t base = 0; base < n_groups; base += P) {
#pragma unroll
    for (int i = 0; i < P; ++i) {
      const int64_t j = base + i;
      if (j >= n_groups) break;  // warp-uniform
      uint4 xv[MB][4];
      const bool x_in = FULL || (g_begin + j) * kWGroup + 32 * tid < a.K;
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          xv[mb][q] = x_in ? __ldg(px[mb] + 16 * j + q) : make_uint4(0, 0, 0, 0);
      w4_group<MB>(acc, ca[i], cb[i], sa[i], sb[i], xv, gg);
      // the slot just consumed takes the group P further on
      load(j + P, ca[i], cb[i], sa[i], sb[i]);
    }
  }
}

// Fragment roles (mma.sync m16n8k16, lane = 4 * gid + tid): A registers a0 / a2 hold
// row gid, a1 / a3 row gid + 8, at logical k (2 tid, 2 tid + 1) and (2 tid + 8,
// 2 tid + 9); B registers b0 / b1 hold activation row gid at the same logical k.
// Lane tid of a 128-element group owns the 32 elements [32 tid, 32 tid + 32) of
// its two weight rows (16 code bytes each) and, in MMA j (0..7), feeds elements
// 32 tid + 4 j + {0, 1} as logical (2 tid, 2 tid + 1) and 32 tid + 4 j + {2, 3} as
// (2 tid + 8, 2 tid + 9). The map from logical to actual k depends on tid and j
// only, so A and B agree for every row and the sum over the group is complete.
template <int MB, int P>
__global__ void __launch_bounds__(kWThreads, 1) w4a16_kernel(const W4Args a) {
  __shared__ float4 red[kWWarps][MB][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tid = lane & 3;
  const int S = a.parts;
  const int tiles_per_block = kWWarps / S;
  const int64_t tiles = (a.N + kWTileRows - 1) / kWTileRows;
  const int64_t blocks = (tiles + tiles_per_block - 1) / tiles_per_block;
  const int64_t groups = (a.K + kWGroup - 1) / kWGroup;
  const int64_t per_part = (groups + S - 1) / S;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * (8 * MB);
  const float g = __ldg(a.g_ptr);
  uint64_t gg;
  asm("mov.b64 %0, {%1, %1};" : "=l"(gg) : "f"(g));

  for (int64_t tb = blockIdx.x; tb < blocks; tb += gridDim.x) {
    const int64_t tile = tb * tiles_per_block + warp / S;
    const int64_t n0 = tile * kWTileRows;
    const int64_t ra = n0 + gid, rb = n0 + gid + 8;
    const int64_t g_begin = (warp % S) * per_part;
    const int64_t g_end = g_begin + per_part < groups ? g_begin + per_part : groups;

    float acc[MB][2][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mb][h][i] = 0.0f;

    if (tile < tiles) {  // warp-uniform
      const bool full = n0 + kWTileRows <= a.N && g_end * kWGroup <= a.K;
      if (full)
        w4_item<MB, P, true>(a, acc, ra, rb, g_begin, g_end, m0, gid, tid, gg);
      else
        w4_item<MB, P, false>(a, acc, ra, rb, g_begin, g_end, m0, gid, tid, gg);
    }

    // the S partial sums of each tile -> outputs
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
      red[warp][mb][lane] = make_float4(acc[mb][0][0] + acc[mb][1][0], acc[mb][0][1] + acc[mb][1][1],
                                        acc[mb][0][2] + acc[mb][1][2], acc[mb][0][3] + acc[mb][1][3]);
    __syncthreads();
    const float* redf = reinterpret_cast<const float*>(red);
    for (int e = threadIdx.x; e < tiles_per_block * MB * 128; e += kWThreads) {
      const int t = e / (MB * 128), rem = e % (MB * 128);
      const int mb = rem >> 7, l = (rem & 127) >> 2, r = rem & 3;
      float sum = 0.0f;  // from +0: a -0 weight gives +0, like an fp32 dot product
      for (int p = 0; p < S; ++p) sum += redf[(((t * S + p) * MB + mb) * 32 + l) * 4 + r];
      const int64_t n = (tb * tiles_per_block + t) * kWTileRows + (l >> 2) + 8 * (r >> 1);
      const int64_t m = m0 + 8 * mb + 2 * (l & 3) + (r & 1);
      if (n < a.N && m < a.M) {
        const float v = a.bias ? sum + __ldg(a.bias + n) : sum;
        const __nv_bfloat16 b = __float2bfloat16_rn(v);
        a.y[m * a.N + n] = *reinterpret_cast<const uint16_t*>(&b);
      }
    }
    __syncthreads();
  }
}

template <int MB, int P>
cudaError_t launch_mb(W4Args args, cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (args.N + kWTileRows - 1) / kWTileRows;
  const int64_t groups = (args.K + kWGroup - 1) / kWGroup;
  const int64_t passes = (args.M + 8 * MB - 1) / (8 * MB);
  if (passes > 65535) return cudaErrorInvalidValue;
  // parts of K per tile: the largest power of two (<= 16, <= the groups) whose
  // items still fit about one wave of warps over the activation-row passes
  const int64_t wave_warps = static_cast<int64_t>(sms) * kWWarps / passes;
  int S = 1;
  while (S < kWWarps && 2 * S <= groups && tiles * 2 * S * 10 <= wave_warps * 11) S *= 2;
  args.parts = S;
  const int64_t blocks = (tiles + kWWarps / S - 1) / (kWWarps / S);
  int64_t bx = sms / passes;
  if (bx < 1) bx = 1;
  if (bx > blocks) bx = blocks;
  dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(passes));
  w4a16_kernel<MB, P><<<grid, kWThreads, 0, s>>>(args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a16_linear(const void* x, int64_t M, int64_t K, const uint8_t* w,
                                const uint8_t* w_scale, int64_t N, const float* weight_scale_2,
                                const float* bias, void* y, cudaStream_t s) {
  W4Args args;
  args.x = static_cast<const uint16_t*>(x);
  args.M = M;
  args.K = K;
  args.N = N;
  args.w = w;
  args.ws = w_scale;
  args.g_ptr = weight_scale_2;
  args.bias = bias;
  args.y = static_cast<uint16_t*>(y);
  args.parts = 1;
  if (M <= 8) return launch_mb<1, 3>(args, s);
  return launch_mb<2, 2>(args, s);
}

}  // namespace ql
