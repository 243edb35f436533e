// INT4 W4A4 linear: the INT4 variant of the 4-bit layer of "Bringing Nunchaku 4-bit
// Diffusion Inference to Diffusers" (section "Introducing Nunchaku Lite": svdq_w4a4,
// "available in INT4 and NVFP4 variants"), without the low-rank branch. The page
// gives no format; the reading is signed 4-bit codes in [-8, 7] with one fp32 scale
// per 64-element group along K for both operands:
//   scale = RN32(amax / 7); codes = clamp(round-half-even(RN32(x * RN32(1 / scale))),
//   -8, 7); zero scale -> zero codes; element 2j in the low nibble of byte j.
//   Y[m, n] = bf16( sum_g xs[m,g] ws[n,g] sum_{k in g} qx[m,k] qw[n,k] + bias[n] )
//
// Why the GEMM looks the way it does on B200: the group scales are arbitrary fp32
// values, so each 64-wide group's integer product sum has to be scaled on its own
// before it joins the accumulator. The tensor cores apply per-block scales only in
// the block formats (the NVFP4 path of this library). Here the tcgen05 integer MMA
// (kind::i8) computes one group's sums at a time into TMEM, and the CUDA cores read
// them back, scale them and add them to fp32 accumulators held in registers.
//
//  * Operands. tcgen05 has no 4-bit integer kind, so the 4-bit codes are widened to
//    int8 in shared memory: a byte's high nibble, kept in place, is the int8 value
//    16 * v, and the low nibble shifted up by 4 is the same (three SIMD operations
//    per 8 codes, no sign fix-up). Both operands carry the factor 16, so the MMA
//    sums are 256 * S exactly (|256 S| <= 2^20); the 2^-8 is applied once per output.
//    Within every 8 codes the even elements come first, then the odd ones, in both
//    operands, which leaves each group's sum unchanged.
//  * Exact int32 -> fp32 without a conversion instruction: the epilogue adds the
//    bits of 1.5 * 2^23 (0x4B400000) to each int32 sum (|256 S| <= 2^20), which
//    gives the bits of the float 1.5 * 2^23 + 256 S, and one packed subtraction
//    recovers 256 S. (Filling the TMEM buffer with the constant first, by TMEM
//    stores from the epilogue or by tcgen05.cp from the MMA thread, and letting
//    the MMA accumulate onto it measured slower: both lengthen the per-group
//    hand-off between the MMA and the epilogue.)
//  * Per output and group: that integer add, one subtraction, one multiply by the
//    weight scale and one fma with the activation scale, the fp32 ones two outputs
//    per packed instruction (all RN). The epilogue reads a group's 64 columns (four
//    16-column TMEM loads, one wait) and hands the buffer back to the MMA before
//    the arithmetic; the group's first MMA overwrites the buffer.
//
// Roles (one CTA per SM, persistent over 128 x 128 output tiles, 12 warps: three per
// SM sub-partition, which leaves 168 registers per thread):
//   warps 0-7   epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (tile rows) and
//               columns 64 (w / 4) .. +63; 64 fp32 accumulators per thread
//   warps 8-10  unpack: thread 0 loads each stage's packed codes (two groups, 64
//               bytes per row, activation and weight rows) by TMA into a ring three
//               stages ahead; every thread copies its rows' scales (cp.async) into
//               the same slot, writes the int8 operands into the 128-byte-swizzled
//               K-major layout the MMA reads (the layout a TMA load with 128-byte
//               swizzle writes) and the stage's scales into a ring of group slots
//   warp 11     MMA: per group, two MMAs (K = 32) into one of two TMEM buffers
// Every wait is bounded (the device status word records a timeout).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

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

// ------------------------------------------------------------------ GEMM
constexpr int kI4Tile = 128;                 // output rows and columns per tile
constexpr int kI4EpiWarps = 8;
constexpr int kI4UnpackWarps = 3;
constexpr int kI4UnpackThreads = kI4UnpackWarps * 32;
constexpr int kI4MmaWarp = kI4EpiWarps + kI4UnpackWarps;
constexpr int kI4Threads = (kI4MmaWarp + 1) * 32;
constexpr int kI4CodeTasks = 2 * kI4Tile * 4;  // 16-byte pieces of packed codes per stage
constexpr int kI4Pieces = (kI4CodeTasks + kI4UnpackThreads - 1) / kI4UnpackThreads;
constexpr int kI4ScRows = (2 * kI4Tile + kI4UnpackThreads - 1) / kI4UnpackThreads;
constexpr int kI4PackAhead = 3;              // stages loaded ahead of the one unpacked
constexpr int kI4PackRing = kI4PackAhead + 1;
constexpr int kI4OpStages = 3;               // int8 operand stages
constexpr int kI4ScSlots = 8;                // group slots of the scale ring
constexpr int kI4PackCodeBytes = 2 * kI4Tile * 64;                    // packed A + B, one stage
constexpr int kI4PackStageBytes = kI4PackCodeBytes + 2 * kI4Tile * 8;  // + 2 scales per row
constexpr int kI4OpStageBytes = 2 * kI4Tile * 128;                    // int8 A + B, one stage
constexpr int kI4ScSlotBytes = 2 * kI4Tile * 4;                       // xs[128], ws[128]
constexpr int kI4Bars = 2 * kI4PackRing + 2 * kI4OpStages + 2 * kI4ScSlots + 2 + 2 + 1;
constexpr int kI4Smem = 1024 + kI4OpStages * kI4OpStageBytes + kI4PackRing * kI4PackStageBytes +
                        kI4ScSlots * kI4ScSlotBytes + kI4Bars * 8 + 16;
constexpr int kI4TmemCols = 2 * kI4Tile;
constexpr uint32_t kI4Magic = 0x4B400000u;   // bits of 1.5 * 2^23
// instruction descriptor: int32 accumulator, signed int8 A and B, K-major, N = M = 128
constexpr uint32_t kI4Idesc = (2u << 4) | (1u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(kI4Tile >> 3) << 17) |
                              (static_cast<uint32_t>(kI4Tile >> 4) << 24);
static_assert(kI4Smem <= 227 * 1024, "shared memory");

struct Int4GemmArgs {
  const float* xs;     // activation group scales [M, K/64]
  const float* ws;     // weight group scales [N, K/64]
  const float* bias;   // [N] or null
  uint16_t* y;         // bf16 [M, N]
  int64_t M, N, K;
  int tiles_m, total_tiles;
  int vec_store;       // y 16-byte aligned and N % 8 == 0
  int* status;
  uint64_t timeout_ns;
};

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
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// 16 * v for the codes in the low / high nibbles of each byte of w, as int8 bytes.
__device__ __forceinline__ uint32_t s4_low_x16(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t s4_high_x16(uint32_t w) { return w & 0xF0F0F0F0u; }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__device__ __forceinline__ void i4_record_timeout(int* status) {
  if (status) atomicCAS(status, 0, static_cast<int>(QL_ERR_TIMEOUT_CODE));
}

__global__ void __launch_bounds__(kI4Threads, 1)
int4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const Int4GemmArgs args) {
  extern __shared__ uint8_t i4_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(i4_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* op = smem;                                               // int8 operand stages
  uint8_t* pack = op + kI4OpStages * kI4OpStageBytes;               // packed codes + scales
  float* scr = reinterpret_cast<float*>(pack + kI4PackRing * kI4PackStageBytes);  // scale slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(scr + kI4ScSlots * 2 * kI4Tile);
  uint64_t* p_full = bars;                       // packed codes of a stage landed (TMA bytes)
  uint64_t* p_empty = p_full + kI4PackRing;      // packed slot read (the unpack warps)
  uint64_t* s_full = p_empty + kI4PackRing;      // operand stage written (the unpack warps)
  uint64_t* s_empty = s_full + kI4OpStages;      // operand stage read by the MMAs (commit)
  uint64_t* sc_full = s_empty + kI4OpStages;     // scale slot written (the unpack warps)
  uint64_t* sc_empty = sc_full + kI4ScSlots;     // scale slot read (the epilogue warps)
  uint64_t* t_full = sc_empty + kI4ScSlots;      // TMEM buffer holds a group's sums (commit)
  uint64_t* t_empty = t_full + 2;                // TMEM buffer read (the epilogue warps)
  uint64_t* drain = t_empty + 2;                 // every MMA of this CTA has completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = static_cast<int>(args.K / 64);
  const int NS = (G + 1) / 2;  // stages per tile (the last one may hold one group)
  const int first = blockIdx.x, step = gridDim.x;
  const int my_tiles = first < args.total_tiles ? (args.total_tiles - 1 - first) / step + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kI4PackRing; ++i) {
      mbar_init(p_full + i, 1);
      mbar_init(p_empty + i, kI4UnpackWarps);
    }
    for (int i = 0; i < kI4OpStages; ++i) {
      mbar_init(s_full + i, kI4UnpackWarps);
      mbar_init(s_empty + i, 1);
    }
    for (int i = 0; i < kI4ScSlots; ++i) {
      mbar_init(sc_full + i, kI4UnpackWarps);
      mbar_init(sc_empty + i, kI4EpiWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(t_full + i, 1);
      mbar_init(t_empty + i, kI4EpiWarps);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == kI4MmaWarp) {
    tmem_alloc(tmem_holder, kI4TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp < kI4EpiWarps) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, h = warp >> 2;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                           static_cast<uint32_t>(h * 64);
    if (lane == 0) {  // both buffers start free
      mbar_arrive(t_empty);
      mbar_arrive(t_empty + 1);
    }
    uint32_t gc = 0;  // groups consumed by this CTA
    bool ok = true;
    for (int ti = 0; ti < my_tiles && ok; ++ti) {
      const int tile = first + ti * step;
      const int m_blk = tile % args.tiles_m, n_blk = tile / args.tiles_m;
      const uint64_t deadline = globaltimer_ns() + args.timeout_ns;
      float2 acc[32];  // columns 2j, 2j + 1 of this warp's 64
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = make_float2(0.0f, 0.0f);
      for (int g = 0; g < G; ++g, ++gc) {
        const uint32_t b = gc & 1u, slot = gc % kI4ScSlots;
        if (!warp_wait_bounded(t_full + b, (gc >> 1) & 1u, deadline) ||
            !warp_wait_bounded(sc_full + slot, (gc / kI4ScSlots) & 1u, deadline)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r[64];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld_32x32b_x16(taddr + b * kI4Tile + 16 * c,
                             *reinterpret_cast<uint32_t(*)[16]>(&r[16 * c]));
        tmem_ld_wait();
        // the sums are in registers: the buffer goes back to the MMA
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(t_empty + b);
        const float* slot_p = scr + slot * (2 * kI4Tile);
        const float2 sx = make_float2(slot_p[q * 32 + lane], slot_p[q * 32 + lane]);
        const float4* ws4 = reinterpret_cast<const float4*>(slot_p + kI4Tile + h * 64);
        const float2 neg_magic = make_float2(-12582912.0f, -12582912.0f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 w = ws4[i];
          float2 f0 = __fadd2_rn(make_float2(__uint_as_float(r[4 * i] + kI4Magic),
                                             __uint_as_float(r[4 * i + 1] + kI4Magic)),
                                 neg_magic);
          float2 f1 = __fadd2_rn(make_float2(__uint_as_float(r[4 * i + 2] + kI4Magic),
                                             __uint_as_float(r[4 * i + 3] + kI4Magic)),
                                 neg_magic);
          f0 = __fmul2_rn(f0, make_float2(w.x, w.y));
          f1 = __fmul2_rn(f1, make_float2(w.z, w.w));
          acc[2 * i] = __ffma2_rn(f0, sx, acc[2 * i]);
          acc[2 * i + 1] = __ffma2_rn(f1, sx, acc[2 * i + 1]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sc_empty + slot);
      }
      if (!ok) break;
      // bf16(acc * 2^-8 + bias), row m, columns n0 .. n0 + 63
      const int64_t m = static_cast<int64_t>(m_blk) * kI4Tile + q * 32 + lane;
      const int64_t n0 = static_cast<int64_t>(n_blk) * kI4Tile + h * 64;
      if (m < args.M) {
        uint16_t* yr = args.y + m * args.N;
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          const int64_t n = n0 + c;
          if (n < args.N) {
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float bv = (args.bias && n + e < args.N) ? __ldg(args.bias + n + e) : 0.0f;
              const float2 a2 = acc[(c + e) >> 1];
              o[e] = fmaf((e & 1) ? a2.y : a2.x, 0.00390625f, bv);
            }
            if (args.vec_store && n + 8 <= args.N) {
              *reinterpret_cast<uint4*>(yr + n) =
                  make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                             pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                if (n + e < args.N) {
                  const __nv_bfloat16 v = __float2bfloat16_rn(o[e]);
                  yr[n + e] = *reinterpret_cast<const uint16_t*>(&v);
                }
              }
            }
          }
        }
      }
    }
    if (!ok) i4_record_timeout(args.status);
  } else if (warp < kI4MmaWarp) {
    // ------------------------------------------------------------ unpack
    const int t = threadIdx.x - kI4EpiWarps * 32;  // 0 .. 95
    const uint32_t pack_base = smem_u32(pack), op_base = smem_u32(op);
    // A stage's packed codes: rows 0-127 activation rows, 128-255 weight rows, 64
    // bytes each (TMA boxes of 64 bytes x 128 rows). Piece L = row * 4 + seg is 16
    // bytes (32 codes) at segment seg of row `row`; thread t unpacks the pieces
    // L = t + 96 i into the two 16-byte chunks 2 seg, 2 seg + 1 of its int8 row,
    // whose places in the 128-byte-swizzled stage do not change from stage to stage.
    uint32_t dst_off[kI4Pieces][2];
#pragma unroll
    for (int i = 0; i < kI4Pieces; ++i) {
      const int L = t + kI4UnpackThreads * i;
      const int row = (L < kI4CodeTasks ? L : 0) >> 2, seg = L & 3, r = row & (kI4Tile - 1);
      const uint32_t rb = (row >= kI4Tile ? kI4Tile * 128 : 0) + (r >> 3) * 1024 + (r & 7) * 128;
      dst_off[i][0] = rb + (((2 * seg) ^ (r & 7)) << 4);
      dst_off[i][1] = rb + (((2 * seg + 1) ^ (r & 7)) << 4);
    }
    // scales: rows t + 96 i of the stage (activation rows, then weight rows), two
    // groups each, by cp.async into the packed slot after the codes
    int f_ti = 0, f_s = 0;  // next stage to fetch: tile index, stage within the tile
    int f_tile_loaded = -1;
    const float* sc_src[kI4ScRows];
    bool sc_in[kI4ScRows];
    uint32_t p_issued = 0;  // TMA stages issued (thread 0)
    auto fetch = [&](uint32_t fs) {  // fs: this CTA's stage index being fetched
      if (f_ti < my_tiles) {
        const int tile = first + f_ti * step;
        const int m_blk = tile % args.tiles_m, n_blk = tile / args.tiles_m;
        if (f_tile_loaded != f_ti) {
          f_tile_loaded = f_ti;
#pragma unroll
          for (int i = 0; i < kI4ScRows; ++i) {
            const int row = t + kI4UnpackThreads * i;
            const bool is_b = row >= kI4Tile;
            const int64_t grow = static_cast<int64_t>(is_b ? n_blk : m_blk) * kI4Tile +
                                 (row & (kI4Tile - 1));
            sc_in[i] = row < 2 * kI4Tile && grow < (is_b ? args.N : args.M);
            sc_src[i] = (is_b ? args.ws : args.xs) + (sc_in[i] ? grow * G : 0);
          }
        }
        const uint32_t slot = fs % kI4PackRing;
        const uint32_t dst = pack_base + slot * kI4PackStageBytes;
        if (t == 0) {
          // the slot's previous contents (stage fs - 4) have been read by every unpack warp
          bool free_ok = mbar_wait_bounded(p_empty + slot, ((fs / kI4PackRing) & 1u) ^ 1u,
                                           globaltimer_ns() + args.timeout_ns);
          if (free_ok) {
            mbar_arrive_expect_tx(p_full + slot, kI4PackCodeBytes);
            tma_load_2d(pack + slot * kI4PackStageBytes, &tmap_a, p_full + slot, f_s * 64,
                        m_blk * kI4Tile);
            tma_load_2d(pack + slot * kI4PackStageBytes + kI4Tile * 64, &tmap_b, p_full + slot,
                        f_s * 64, n_blk * kI4Tile);
            ++p_issued;
          } else {
            i4_record_timeout(args.status);
          }
        }
#pragma unroll
        for (int i = 0; i < kI4ScRows; ++i) {
          const int row = t + kI4UnpackThreads * i;
          if (row < 2 * kI4Tile) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const bool ok = sc_in[i] && 2 * f_s + j < G;
              cp_async4(dst + kI4PackCodeBytes + row * 8 + j * 4,
                        sc_src[i] + (ok ? 2 * f_s + j : 0), ok);
            }
          }
        }
        if (++f_s == NS) {
          f_s = 0;
          ++f_ti;
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int i = 0; i < kI4PackAhead; ++i) fetch(i);
    uint32_t sc = 0, gc = 0;  // stages and groups produced by this CTA
    bool ok = true;
    for (int ti = 0; ti < my_tiles && ok; ++ti) {
      const uint64_t deadline = globaltimer_ns() + args.timeout_ns;
      for (int s = 0; s < NS; ++s, ++sc) {
        fetch(sc + kI4PackAhead);
        cp_async_wait<kI4PackAhead>();  // this thread's scale copies of stage sc have landed
        const uint32_t ps = sc % kI4PackRing, os = sc % kI4OpStages;
        if (!warp_wait_bounded(p_full + ps, (sc / kI4PackRing) & 1u, deadline) ||
            !warp_wait_bounded(s_empty + os, ((sc / kI4OpStages) & 1u) ^ 1u, deadline)) {
          ok = false;
          break;
        }
        const uint32_t src = pack_base + ps * kI4PackStageBytes;
        const uint32_t dst = op_base + os * kI4OpStageBytes;
        // all loads first, then the stores: the shared-memory accesses are ordered
        // asm statements, so interleaving them would wait out each load's latency
        const bool last_piece = t + kI4UnpackThreads * (kI4Pieces - 1) < kI4CodeTasks;
        uint4 w[kI4Pieces];
#pragma unroll
        for (int i = 0; i < kI4Pieces; ++i)
          if (i + 1 < kI4Pieces || last_piece) w[i] = lds128(src + (t + kI4UnpackThreads * i) * 16);
#pragma unroll
        for (int i = 0; i < kI4Pieces; ++i) {
          if (i + 1 < kI4Pieces || last_piece) {
            sts128(dst + dst_off[i][0], s4_low_x16(w[i].x), s4_high_x16(w[i].x),
                   s4_low_x16(w[i].y), s4_high_x16(w[i].y));
            sts128(dst + dst_off[i][1], s4_low_x16(w[i].z), s4_high_x16(w[i].z),
                   s4_low_x16(w[i].w), s4_high_x16(w[i].w));
          }
        }
        fence_proxy_async_shared();  // the MMA (async proxy) reads what was just written
        const int ng = (G - 2 * s) < 2 ? (G - 2 * s) : 2;
        float sv[kI4ScRows][2];
#pragma unroll
        for (int i = 0; i < kI4ScRows; ++i) {
          const int row = t + kI4UnpackThreads * i;
          if (row < 2 * kI4Tile) {
            sv[i][0] = *reinterpret_cast<const float*>(pack + ps * kI4PackStageBytes +
                                                       kI4PackCodeBytes + row * 8);
            sv[i][1] = *reinterpret_cast<const float*>(pack + ps * kI4PackStageBytes +
                                                       kI4PackCodeBytes + row * 8 + 4);
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(s_full + os);
          mbar_arrive(p_empty + ps);  // the packed slot has been read
        }
        for (int j = 0; j < ng; ++j, ++gc) {
          const uint32_t slot = gc % kI4ScSlots;
          if (!warp_wait_bounded(sc_empty + slot, ((gc / kI4ScSlots) & 1u) ^ 1u, deadline)) {
            ok = false;
            break;
          }
          // slot layout: xs of the tile's 128 rows, then ws of its 128 columns
          float* slot_p = scr + slot * (2 * kI4Tile);
#pragma unroll
          for (int i = 0; i < kI4ScRows; ++i) {
            const int row = t + kI4UnpackThreads * i;
            if (row < 2 * kI4Tile) slot_p[row] = j ? sv[i][1] : sv[i][0];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(sc_full + slot);
        }
        if (!ok) break;
      }
    }
    cp_async_wait<0>();
    if (t == 0) {
      // the TMA loads issued ahead of the last stage processed complete before exit
      const uint64_t dl = globaltimer_ns() + 100000000ull;
      for (uint32_t fs = sc; fs < p_issued; ++fs)
        mbar_wait_bounded(p_full + fs % kI4PackRing, (fs / kI4PackRing) & 1u, dl);
    }
    if (!ok) i4_record_timeout(args.status);
  } else {
    // ------------------------------------------------------------ MMA issuer
    uint32_t sc = 0, gc = 0;
    bool ok = true;
    const uint32_t op_base = smem_u32(op);
    for (int ti = 0; ti < my_tiles && ok; ++ti) {
      const uint64_t deadline = globaltimer_ns() + args.timeout_ns;
      for (int s = 0; s < NS; ++s, ++sc) {
        const uint32_t os = sc % kI4OpStages;
        if (!warp_wait_bounded(s_full + os, (sc / kI4OpStages) & 1u, deadline)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = op_base + os * kI4OpStageBytes;
        const uint32_t b_addr = a_addr + kI4Tile * 128;
        const int ng = (G - 2 * s) < 2 ? (G - 2 * s) : 2;
        for (int j = 0; j < ng; ++j, ++gc) {
          const uint32_t b = gc & 1u;
          if (!warp_wait_bounded(t_empty + b, (gc >> 1) & 1u, deadline)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            // the group's first MMA overwrites the buffer, the second accumulates
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
              const uint32_t koff = static_cast<uint32_t>((2 * j + kb) * 32);
              mma_i8(tmem_base + b * kI4Tile, smem_desc(a_addr + koff, 16, 1024, 2),
                     smem_desc(b_addr + koff, 16, 1024, 2), kI4Idesc, kb);
            }
            tc_commit(t_full + b);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) tc_commit(s_empty + os);
        __syncwarp();
      }
    }
    // every MMA issued here has completed before TMEM is released
    if (elect_one()) tc_commit(drain);
    __syncwarp();
    if (!mbar_wait_bounded(drain, 0, globaltimer_ns() + 100000000ull)) ok = false;
    if (!ok) i4_record_timeout(args.status);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kI4MmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kI4TmemCols);
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
                             void* y, int* status, uint64_t timeout_ns, cudaStream_t s) {
  // per device: the kernel's shared-memory limit (a per-device attribute) and the SM count
  static int sms[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  int nsm = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (sms[dev] == 0) {
      e = cudaFuncSetAttribute(int4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kI4Smem);
      if (e != cudaSuccess) return e;
      int n = 0;
      e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      sms[dev] = n;
    }
    nsm = sms[dev];
  }
  const int64_t tm = (M + kI4Tile - 1) / kI4Tile, tn = (N + kI4Tile - 1) / kI4Tile;
  if (tm * tn > (1ll << 30)) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, static_cast<uint64_t>(K / 2),
                 static_cast<uint64_t>(M), static_cast<uint64_t>(K / 2), 64, kI4Tile,
                 CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
      !encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, static_cast<uint64_t>(K / 2),
                 static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2), 64, kI4Tile,
                 CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
    return cudaErrorInvalidValue;
  Int4GemmArgs a;
  a.xs = xs;
  a.ws = ws;
  a.bias = bias;
  a.y = static_cast<uint16_t*>(y);
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = static_cast<int>(tm);
  a.total_tiles = static_cast<int>(tm * tn);
  a.vec_store = (N % 8 == 0) && (reinterpret_cast<uintptr_t>(y) & 15u) == 0;
  a.status = status;
  a.timeout_ns = timeout_ns;
  const int grid = a.total_tiles < nsm ? a.total_tiles : nsm;
  int4_gemm_kernel<<<grid, kI4Threads, kI4Smem, s>>>(ta, tb, a);
  return cudaGetLastError();
}

}  // namespace ql
