// Tensor-core GEMMs of the quantized linear (sm_100a, tcgen05):
//   FP4 = true : Y = bf16(input_scale * weight_scale_2 * sum_k A*SFA * B*SFB + bias),
//                A, B packed E2M1, SFA/SFB E4M3 per 16 elements (kind::mxf4nvf4);
//   FP4 = false: Y = bf16(x_scale[m] * w_scale[n] * sum_k A * B + bias),
//                A, B E4M3 (kind::f8f6f4).
// The block-scaled FP4 GEMM is the "mm_fp4" step and the FP8 one the "scaled GEMM
// with row-wise scales" step of the Diffusers page "BFL (fp8r / nvfp4)", section
// "Kernels", table.
//
// Structure: persistent CTAs, CG = 1 (one SM per 128 x BN tile) or CG = 2 (a CTA
// pair per 256 x BN tile: one tcgen05 MMA spans both SMs; each CTA holds 128 rows
// of A, half of B and the scales its MMA rows need, so each SM streams about half
// the B bytes per flop). Per CTA:
//   warp 0     TMA producer: A, B tiles (128-byte swizzle) and scale atoms into a
//              STAGES-deep shared-memory ring; in a pair every load's bytes are
//              counted on the leader CTA's barrier;
//   warp 1     TMEM allocation; in the leader CTA, one thread per stage copies the
//              scale atoms into TMEM (tcgen05.cp) and issues 4 MMAs of K = 64 (FP4)
//              or K = 32 (FP8) into a TMEM accumulator;
//   warps 2-5  epilogue: TMEM -> registers (tcgen05.ld), scale, bias, bf16,
//              128-byte-swizzled staging tile, TMA store.
// Accumulators are double-buffered in TMEM (for 256-column FP4 tiles the two
// buffers share one 64-column slab), so the epilogue of one tile overlaps the main
// loop of the next.
// Every wait is bounded by a deadline; on expiry the kernel records
// QL_ERR_TIMEOUT in the device status word, drains its own copies and MMAs,
// frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "internal.h"
#include "layout.cuh"
#include "ptx.cuh"

namespace ql {

// SM clock seen by the GEMM: CTA 0 of every GEMM launch stores its elapsed SM
// cycles (%clock64) and nanoseconds (%globaltimer) from set-up to teardown, so
// the clock the tensor cores ran at under the kernel's own load can be read back
// (it is below the idle boost clock when the part runs at its power limit).
__device__ unsigned long long g_gemm_clock[2];

namespace {

constexpr int kRowsPerCta = 128;
constexpr int kThreads = 192;       // producer, MMA, 4 epilogue warps
constexpr int kThreadsFused = 256;  // 8 warps share the quantization; warps 6, 7 stop there
constexpr int kSmemLimit = 232448;  // 227 KB opt-in per block
constexpr int kTmemCols = 512;
constexpr int kEpiBufBytes = 32 * 128;  // 32 rows x 64 bf16 (128-byte swizzled), one TMA box
// One staging buffer per epilogue warp: the shared memory goes to one more
// pipeline stage instead (the TMA store reads a 4 KB buffer long before the warp
// has its next slab ready).
constexpr int kEpiBufsPerWarp = 1;

struct GemmArgs {
  int M, N, K;
  int tiles_m, tiles_n, num_k_tiles, total_tiles;
  int64_t kg;               // FP4: 64-element scale groups per row (padded)
  const float* scale_a;     // FP4: input_scale (scalar)   FP8: x_scale [M]
  const float* scale_b;     // FP4: weight_scale_2 (scalar) FP8: w_scale [N]
  const float* bias;        // [N] or null
  uint16_t* y;              // bf16 [M, N]
  int* status;              // device status word
  uint64_t timeout_ns;
  int inject_fault;
  int wait_prior_grid;
  int b_ready;              // plain non-skinny mode: B is not written by the previous kernel, so
                            // the producer starts its first stages' B loads before the wait
  int use_tma_store;        // Y written through shared memory + TMA (needs N % 8 == 0)
  int raster_n;             // tile order: 1 = N fastest (m_blk = tile / tiles_n), 0 = M fastest
  // in-launch activation quantization (FP4, K % 256 == 0)
  const uint16_t* x;        // bf16 [M, K]
  uint8_t* xq;              // packed codes [M, K/2]: written here, read as A
  uint8_t* xs;              // activation scale atoms: written here, read as SFA
  const uint8_t* w_scale;   // weight scales, row-major E4M3 [N, K/16]
  uint8_t* ws_atoms;        // weight scale atoms for tile width BN: written here, read as SFB
  uint64_t* sync;           // sync_words tagged counters (see kSyncBarrier)
  // GELU-quantize epilogue (FP4): NVFP4 of GELU(Y) with global scale *gq_scale
  uint8_t* gq_codes;        // packed E2M1 [M, N/2]
  uint8_t* gq_atoms;        // E4M3 scales in the activation atom layout (K' = N)
  const float* gq_scale;
  int sync_words;
  uint32_t tag;             // this launch's tag, odd
  // low-rank branch (FP4, plain mode): after a tile's K tiles, one more stage of
  // bf16 operands (tmap_lra: [M, r] activations pre-divided by alpha; tmap_lrb:
  // [N, r]) and lr_k16 = ceil(r / 16) MMAs of K = 16 into the same accumulator
  int lr_k16;
  // rows of A one CTA loads per K tile: 128, or M rounded up to 8 when a lone CTA's
  // tile has fewer valid rows (rows past it keep stale shared memory, which only
  // reaches accumulator rows that are never stored; their scale atoms are zero)
  int a_box_rows;
  // skinny kernels: weight scales taken row-major from w_scale ([N, K/16], ks_bytes
  // per row; 16-byte loads when sfb_vec16) instead of atoms in the workspace
  int sfb_rowmajor;
  int ks_bytes;
  int sfb_vec16;
};

// AROWS: rows of A a pipeline stage holds. 128 for every tile, or 16 / 32 / 64 for
// the skinny kernels (M <= AROWS, one CTA per tile): the MMA still runs M = 128
// and reads past the stage's rows into neighbouring shared memory, which only
// reaches accumulator rows >= M (never stored); the stage being smaller, more
// stages fit, so more weight bytes are in flight per SM.
template <bool FP4, int BN, int CG, int AROWS = kRowsPerCta>
struct Cfg {
  static constexpr int NA = (BN + 127) / 128;                        // 128-row scale atoms of B
  static constexpr int B_ROWS = BN / CG;                             // B rows held by one CTA
  static constexpr int A_BYTES = AROWS * 128;
  static constexpr int B_BYTES = B_ROWS * 128;
  static constexpr int SFA_BYTES = FP4 ? 4 * kSfAtomBytes : 0;       // 4 K-groups x 1 atom
  static constexpr int SFB_BYTES = FP4 ? 4 * NA * kSfAtomBytes : 0;  // 4 K-groups x NA atoms
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int EPI_BUFS = kEpiBufsPerWarp;
  static constexpr int EPI_BYTES = 4 * EPI_BUFS * kEpiBufBytes;      // 4 epilogue warps
  static constexpr int COLVEC_BYTES = 2 * 2 * 256 * 4;  // bias + column scales, 2 tiles deep
  static constexpr int RESERVED = 1024 /*alignment*/ + 1024 /*barriers*/ + EPI_BYTES + COLVEC_BYTES;
  static constexpr int STAGES_FIT = (kSmemLimit - RESERVED) / STAGE_BYTES;
  static constexpr int MAX_STAGES = AROWS < kRowsPerCta ? 12 : 8;
  static constexpr int STAGES = STAGES_FIT > MAX_STAGES ? MAX_STAGES : STAGES_FIT;
  static constexpr int SF_COLS = FP4 ? 16 + 4 * NA * 4 : 0;
  // Two accumulator buffers. When two full BN-column buffers and the scale columns
  // do not fit in TMEM (BN = 256 with scales), the second buffer starts 64 columns
  // early and the two share one 64-column slab: the epilogue drains that slab
  // first and hands the buffer back right after it.
  static constexpr bool OVERLAP = (2 * BN + SF_COLS > kTmemCols);
  static constexpr int ACC_STRIDE = OVERLAP ? BN - 64 : BN;  // column of buffer 1
  static constexpr int SFA_COL = ACC_STRIDE + BN;
  static constexpr int SFB_COL = SFA_COL + 16;
  static constexpr int SMEM = RESERVED + STAGES * STAGE_BYTES;
  static constexpr int TILE_M = kRowsPerCta * CG;
  // instruction descriptor: M = 128 * CG, N = BN, K-major A and B, fp32 accumulate;
  // FP4: E2M1 x E2M1 with UE4M3 scales; FP8: E4M3 x E4M3.
  static constexpr uint32_t IDESC =
      FP4 ? ((1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(TILE_M >> 4) << 24))
          : ((1u << 4) | (uint32_t(BN >> 3) << 17) | (uint32_t(TILE_M >> 4) << 24));
  // the low-rank branch's bf16 x bf16 MMAs (K = 16 each) into the same accumulator
  static constexpr uint32_t IDESC_BF16 = (1u << 4) | (1u << 7) | (1u << 10) |
                                         (uint32_t(BN >> 3) << 17) | (uint32_t(TILE_M >> 4) << 24);
  static_assert(STAGES >= 2, "shared memory too small for two stages");
  static_assert(SFA_COL + SF_COLS <= kTmemCols, "TMEM budget");
  static_assert(!OVERLAP || BN == 256, "only the 256-column tile shares a slab");
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "tile width");
  // epilogue slab: 64 columns (128-byte rows, 128-byte swizzle) when BN allows,
  // else 32 columns (64-byte rows, 64-byte swizzle)
  static constexpr int SLAB = (BN % 64 == 0) ? 64 : 32;
  static constexpr int NSLAB = BN / SLAB;
  static_assert(CG == 1 || CG == 2, "one SM or a CTA pair");
  static_assert(AROWS == kRowsPerCta || (CG == 1 && AROWS % 16 == 0 && AROWS <= 64),
                "skinny stages: one CTA per tile, 16 / 32 / 64 rows of A");
  static_assert(B_ROWS % 8 == 0, "B half must be whole 8-row core groups");
};

__device__ __forceinline__ void tile_coords(int tile, const GemmArgs& a, int& m_blk, int& n_blk) {
  if (a.raster_n) {
    m_blk = tile / a.tiles_n;
    n_blk = tile - m_blk * a.tiles_n;
  } else {
    m_blk = tile % a.tiles_m;
    n_blk = tile / a.tiles_m;
  }
}

__device__ __forceinline__ void record_timeout(int* status) {
  if (status) atomicCAS(status, 0, static_cast<int>(QL_ERR_TIMEOUT_CODE));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// ---------------------------------------------------------------- in-launch quantization
// The single-launch NVFP4 linear first quantizes the activations and lays out the
// weight scales into its workspace with every warp of every CTA, then meets at a
// grid-wide barrier, then runs the GEMM below on that workspace (which stays in
// L2). Words shared by the CTAs, in the workspace: the barrier count and the
// count of CTAs that have finished. Each word holds (tag << 32) | count; a word
// carrying another launch's tag (or leftover bytes) counts as zero. The last CTA
// to finish writes them back to zero, so a replay of the same launch (same tag,
// e.g. from a CUDA graph) also starts from zero. The grid is one wave of resident
// CTAs, so the barrier does not wait for CTAs that cannot start; its wait is
// bounded all the same.
constexpr int kSyncBarrier = 0;
constexpr int kSyncExit = 1;

__device__ __forceinline__ uint32_t tagged_count(uint64_t w, uint32_t tag) {
  return static_cast<uint32_t>(w >> 32) == tag ? static_cast<uint32_t>(w) : 0u;
}

// Gives a sync word this launch's tag (count 0) unless it carries it already.
__device__ __forceinline__ void sync_word_adopt(uint64_t* w, uint32_t tag) {
  const uint64_t fresh = static_cast<uint64_t>(tag) << 32;
  uint64_t cur = ld_relaxed_gpu(w);
  while (static_cast<uint32_t>(cur >> 32) != tag) {
    const uint64_t seen = atom_cas_gpu(w, cur, fresh);
    if (seen == cur) break;
    cur = seen;
  }
}

// 256-element chunks of the activation rows, quantized with the arithmetic of
// nvfp4_quantize_act (per 16-element block: amax, E4M3 scale through the global
// scale g, E2M1 codes): codes row-major, scales in the atom layout. Chunk c = row
// c / (K/256), K chunk c % (K/256); each CTA takes a contiguous range of chunks.
// Lane l holds elements 8l .. 8l+7 of a chunk, so lanes 2j and 2j+1 share block j.
// Needs K % 256 == 0.
// Activation staging of the quantization phase: 16 KB slots (32 chunks) of the
// pipeline's shared memory, filled by bulk copies (warp 0) and encoded by warps
// 1..7, each taking a contiguous part of a slot.
constexpr int kQSlotChunks = 32;
constexpr int kQSlotBytes = kQSlotChunks * 512;
constexpr int kQMaxSlots = 12;
constexpr int kQConsumers = 7;
constexpr int kQPerWarp = (kQSlotChunks + kQConsumers - 1) / kQConsumers;

// `inv_of` holds, for each block scale code s (the amax is >= 0, so s < 128),
// 1 / (value(s) * g) rounded as nvfp4_quantize_act computes it, and 0 where
// value(s) * g == 0 (then all codes are 0): a table read instead of a branch.

// Consumer warp wq's part of a staged slot (chunks cs .. cs + n - 1): chunks
// [wq * 32 / 7, (wq + 1) * 32 / 7) of the slot, read from shared memory and
// encoded branch-free (chunks past the slot's end are predicated off). The
// stages run across all the warp's chunks (every table read before any store),
// so the chunks' dependency chains overlap.
__device__ __forceinline__ void quantize_slot_part(const GemmArgs& a, const uint8_t* slot,
                                                   int64_t cs, int n, int wq, const float* inv_of,
                                                   float cinv, int lane) {
  const int j0 = wq * kQSlotChunks / kQConsumers;
  const int j1 = (wq + 1) * kQSlotChunks / kQConsumers;
  constexpr int P = kQPerWarp;
  uint4 v[P];
  bool valid[P];
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const int j = j0 + i;
    valid[i] = j < j1 && j < n;
    v[i] = valid[i] ? *reinterpret_cast<const uint4*>(slot + j * 512 + lane * 16)
                    : make_uint4(0u, 0u, 0u, 0u);
  }
  uint32_t sc[P];
  float inv[P];
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const float part = bf16x8_amax(v[i].x, v[i].y, v[i].z, v[i].w);
    const float amax = fmaxf(part, __shfl_xor_sync(0xffffffffu, part, 1));
    sc[i] = cvt_e4m3x4(__fmul_rn(amax, cinv), 0.0f, 0.0f, 0.0f) & 0x7Fu;
  }
#pragma unroll
  for (int i = 0; i < P; ++i) inv[i] = inv_of[sc[i]];
  uint32_t codes[P], word[P];
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const float f[8] = {__fmul_rn(bf16_lo(v[i].x), inv[i]), __fmul_rn(bf16_hi(v[i].x), inv[i]),
                        __fmul_rn(bf16_lo(v[i].y), inv[i]), __fmul_rn(bf16_hi(v[i].y), inv[i]),
                        __fmul_rn(bf16_lo(v[i].z), inv[i]), __fmul_rn(bf16_hi(v[i].z), inv[i]),
                        __fmul_rn(bf16_lo(v[i].w), inv[i]), __fmul_rn(bf16_hi(v[i].w), inv[i])};
    codes[i] = inv[i] != 0.0f ? cvt_e2m1x8(f) : 0u;
    // the scales of blocks 4q .. 4q+3 (one 64-element group) sit in lanes 8q,
    // 8q+2, 8q+4, 8q+6; lane 8q writes them as one word
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc[i], 2);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc[i], 4);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc[i], 6);
    word[i] = sc[i] | (s1 << 8) | (s2 << 16) | (s3 << 24);
  }
  const int kc = a.K >> 8;
  int64_t r = (cs + j0) / kc;
  int ck = static_cast<int>(cs + j0 - r * kc);
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const int64_t c = cs + j0 + i;
    if (valid[i]) {
      *reinterpret_cast<uint32_t*>(a.xq + c * 128 + lane * 4) = codes[i];  // row r, bytes 128 ck + 4 l
      if ((lane & 7) == 0)
        *reinterpret_cast<uint32_t*>(a.xs + (r >> 7) * a.kg * kSfAtomBytes + (r & 31) * 16 +
                                     ((r >> 5) & 3) * 4 + (ck * 4 + (lane >> 3)) * kSfAtomBytes) =
            word[i];
    }
    const bool wrap = ++ck == kc;
    ck = wrap ? 0 : ck;
    r += wrap ? 1 : 0;
  }
}

// One weight-scale job: atom `at` (128 rows) of weight tile t for K tile kt, i.e.
// 4 atoms (one per 64-element group) of the layout the GEMM's scale loads read.
// Line l of atom (kg, at) holds group kg of rows 128 at + l, + 32, + 64, + 96 of
// the tile, read from the row-major [N, K/16] scales (16 bytes per row per K
// tile); rows beyond the tile or N are zero.
template <int BN, int NA>
__device__ __forceinline__ void weight_scale_job(const GemmArgs& a, int64_t job, int lane) {
  const int64_t per_tile = static_cast<int64_t>(NA) * a.num_k_tiles;
  const int64_t t = job / per_tile;
  const int at = static_cast<int>((job - t * per_tile) / a.num_k_tiles);
  const int kt = static_cast<int>(job - t * per_tile - static_cast<int64_t>(at) * a.num_k_tiles);
  const int64_t ks = a.K >> 4;
  uint4 v[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int nn = 128 * at + 32 * q + lane;
    const int64_t n = t * BN + nn;
    v[q] = (nn < BN && n < a.N)
               ? __ldg(reinterpret_cast<const uint4*>(a.w_scale + n * ks + kt * 16))
               : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint4 line = g == 0   ? make_uint4(v[0].x, v[1].x, v[2].x, v[3].x)
                       : g == 1 ? make_uint4(v[0].y, v[1].y, v[2].y, v[3].y)
                       : g == 2 ? make_uint4(v[0].z, v[1].z, v[2].z, v[3].z)
                                : make_uint4(v[0].w, v[1].w, v[2].w, v[3].w);
    const int64_t atom = (t * a.kg + kt * 4 + g) * NA + at;
    *reinterpret_cast<uint4*>(a.ws_atoms + atom * kSfAtomBytes + lane * 16) = line;
  }
}

// GELU-quantize epilogue, one lane's row m of one slab (SLAB columns n0 ..):
//   v = bf16(alpha * acc + bias)        (the value the plain epilogue stores as Y)
//   h = bf16(0.5 v * erfc(-v / sqrt 2)) (exact GELU, fp32, erfc form for the tail)
// then h in 16-column blocks as nvfp4_quantize_act quantizes a row (global scale
// g, c = 1 / (6 g)): codes to gq_codes[m, n0/2 ..], the block scales into the atom
// layout of the next layer's activations (K' = N, KG' = N/64 groups of 4 scales).
// Rows in [M, 128-row padding) get zero scales and no codes.
// The GELU of a bf16 value with 2^-16 <= |v| < 2^6 is read from a table of those
// 5632 values (the same formula, evaluated once per CTA). inv_of[s] =
// 1 / (value(s) * g) per block scale code (0: zero codes).
constexpr int kGeluTabExpLo = 127 - 16;  // biased bf16 exponents of the table
constexpr int kGeluTabExps = 22;
constexpr int kGeluTabSize = 2 * kGeluTabExps * 128;

__device__ __forceinline__ float gelu_bf16_formula(float v) {
  constexpr float kRsqrt2 = 0.70710678118654752f;
  const float e = erfcf(__fmul_rn(v, -kRsqrt2));
  return __bfloat162float(__float2bfloat16_rn(__fmul_rn(__fmul_rn(0.5f, v), e)));
}

// Table entry i: sign i / (14 * 128), biased exponent 119 + (i / 128) % 14,
// mantissa i % 128.
__device__ __forceinline__ float gelu_tab_input(int i) {
  const uint32_t sign = static_cast<uint32_t>(i / (kGeluTabExps * 128)) << 15;
  const uint32_t e = static_cast<uint32_t>(kGeluTabExpLo + (i / 128) % kGeluTabExps);
  const uint32_t bits = sign | (e << 7) | static_cast<uint32_t>(i % 128);
  return __uint_as_float(bits << 16);
}

// Branch-free: outside the table, v >= 64 gives v (Phi(v) is 1 in fp32), v <= -64
// gives -0 (v * Phi(v) is below the bf16 range), and |v| < 2^-16 gives 0.5 v: there
// v * Phi(v) = 0.5 v (1 + d) with |d| < 2^-16, and 0.5 v is a bf16 value, so no bf16
// rounding boundary lies between them (up to ties at a subnormal midpoint, which the
// oracle marks as ambiguous). Selects rather than branches keep the 16 elements of a
// block in one basic block, so they interleave (measured: a per-lane branch costs
// 60% more, a table-or-formula branch 2.6x). Nothing here is warp-collective: it
// runs after per-lane returns.
__device__ __forceinline__ float gelu_bf16(float v, const uint16_t* tab) {
  const uint32_t bits = __float_as_uint(v) >> 16;  // v is a bf16 value
  const uint32_t mag = (bits & 0x7FFFu) - (static_cast<uint32_t>(kGeluTabExpLo) << 7);
  const bool in_tab = mag < static_cast<uint32_t>(kGeluTabExps * 128);
  const uint32_t i = in_tab ? mag + (bits >> 15) * (kGeluTabExps * 128) : 0u;
  const float t = __uint_as_float(static_cast<uint32_t>(tab[i]) << 16);
  const bool tiny = (bits & 0x7FFFu) < (static_cast<uint32_t>(kGeluTabExpLo) << 7);
  const float outside = tiny ? __fmul_rn(0.5f, v) : (v > 0.0f ? v : -0.0f);
  return in_tab ? t : outside;
}

template <int SLAB>
__device__ __forceinline__ void gelu_quant_slab(const GemmArgs& a, const uint32_t (&r)[SLAB],
                                                const float* cv_bias_slab, float alpha, int m,
                                                int n0, const uint16_t* gelu_tab,
                                                const float* inv_of, float cinv) {
  const int m_pad = (a.M + 127) & ~127;
  if (m >= m_pad) return;
  const int64_t kg_total = a.N >> 6;
  uint8_t* sc = a.gq_atoms + ((static_cast<int64_t>(m >> 7) * kg_total + (n0 >> 6)) * kSfAtomBytes) +
                (m & 31) * 16 + ((m >> 5) & 3) * 4 + ((n0 & 63) >> 4);
  if (m >= a.M) {
    if constexpr (SLAB == 32)
      *reinterpret_cast<uint16_t*>(sc) = 0;
    else
      *reinterpret_cast<uint32_t*>(sc) = 0u;
    return;
  }
  uint32_t scales = 0;
  uint32_t codes[SLAB / 8];
#pragma unroll
  for (int b = 0; b < SLAB / 16; ++b) {
    float h[16];
    float bias[16];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(&bias[4 * i]) =
          *reinterpret_cast<const float4*>(cv_bias_slab + 16 * b + 4 * i);
    // v = bf16(alpha * acc + bias), two elements per packed fma and conversion
    uint32_t vb[16];  // bf16 bits of v
#pragma unroll
    for (int p2 = 0; p2 < 8; ++p2) {
      const int j = 16 * b + 2 * p2;
      uint32_t o0, o1;
      asm("{\n\t.reg .b64 a, s, c;\n\t"
          "mov.b64 a, {%2, %3};\n\t"
          "mov.b64 s, {%4, %4};\n\t"
          "mov.b64 c, {%5, %6};\n\t"
          "fma.rn.f32x2 a, a, s, c;\n\t"
          "mov.b64 {%0, %1}, a;\n\t}"
          : "=r"(o0), "=r"(o1)
          : "f"(__uint_as_float(r[j])), "f"(__uint_as_float(r[j + 1])), "f"(alpha),
            "f"(bias[2 * p2]), "f"(bias[2 * p2 + 1]));
      // RN-even to bf16 in integer arithmetic (finite values): the conversion pipe is
      // the epilogue's bottleneck, the integer pipe has room
      vb[2 * p2] = (o0 + 0x7FFFu + ((o0 >> 16) & 1u)) >> 16;
      vb[2 * p2 + 1] = (o1 + 0x7FFFu + ((o1 >> 16) & 1u)) >> 16;
    }
    // fast path: every element's GELU from the table (index clamped into it), with
    // a flag for elements outside the table's range
    bool outside = false;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t bits = vb[i];
      const uint32_t mag = (bits & 0x7FFFu) - (static_cast<uint32_t>(kGeluTabExpLo) << 7);
      outside |= mag >= static_cast<uint32_t>(kGeluTabExps * 128);
      const uint32_t idx = min(mag, static_cast<uint32_t>(kGeluTabExps * 128 - 1)) +
                           (bits >> 15) * static_cast<uint32_t>(kGeluTabExps * 128);
      h[i] = __uint_as_float(static_cast<uint32_t>(gelu_tab[idx]) << 16);
    }
    // rare (|v| < 2^-16 or >= 64 somewhere in the block): the exact rule for all 16
    if (outside) {
#pragma unroll
      for (int i = 0; i < 16; ++i) h[i] = gelu_bf16(__uint_as_float(vb[i] << 16), gelu_tab);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(h[i]));
    const uint32_t s = cvt_e4m3x4(__fmul_rn(amax, cinv), 0.0f, 0.0f, 0.0f) & 0x7Fu;
    const float inv = inv_of[s];
    float f0[8], f1[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {  // RN products, two lanes per packed multiply
      asm("{\n\t.reg .b64 a, s;\n\t"
          "mov.b64 s, {%4, %4};\n\t"
          "mov.b64 a, {%2, %3};\n\t"
          "mul.rn.f32x2 a, a, s;\n\t"
          "mov.b64 {%0, %1}, a;\n\t}"
          : "=f"(f0[i]), "=f"(f0[i + 1])
          : "f"(h[i]), "f"(h[i + 1]), "f"(inv));
      asm("{\n\t.reg .b64 a, s;\n\t"
          "mov.b64 s, {%4, %4};\n\t"
          "mov.b64 a, {%2, %3};\n\t"
          "mul.rn.f32x2 a, a, s;\n\t"
          "mov.b64 {%0, %1}, a;\n\t}"
          : "=f"(f1[i]), "=f"(f1[i + 1])
          : "f"(h[8 + i]), "f"(h[8 + i + 1]), "f"(inv));
    }
    codes[2 * b] = inv != 0.0f ? cvt_e2m1x8(f0) : 0u;
    codes[2 * b + 1] = inv != 0.0f ? cvt_e2m1x8(f1) : 0u;
    scales |= s << (8 * b);
  }
  uint8_t* q = a.gq_codes + static_cast<int64_t>(m) * (a.N >> 1) + (n0 >> 1);
#pragma unroll
  for (int i = 0; i < SLAB / 32; ++i)
    *reinterpret_cast<uint4*>(q + 16 * i) =
        make_uint4(codes[4 * i], codes[4 * i + 1], codes[4 * i + 2], codes[4 * i + 3]);
  if constexpr (SLAB == 32)
    *reinterpret_cast<uint16_t*>(sc) = static_cast<uint16_t>(scales);
  else
    *reinterpret_cast<uint32_t*>(sc) = scales;
}

// Kernel modes: the plain GEMM; the single-launch NVFP4 linear (quantization
// phase, grid barrier, GEMM); the GEMM whose epilogue writes NVFP4 codes and scale
// atoms of GELU(Y) instead of Y (the MLP up projection feeding the down projection).
constexpr int kModePlain = 0;
constexpr int kModeSingleLaunch = 1;
constexpr int kModeGeluQuant = 2;

// Epilogue warps: 4 (one per TMEM lane quadrant); the GELU-quantize epilogue,
// which does much more work per element and stages nothing, uses 8 (two per
// quadrant, taking alternate slabs).
template <int MODE>
constexpr int epi_warps() { return MODE == kModeGeluQuant ? 8 : 4; }
// The skinny kernels (AROWS < 128) add one warp after the epilogue warps: it lays out
// the weight scales of each stage in shared memory from the row-major scales.
template <int MODE, int AROWS = kRowsPerCta>
constexpr int block_threads() {
  return MODE == kModeSingleLaunch ? kThreadsFused
                                   : 64 + 32 * epi_warps<MODE>() + (AROWS < kRowsPerCta ? 32 : 0);
}

// F16 (FP8 path, plain mode): the operands are f16 and the MMAs kind::f16.
template <bool FP4, int BN, int CG, int MODE, int AROWS = kRowsPerCta, bool F16 = false>
__global__ void __launch_bounds__(block_threads<MODE, AROWS>(), 1)
qgemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
             const __grid_constant__ CUtensorMap tmap_sfa,
             const __grid_constant__ CUtensorMap tmap_sfb,
             const __grid_constant__ CUtensorMap tmap_y,
             const __grid_constant__ CUtensorMap tmap_lra,
             const __grid_constant__ CUtensorMap tmap_lrb, const GemmArgs args) {
  using C = Cfg<FP4, BN, CG, AROWS>;
  constexpr bool FUSED = MODE == kModeSingleLaunch;
  constexpr bool GQ = MODE == kModeGeluQuant;
  constexpr bool SKINNY = AROWS < kRowsPerCta;
  constexpr int EPI_WARPS = epi_warps<MODE>();
  constexpr int SF_WARP = 2 + EPI_WARPS;  // skinny kernels: the weight-scale warp
  // skinny kernels given the row-major weight scales: SF_WARP writes each stage's
  // scale atoms (no TMA load of them) and is a second arrival on the stage's barrier
  const bool sfb_rm = SKINNY && args.sfb_rowmajor != 0;
  constexpr int EPI_THREADS = 32 * EPI_WARPS;
  constexpr int EPI_HALVES = EPI_WARPS / 4;  // warps per TMEM lane quadrant
  static_assert(!GQ || !C::OVERLAP, "two warps per quadrant need whole accumulator buffers");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* smem_a = smem;
  uint8_t* smem_b = smem_a + C::STAGES * C::A_BYTES;
  uint8_t* smem_sfa = smem_b + C::STAGES * C::B_BYTES;
  uint8_t* smem_sfb = smem_sfa + C::STAGES * C::SFA_BYTES;
  uint8_t* smem_epi = smem_sfb + C::STAGES * C::SFB_BYTES;  // 1024-aligned
  // per-tile column vectors for the epilogue: [2 tiles][bias | column scale][256]
  float* colvec = reinterpret_cast<float*>(smem_epi + C::EPI_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_epi + C::EPI_BYTES + C::COLVEC_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + C::STAGES;
  uint64_t* tfull_bar = bars + 2 * C::STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* drain_bar = tempty_bar + 2;
  uint64_t* never_bar = drain_bar + 1;
  uint64_t* qfull_bar = never_bar + 1;           // fused: staging slot filled
  uint64_t* qfree_bar = qfull_bar + kQMaxSlots;  // fused: staging slot encoded
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qfree_bar + kQMaxSlots);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;  // 0 = leader of the pair
  const bool leader = rank == 0;
  const int group = (CG == 2) ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int ngroups = (CG == 2) ? static_cast<int>(nclusters_x()) : static_cast<int>(gridDim.x);
  const uint64_t deadline = globaltimer_ns() + args.timeout_ns;
  // skinny kernels: the next layer's prologue (a programmatic dependent) may be
  // scheduled now; it waits for this grid to complete before it reads or writes
  // memory, and its launch gap is a large part of a layer this short. (Beside the
  // large persistent GEMMs, early-resident prologue blocks cost more than they save:
  // measured 74.3 -> 76.9 us per step on the 4096 x 3072 x 12288 layer.)
  if constexpr (SKINNY) grid_dependents_launch();
  unsigned long long clk_cycles0 = 0, clk_ns0 = 0;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(clk_cycles0));
    clk_ns0 = globaltimer_ns();
  }

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    if constexpr (FP4) {
      prefetch_tmap(&tmap_sfa);
      if (!sfb_rm) prefetch_tmap(&tmap_sfb);
    }
    if (args.use_tma_store) prefetch_tmap(&tmap_y);
    if (args.lr_k16 > 0) {
      prefetch_tmap(&tmap_lra);
      prefetch_tmap(&tmap_lrb);
    }
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_bar[s], sfb_rm ? 2 : 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], EPI_WARPS * CG);
    }
    mbar_init(drain_bar, 1);
    mbar_init(never_bar, 1);
    if constexpr (FUSED) {
      for (int q = 0; q < kQMaxSlots; ++q) {
        mbar_init(&qfull_bar[q], 1);
        mbar_init(&qfree_bar[q], kQConsumers);
      }
    }
    fence_mbar_init();
    if (SKINNY && args.wait_prior_grid && !args.inject_fault && group < args.total_tiles) {
      // skinny kernels: the weight loads of the first stages go out now, before the
      // TMEM allocation and the block's first barrier (the producer issues the rest)
      int m_blk, n_blk;
      tile_coords(group, args, m_blk, n_blk);
      const int pre = args.num_k_tiles < C::STAGES ? args.num_k_tiles : C::STAGES;
      const uint32_t kTx = C::A_BYTES + C::B_BYTES + C::SFA_BYTES + (sfb_rm ? 0u : C::SFB_BYTES);
      for (int kt = 0; kt < pre; ++kt) {
        mbar_arrive_expect_tx(&full_bar[kt], kTx);
        tma_load_2d(smem_b + kt * C::B_BYTES, &tmap_b, &full_bar[kt], kt * 128, n_blk * BN);
      }
    }
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(tmem_holder, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync_all();  // peer barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // The leader's barriers, addressed from either CTA of the pair.
  const uint32_t full_bar0 = (CG == 2) ? map_to_cta(smem_u32(full_bar), 0) : smem_u32(full_bar);
  const uint32_t tempty_bar0 =
      (CG == 2) ? map_to_cta(smem_u32(tempty_bar), 0) : smem_u32(tempty_bar);

  // Everything above overlaps the tail of the previous kernel on the stream;
  // global inputs are read only after it has completed. In the skinny kernels only
  // the producer waits, and only after it has started the weight loads (the weights
  // and their scales do not come from the previous kernel; the MMA and epilogue
  // warps read nothing it writes).
  // (Plain mode with b_ready: the same, the producer waits after its first B loads.)
  if (args.wait_prior_grid && !SKINNY && !(MODE == kModePlain && args.b_ready))
    grid_dependency_wait();


  bool run = true;
  if (args.inject_fault) {
    run = false;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      if (!mbar_wait_bounded(never_bar, 0, deadline)) record_timeout(args.status);
    }
  }

  if constexpr (FUSED) {
    // thread 0 gives the sync words this launch's tag before any count on them
    if (threadIdx.x == 0) {
      sync_word_adopt(args.sync + kSyncBarrier, args.tag);
      sync_word_adopt(args.sync + kSyncExit, args.tag);
    }
    // 1 / (value(s) * g) per block scale code, in the (still unused) epilogue
    // staging memory
    float* inv_table = reinterpret_cast<float*>(smem_epi);
    if (threadIdx.x < 128) {
      const float d = __fmul_rn(e4m3_to_float(threadIdx.x), __ldg(args.scale_a));
      inv_table[threadIdx.x] = d != 0.0f ? __frcp_rn(d) : 0.0f;
    }
    __syncthreads();
    if (run) {
      // ---------------------------------------------------------- quantization
      // this CTA's contiguous range of activation chunks, staged through the
      // pipeline's shared memory (unused until the GEMM starts) by bulk copies
      const int64_t chunks = static_cast<int64_t>(args.M) * (args.K >> 8);
      const int64_t cb = chunks * blockIdx.x / gridDim.x;
      const int64_t ce = chunks * (blockIdx.x + 1) / gridDim.x;
      const int nslots = static_cast<int>((ce - cb + kQSlotChunks - 1) / kQSlotChunks);
      constexpr int kRing = (C::STAGES * C::STAGE_BYTES) / kQSlotBytes < kQMaxSlots
                                ? (C::STAGES * C::STAGE_BYTES) / kQSlotBytes
                                : kQMaxSlots;
      static_assert(kRing >= 2, "staging ring");
      uint8_t* ring = smem;
      if (warp == 0) {
        if (lane == 0) {
          for (int si = 0; si < nslots; ++si) {
            const int slot = si % kRing;
            const int round = si / kRing;
            if (round > 0 && !mbar_wait_bounded(&qfree_bar[slot], (round - 1) & 1, deadline)) {
              record_timeout(args.status);
              break;
            }
            const int64_t cs = cb + static_cast<int64_t>(si) * kQSlotChunks;
            const int64_t n = ce - cs < kQSlotChunks ? ce - cs : kQSlotChunks;
            mbar_arrive_expect_tx(&qfull_bar[slot], static_cast<uint32_t>(n * 512));
            bulk_load(ring + slot * kQSlotBytes, args.x + cs * 256, static_cast<uint32_t>(n * 512),
                      &qfull_bar[slot]);
          }
        }
        __syncwarp();
      } else {
        const int wq = warp - 1;
        // weight-scale jobs first, while the first slots land
        const int64_t nwq = static_cast<int64_t>(gridDim.x) * kQConsumers;
        const int64_t gwq = static_cast<int64_t>(blockIdx.x) * kQConsumers + wq;
        const int64_t jobs = static_cast<int64_t>(args.tiles_n) * C::NA * args.num_k_tiles;
        for (int64_t j = gwq; j < jobs; j += nwq) weight_scale_job<BN, C::NA>(args, j, lane);
        const float cinv = __frcp_rn(__fmul_rn(6.0f, __ldg(args.scale_a)));
        for (int si = 0; si < nslots; ++si) {
          const int slot = si % kRing;
          if (!warp_wait_bounded(&qfull_bar[slot], (si / kRing) & 1, deadline)) {
            record_timeout(args.status);
            break;
          }
          const int64_t cs = cb + static_cast<int64_t>(si) * kQSlotChunks;
          const int n = static_cast<int>(ce - cs < kQSlotChunks ? ce - cs : kQSlotChunks);
          quantize_slot_part(args, ring + slot * kQSlotBytes, cs, n, wq, inv_table, cinv, lane);
          __syncwarp();
          if (lane == 0) mbar_arrive(&qfree_bar[slot]);
        }
      }
      // the staging memory is the GEMM's next (TMA-written) pipeline memory; this
      // CTA's workspace writes are visible GPU-wide, to TMA reads too, before it counts
      fence_proxy_async_shared();
      __threadfence();
      fence_proxy_async_global();
    }
    __syncthreads();
    int* s_barrier_ok = reinterpret_cast<int*>(tmem_holder + 1);
    if (threadIdx.x == 0) {
      int ok = 1;
      if (run) {
        red_add_release_gpu(args.sync + kSyncBarrier, 1ull);
        uint32_t n = 0;
        while (tagged_count(ld_acquire_gpu(args.sync + kSyncBarrier), args.tag) < gridDim.x) {
          if ((++n & 15u) == 0 && globaltimer_ns() > deadline) {
            ok = 0;
            record_timeout(args.status);
            break;
          }
          __nanosleep(100);
        }
      }
      *s_barrier_ok = ok;
    }
    __syncthreads();
    fence_proxy_async_global();  // the TMA loads below see every CTA's workspace writes
    if (!*s_barrier_ok) run = false;
  }

  if (SKINNY && run && warp == 0) {
    // ------------------------------------------------------------ TMA producer (skinny)
    // As below, one CTA per tile; on the first tile the weight loads of the first
    // stages go out before the wait for the kernel that writes the activations.
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int issued = 0;
    bool waited = !args.wait_prior_grid;
    const uint32_t kTx = C::A_BYTES + C::B_BYTES + C::SFA_BYTES + (sfb_rm ? 0u : C::SFB_BYTES);
    for (int tile = group; ok && tile < args.total_tiles; tile += ngroups) {
      int m_blk, n_blk;
      tile_coords(tile, args, m_blk, n_blk);
      const int a_row = m_blk * C::TILE_M;
      const int b_row = n_blk * BN;
      int pre = 0;
      if (!waited) {
        // stages 0 .. pre-1 of a fresh pipeline: their weight loads went out during
        // the set-up (thread 0); the rest of each stage follows the wait
        pre = args.num_k_tiles < C::STAGES ? args.num_k_tiles : C::STAGES;
        grid_dependency_wait();
        waited = true;
        for (int kt = 0; kt < pre; ++kt) {
          if (elect_one()) {
            tma_load_2d(smem_a + kt * C::A_BYTES, &tmap_a, &full_bar[kt], kt * 128, a_row);
            if constexpr (FP4) {
              tma_load_2d(smem_sfa + kt * C::SFA_BYTES, &tmap_sfa, &full_bar[kt], 0,
                          static_cast<int>(static_cast<int64_t>(m_blk) * args.kg + kt * 4));
              if (!sfb_rm)
                tma_load_2d(smem_sfb + kt * C::SFB_BYTES, &tmap_sfb, &full_bar[kt], 0,
                            static_cast<int>((static_cast<int64_t>(n_blk) * args.kg + kt * 4) *
                                             C::NA));
            }
          }
          __syncwarp();
        }
        issued = pre;
        stage = pre == C::STAGES ? 0 : pre;
        phase = pre == C::STAGES ? 1u : 0u;
      }
      for (int kt = pre; kt < args.num_k_tiles; ++kt) {
        if (!warp_wait_bounded(&empty_bar[stage], phase ^ 1u, deadline)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(&full_bar[stage], kTx);
          tma_load_2d(smem_a + stage * C::A_BYTES, &tmap_a, &full_bar[stage], kt * 128, a_row);
          tma_load_2d(smem_b + stage * C::B_BYTES, &tmap_b, &full_bar[stage], kt * 128, b_row);
          if constexpr (FP4) {
            tma_load_2d(smem_sfa + stage * C::SFA_BYTES, &tmap_sfa, &full_bar[stage], 0,
                        static_cast<int>(static_cast<int64_t>(m_blk) * args.kg + kt * 4));
            if (!sfb_rm)
              tma_load_2d(smem_sfb + stage * C::SFB_BYTES, &tmap_sfb, &full_bar[stage], 0,
                          static_cast<int>((static_cast<int64_t>(n_blk) * args.kg + kt * 4) *
                                           C::NA));
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && args.lr_k16 > 0) {
        // the low-rank branch's operands (AROWS rows of them), as in the kernels below
        if (!warp_wait_bounded(&empty_bar[stage], phase ^ 1u, deadline)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(&full_bar[stage], C::A_BYTES + C::B_BYTES);
          tma_load_2d(smem_a + stage * C::A_BYTES, &tmap_lra, &full_bar[stage], 0, a_row);
          tma_load_2d(smem_b + stage * C::B_BYTES, &tmap_lrb, &full_bar[stage], 0, b_row);
        }
        __syncwarp();
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!waited) grid_dependency_wait();  // no tile: still ordered after the previous kernel
    if (!ok) {
      record_timeout(args.status);
      const uint64_t drain_deadline = globaltimer_ns() + 100000000ull;
      const int n = issued < C::STAGES ? issued : C::STAGES;
      int st = stage;
      uint32_t ph = phase;
      for (int i = 0; i < n; ++i) {
        if (--st < 0) {
          st = C::STAGES - 1;
          ph ^= 1u;
        }
        mbar_wait_bounded(&full_bar[st], ph, drain_deadline);
      }
    }
  } else if (run && warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int issued = 0;
    // b_ready: the first tile's first `pre` stages get their byte counts and weight
    // loads before the wait for the previous kernel (which writes A and its scales)
    int pre = 0;
    if (MODE == kModePlain && args.wait_prior_grid && args.b_ready) {
      if (group < args.total_tiles) {
        int m_blk0, n_blk0;
        tile_coords(group, args, m_blk0, n_blk0);
        const int b_row0 = n_blk0 * BN + static_cast<int>(rank) * C::B_ROWS;
        pre = args.num_k_tiles < C::STAGES ? args.num_k_tiles : C::STAGES;
        const uint32_t kTx0 = C::STAGE_BYTES - C::A_BYTES + args.a_box_rows * 128;
        if (elect_one()) {
          for (int kt = 0; kt < pre; ++kt) {
            uint8_t* sb = smem_b + kt * C::B_BYTES;
            if constexpr (CG == 2) {
              if (leader) mbar_arrive_expect_tx(&full_bar[kt], CG * kTx0);
              tma_load_2d_pair(sb, &tmap_b, full_bar0 + kt * 8u, kt * 128, b_row0);
            } else {
              mbar_arrive_expect_tx(&full_bar[kt], kTx0);
              tma_load_2d(sb, &tmap_b, &full_bar[kt], kt * 128, b_row0);
            }
          }
        }
        __syncwarp();
      }
      grid_dependency_wait();
    }
    for (int tile = group; ok && tile < args.total_tiles; tile += ngroups) {
      int m_blk, n_blk;
      tile_coords(tile, args, m_blk, n_blk);
      const int a_row = m_blk * C::TILE_M + static_cast<int>(rank) * kRowsPerCta;
      const int b_row = n_blk * BN + static_cast<int>(rank) * C::B_ROWS;
      for (int kt = 0; kt < args.num_k_tiles; ++kt) {
        if (!warp_wait_bounded(&empty_bar[stage], phase ^ 1u, deadline)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          const uint32_t fb = full_bar0 + stage * 8u;
          uint8_t* sa = smem_a + stage * C::A_BYTES;
          uint8_t* sb = smem_b + stage * C::B_BYTES;
          uint8_t* ssa = smem_sfa + stage * C::SFA_BYTES;
          uint8_t* ssb = smem_sfb + stage * C::SFB_BYTES;
          // scale atoms: rows of the 2-D atom maps are 512-byte atoms
          const int sfa_atom = static_cast<int>((static_cast<int64_t>(m_blk) * CG + rank) * args.kg +
                                                kt * 4);
          const int sfb_atom = static_cast<int>((static_cast<int64_t>(n_blk) * args.kg + kt * 4) *
                                                C::NA);

          const uint32_t kTx = C::STAGE_BYTES - C::A_BYTES + args.a_box_rows * 128;
          // a prefetched stage already has its byte count and its B load
          const bool fresh = !(tile == group && kt < pre);
          if constexpr (CG == 2) {
            if (leader && fresh) mbar_arrive_expect_tx(&full_bar[stage], CG * kTx);
            tma_load_2d_pair(sa, &tmap_a, fb, kt * 128, a_row);
            if (fresh) tma_load_2d_pair(sb, &tmap_b, fb, kt * 128, b_row);
            if constexpr (FP4) {
              tma_load_2d_pair(ssa, &tmap_sfa, fb, 0, sfa_atom);
              tma_load_2d_pair(ssb, &tmap_sfb, fb, 0, sfb_atom);
            }
          } else {
            if (fresh) mbar_arrive_expect_tx(&full_bar[stage], kTx);
            tma_load_2d(sa, &tmap_a, &full_bar[stage], kt * 128, a_row);
            if (fresh) tma_load_2d(sb, &tmap_b, &full_bar[stage], kt * 128, b_row);
            if constexpr (FP4) {
              tma_load_2d(ssa, &tmap_sfa, &full_bar[stage], 0, sfa_atom);
              tma_load_2d(ssb, &tmap_sfb, &full_bar[stage], 0, sfb_atom);
            }
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && args.lr_k16 > 0) {
        // the low-rank branch's operands, one stage in the A and B areas (same
        // 128-byte rows and swizzle as a K tile; columns r .. 63 read as zeros)
        if (!warp_wait_bounded(&empty_bar[stage], phase ^ 1u, deadline)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          const uint32_t fb = full_bar0 + stage * 8u;
          uint8_t* sa = smem_a + stage * C::A_BYTES;
          uint8_t* sb = smem_b + stage * C::B_BYTES;
          if constexpr (CG == 2) {
            if (leader) mbar_arrive_expect_tx(&full_bar[stage], CG * (C::A_BYTES + C::B_BYTES));
            tma_load_2d_pair(sa, &tmap_lra, fb, 0, a_row);
            tma_load_2d_pair(sb, &tmap_lrb, fb, 0, b_row);
          } else {
            mbar_arrive_expect_tx(&full_bar[stage], C::A_BYTES + C::B_BYTES);
            tma_load_2d(sa, &tmap_lra, &full_bar[stage], 0, a_row);
            tma_load_2d(sb, &tmap_lrb, &full_bar[stage], 0, b_row);
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      record_timeout(args.status);
      // wait (bounded) for the copies still in flight: in a pair their bytes are
      // counted on the leader's full barriers, which the leader drains
      if (leader) {
        const uint64_t drain_deadline = globaltimer_ns() + 100000000ull;
        const int n = issued < C::STAGES ? issued : C::STAGES;
        int s = stage;
        uint32_t p = phase;
        for (int i = 0; i < n; ++i) {
          if (--s < 0) {
            s = C::STAGES - 1;
            p ^= 1u;
          }
          mbar_wait_bounded(&full_bar[s], p, drain_deadline);
        }
      }
    }
  } else if (run && warp == 1 && leader) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    bool issued_any = false;
    for (int tile = group; ok && tile < args.total_tiles; tile += ngroups) {
      // with shared slabs one barrier pair orders consecutive tiles (the next
      // tile's MMAs wait for this tile's shared slab); otherwise one per buffer
      const int bi = C::OVERLAP ? 0 : acc;
      if (!warp_wait_bounded(&tempty_bar[bi], acc_phase ^ 1u, deadline)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::ACC_STRIDE);
      for (int kt = 0; kt < args.num_k_tiles; ++kt) {
        if (!warp_wait_bounded(&full_bar[stage], phase, deadline)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t a_addr = smem_u32(smem_a + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(smem_b + stage * C::B_BYTES);
          if constexpr (FP4) {
            const uint32_t sfa_addr = smem_u32(smem_sfa + stage * C::SFA_BYTES);
            const uint32_t sfb_addr = smem_u32(smem_sfb + stage * C::SFB_BYTES);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint64_t da = smem_desc(sfa_addr + kb * kSfAtomBytes, 0, 128, 0);
              if constexpr (CG == 2)
                tmem_cp_32x128b_x4_pair(tmem_base + C::SFA_COL + kb * 4, da);
              else
                tmem_cp_32x128b_x4(tmem_base + C::SFA_COL + kb * 4, da);
#pragma unroll
              for (int a = 0; a < C::NA; ++a) {
                const uint64_t db = smem_desc(sfb_addr + (kb * C::NA + a) * kSfAtomBytes, 0, 128, 0);
                const uint32_t col = tmem_base + C::SFB_COL + (kb * C::NA + a) * 4;
                if constexpr (CG == 2)
                  tmem_cp_32x128b_x4_pair(col, db);
                else
                  tmem_cp_32x128b_x4(col, db);
              }
            }
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint64_t ad = smem_desc(a_addr + kb * 32, 16, 1024, 2);
              const uint64_t bd = smem_desc(b_addr + kb * 32, 16, 1024, 2);
              const uint32_t sfa = tmem_base + C::SFA_COL + kb * 4;
              const uint32_t sfb = tmem_base + C::SFB_COL + kb * C::NA * 4;
              const uint32_t accum = (kt | kb) != 0 ? 1u : 0u;
              if constexpr (CG == 2)
                mma_nvf4_pair(d_tmem, ad, bd, C::IDESC, sfa, sfb, accum);
              else
                mma_nvf4(d_tmem, ad, bd, C::IDESC, sfa, sfb, accum);
            }
          } else {
            // 32 bytes of K per MMA: 32 E4M3 elements (kind::f8f6f4) or 16 f16
            // elements (kind::f16); the instruction descriptor is the same word
            // (E4M3 and f16 are both format 0 of their kinds)
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint64_t ad = smem_desc(a_addr + kb * 32, 16, 1024, 2);
              const uint64_t bd = smem_desc(b_addr + kb * 32, 16, 1024, 2);
              const uint32_t accum = (kt | kb) != 0 ? 1u : 0u;
              if constexpr (F16) {
                if constexpr (CG == 2)
                  mma_bf16_pair(d_tmem, ad, bd, C::IDESC, accum);
                else
                  mma_bf16(d_tmem, ad, bd, C::IDESC, accum);
              } else {
                if constexpr (CG == 2)
                  mma_f8f6f4_pair(d_tmem, ad, bd, C::IDESC, accum);
                else
                  mma_f8f6f4(d_tmem, ad, bd, C::IDESC, accum);
              }
            }
          }
          // frees the stage (in both CTAs of a pair) once these MMAs have read it
          if constexpr (CG == 2)
            tc_commit_pair(&empty_bar[stage], 0x3);
          else
            tc_commit(&empty_bar[stage]);
        }
        __syncwarp();
        issued_any = true;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && FP4 && args.lr_k16 > 0) {
        // low-rank up projection: (D / alpha) x up^T, bf16, K = 16 per MMA, into the
        // same accumulator (always accumulating: the K tiles came first)
        if (!warp_wait_bounded(&full_bar[stage], phase, deadline)) {
          ok = false;
        } else {
          tc_fence_after();
          if (elect_one()) {
            const uint32_t a_addr = smem_u32(smem_a + stage * C::A_BYTES);
            const uint32_t b_addr = smem_u32(smem_b + stage * C::B_BYTES);
            for (int kb = 0; kb < args.lr_k16; ++kb) {
              const uint64_t ad = smem_desc(a_addr + kb * 32, 16, 1024, 2);
              const uint64_t bd = smem_desc(b_addr + kb * 32, 16, 1024, 2);
              if constexpr (CG == 2)
                mma_bf16_pair(d_tmem, ad, bd, C::IDESC_BF16, 1u);
              else
                mma_bf16(d_tmem, ad, bd, C::IDESC_BF16, 1u);
            }
            if constexpr (CG == 2)
              tc_commit_pair(&empty_bar[stage], 0x3);
            else
              tc_commit(&empty_bar[stage]);
          }
          __syncwarp();
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) break;
      if (elect_one()) {  // accumulator ready for the epilogue (of both CTAs)
        if constexpr (CG == 2)
          tc_commit_pair(&tfull_bar[bi], 0x3);
        else
          tc_commit(&tfull_bar[bi]);
      }
      __syncwarp();
      acc ^= 1;
      if (C::OVERLAP || acc == 0) acc_phase ^= 1u;
    }
    if (!ok) {
      record_timeout(args.status);
      if (issued_any) {  // wait (bounded) for this thread's MMAs and copies to finish
        if (elect_one()) {
          if constexpr (CG == 2)
            tc_commit_pair(drain_bar, 0x1);
          else
            tc_commit(drain_bar);
        }
        __syncwarp();
        mbar_wait_bounded(drain_bar, 0, globaltimer_ns() + 100000000ull);
      }
    }
  } else if (run && warp >= 2 && warp < 2 + EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const int q = warp % 4;  // TMEM lane quadrant this warp may access
    const int half = (warp - 2) / 4;  // which of the quadrant's warps: slabs it % EPI_HALVES
    const int row_in_tile = static_cast<int>(rank) * kRowsPerCta + q * 32 + lane;
    uint8_t* stage = smem_epi + (warp - 2) * C::EPI_BUFS * kEpiBufBytes;
    int buf = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    float alpha = 1.0f;
    if constexpr (FP4) alpha = __fmul_rn(__ldg(args.scale_a), __ldg(args.scale_b));
    // GELU-quantize: 1 / (6 g), and the GELU and block-reciprocal tables in the
    // staging memory (this mode stores no Y through it)
    float gq_c = 0.0f;
    uint16_t* gelu_tab = reinterpret_cast<uint16_t*>(smem_epi);
    float* inv_of = reinterpret_cast<float*>(smem_epi + kGeluTabSize * 2);
    if constexpr (GQ) {
      static_assert(kGeluTabSize * 2 + 128 * 4 <= C::EPI_BYTES, "tables fit the staging memory");
      const float g = __ldg(args.gq_scale);
      gq_c = __frcp_rn(__fmul_rn(6.0f, g));
      const int t = threadIdx.x - 64;  // 0 .. EPI_THREADS - 1
      for (int i = t; i < kGeluTabSize; i += EPI_THREADS)
        gelu_tab[i] = static_cast<uint16_t>(__float_as_uint(gelu_bf16_formula(gelu_tab_input(i))) >> 16);
      if (t < 128) {
        const float d = __fmul_rn(e4m3_to_float(static_cast<uint32_t>(t)), g);
        inv_of[t] = d != 0.0f ? __frcp_rn(d) : 0.0f;
      }
      asm volatile("bar.sync 2, %0;" ::"n"(EPI_THREADS) : "memory");
    }
    int titer = 0;
    for (int tile = group; tile < args.total_tiles; tile += ngroups, ++titer) {
      int m_blk, n_blk;
      tile_coords(tile, args, m_blk, n_blk);
      const int bi = C::OVERLAP ? 0 : acc;
      // the tile's bias and column scales into shared memory (double-buffered by
      // tile), loaded by the 128 epilogue threads while the accumulator is
      // still being computed; one barrier among the epilogue warps per tile (all
      // of them have finished the previous tile, whose buffer the next load uses)
      float* cv_bias = colvec + (titer & 1) * 512;
      float* cv_scale = cv_bias + 256;
      for (int j = threadIdx.x - 64; j < BN; j += EPI_THREADS) {
        const int n = n_blk * BN + j;
        const bool in = n < args.N;
        cv_bias[j] = (args.bias && in) ? __ldg(args.bias + n) : 0.0f;
        if constexpr (!FP4) cv_scale[j] = in ? __ldg(args.scale_b + n) : 0.0f;
      }
      const bool ready = warp_wait_bounded(&tfull_bar[bi], acc_phase, deadline);
      // publishes the column vectors to all epilogue warps, and makes every
      // epilogue warp leave together if any wait expired
      if (barrier1_any<EPI_THREADS>(!ready)) {
        record_timeout(args.status);
        break;
      }
      tc_fence_after();
      const int m = m_blk * C::TILE_M + row_in_tile;
      const int row0 = m_blk * C::TILE_M + static_cast<int>(rank) * kRowsPerCta + q * 32;
      float row_scale = 1.0f;
      if constexpr (!FP4) row_scale = (m < args.M) ? __ldg(args.scale_a + m) : 0.0f;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * C::ACC_STRIDE);
      // a warp whose 32 rows all lie past M has nothing to store (the GELU-quantize
      // epilogue still writes their zero scales): hand the buffer back at once
      const bool rows_out = !GQ && row0 >= args.M;
      if (rows_out) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_bar0 + bi * 8u);
      }
#pragma unroll 1
      for (int it = 0; it < (rows_out ? 0 : C::NSLAB); ++it) {
        if (EPI_HALVES > 1 && it % EPI_HALVES != half) continue;  // warp-uniform
        // slab order: with shared slabs, buffer 0 drains its last slab (the shared
        // one) first; otherwise slabs go in order
        const int sl = (C::OVERLAP && acc == 0) ? (it + C::NSLAB - 1) % C::NSLAB : it;
        uint32_t r[C::SLAB];
        __syncwarp();  // tcgen05.ld is warp-collective
#pragma unroll
        for (int h = 0; h < C::SLAB / 32; ++h)
          tmem_ld_32x32b_x32(tbase + sl * C::SLAB + 32 * h,
                             *reinterpret_cast<uint32_t(*)[32]>(&r[32 * h]));
        tmem_ld_wait();
        // hand the buffer back once the MMA can no longer overwrite unread columns:
        // after the shared slab, or after this warp's last slab
        if (C::OVERLAP ? it == 0 : it + EPI_HALVES >= C::NSLAB) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_bar0 + bi * 8u);
        }
        const int n0 = n_blk * BN + sl * C::SLAB;
        if (n0 >= args.N) continue;  // warp-uniform
        if constexpr (GQ) {
          gelu_quant_slab<C::SLAB>(args, r, cv_bias + sl * C::SLAB, alpha, m, n0, gelu_tab, inv_of,
                                   gq_c);
          continue;
        }
        if (args.use_tma_store) {
          // columns n0 .. n0+SLAB-1 of this warp's 32 rows: scale, bias, bf16, into a
          // swizzled staging tile, then one TMA store per warp.
          uint32_t packed[C::SLAB / 2];
#pragma unroll
          for (int i = 0; i < C::SLAB / 4; ++i) {
            const int j = sl * C::SLAB + 4 * i;  // column within the tile
            const float4 b4 = *reinterpret_cast<const float4*>(cv_bias + j);
            float4 s4 = make_float4(alpha, alpha, alpha, alpha);
            if constexpr (!FP4) {
              const float4 w4 = *reinterpret_cast<const float4*>(cv_scale + j);
              s4 = make_float4(__fmul_rn(row_scale, w4.x), __fmul_rn(row_scale, w4.y),
                               __fmul_rn(row_scale, w4.z), __fmul_rn(row_scale, w4.w));
            }
            packed[2 * i] = pack_bf16(__fmaf_rn(__uint_as_float(r[4 * i]), s4.x, b4.x),
                                      __fmaf_rn(__uint_as_float(r[4 * i + 1]), s4.y, b4.y));
            packed[2 * i + 1] = pack_bf16(__fmaf_rn(__uint_as_float(r[4 * i + 2]), s4.z, b4.z),
                                          __fmaf_rn(__uint_as_float(r[4 * i + 3]), s4.w, b4.w));
          }
          uint8_t* sbuf = stage + buf * kEpiBufBytes;
          if (lane == 0) {  // the store that last used this buffer has read it
            if constexpr (C::EPI_BUFS == 1)
              bulk_wait_group_read<0>();
            else
              bulk_wait_group_read<1>();
          }
          __syncwarp();
          // 16-byte chunk j of row `lane` goes to chunk j ^ f(row), the TMA's swizzle
          // (128-byte rows: f = row % 8; 64-byte rows: f = (row / 2) % 4)
#pragma unroll
          for (int j = 0; j < C::SLAB / 8; ++j) {
            const int pos = (C::SLAB == 64) ? (j ^ (lane & 7)) : (j ^ ((lane >> 1) & 3));
            *reinterpret_cast<uint4*>(sbuf + lane * (C::SLAB * 2) + pos * 16) =
                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmap_y, sbuf, n0, row0);
            bulk_commit_group();
          }
          buf = (buf + 1) % C::EPI_BUFS;
        } else {
          if (m >= args.M) continue;
          uint16_t* yrow = args.y + static_cast<int64_t>(m) * args.N;
#pragma unroll
          for (int i = 0; i < C::SLAB; ++i) {
            const int n = n0 + i;
            if (n < args.N) {
              const float sc = FP4 ? alpha : __fmul_rn(row_scale, __ldg(args.scale_b + n));
              const float b = args.bias ? __ldg(args.bias + n) : 0.0f;
              const __nv_bfloat16 h = __float2bfloat16_rn(__fmaf_rn(__uint_as_float(r[i]), sc, b));
              yrow[n] = *reinterpret_cast<const uint16_t*>(&h);
            }
          }
        }
      }
      acc ^= 1;
      if (C::OVERLAP || acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_group_all();  // outstanding stores complete before exit
  } else if (SKINNY && run && warp == SF_WARP && sfb_rm) {
    // ------------------------------------------------------------ weight scales (skinny)
    // Per stage: the 16 scales of each of the tile's BN weight rows for the stage's
    // K tile (row-major [N, K/16], 16 bytes per row), rearranged into the 4 atoms
    // the MMA's scale copies read (atom g, line l: group g of rows l, l+32, l+64,
    // l+96); rows past the tile or N are zero. Lane l holds rows l + 32 j. The
    // loads of a stage go out before the wait for its slot.
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    const int64_t ks = args.ks_bytes;
    for (int tile = group; ok && tile < args.total_tiles; tile += ngroups) {
      int m_blk, n_blk;
      tile_coords(tile, args, m_blk, n_blk);
      for (int kt = 0; kt < args.num_k_tiles; ++kt) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int nn = lane + 32 * j;
          const int64_t n = static_cast<int64_t>(n_blk) * BN + nn;
          v[j] = make_uint4(0u, 0u, 0u, 0u);
          if (nn < BN && n < args.N) {
            const uint8_t* src = args.w_scale + n * ks + kt * 16;
            if (args.sfb_vec16) {
              v[j] = __ldg(reinterpret_cast<const uint4*>(src));
            } else {
              uint32_t w[4] = {0u, 0u, 0u, 0u};
              for (int b = 0; b < 16; ++b)
                if (kt * 16 + b < ks) w[b >> 2] |= static_cast<uint32_t>(__ldg(src + b)) << (8 * (b & 3));
              v[j] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        if (!warp_wait_bounded(&empty_bar[stage], phase ^ 1u, deadline)) {
          ok = false;
          break;
        }
        uint8_t* ssb = smem_sfb + stage * C::SFB_BYTES;
        *reinterpret_cast<uint4*>(ssb + 0 * kSfAtomBytes + lane * 16) = make_uint4(v[0].x, v[1].x, v[2].x, v[3].x);
        *reinterpret_cast<uint4*>(ssb + 1 * kSfAtomBytes + lane * 16) = make_uint4(v[0].y, v[1].y, v[2].y, v[3].y);
        *reinterpret_cast<uint4*>(ssb + 2 * kSfAtomBytes + lane * 16) = make_uint4(v[0].z, v[1].z, v[2].z, v[3].z);
        *reinterpret_cast<uint4*>(ssb + 3 * kSfAtomBytes + lane * 16) = make_uint4(v[0].w, v[1].w, v[2].w, v[3].w);
        fence_proxy_async_shared();  // the MMA thread's scale copies read these bytes
        __syncwarp();
        if (lane == 0) mbar_arrive(&full_bar[stage]);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && args.lr_k16 > 0) {  // the low-rank stage needs this warp's arrival too
        if (!warp_wait_bounded(&empty_bar[stage], phase ^ 1u, deadline)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive(&full_bar[stage]);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) record_timeout(args.status);
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    unsigned long long c1;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(c1));
    g_gemm_clock[0] = c1 - clk_cycles0;
    g_gemm_clock[1] = globaltimer_ns() - clk_ns0;
  }
  if constexpr (CG == 2) cluster_sync_all();  // no peer accesses this CTA's memory any more
  if constexpr (FUSED) {
    // this CTA is done with the sync words; the last CTA out resets them
    if (threadIdx.x == 0) {
      __threadfence();
      const uint64_t old = atom_add_relaxed_gpu(args.sync + kSyncExit, 1ull);
      if (tagged_count(old, args.tag) + 1u == gridDim.x) {
        __threadfence();
        for (int i = 0; i < args.sync_words; ++i) st_relaxed_gpu(args.sync + i, 0ull);
      }
    }
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2)
      tmem_dealloc_pair(tmem_base, kTmemCols);
    else
      tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool encode_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
               uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
               CUtensorMapSwizzle swz, CUtensorMapL2promotion promo) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, promo,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <bool FP4, int BN, int CG, int MODE, int AROWS = kRowsPerCta, bool F16 = false>
cudaError_t launch_typed(const GemmProblem& p, cudaStream_t stream) {
  using Cf = Cfg<FP4, BN, CG, AROWS>;
  constexpr bool FUSED = MODE == kModeSingleLaunch;
  static_assert(!F16 || (!FP4 && MODE == kModePlain), "f16 operands: FP8 path, plain mode");
  auto kern = qgemm_kernel<FP4, BN, CG, MODE, AROWS, F16>;
  if (p.f16_operands != F16) return cudaErrorInvalidValue;
  if (AROWS < kRowsPerCta && p.M > AROWS) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && !attr_set[dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

  const int64_t k_bytes = FP4 ? p.K / 2 : (F16 ? 2 * p.K : p.K);
  CUtensorMap ta, tb, tsa, tsb, ty, tla, tlb;
  std::memset(&tla, 0, sizeof(tla));
  std::memset(&tlb, 0, sizeof(tlb));
  std::memset(&tsa, 0, sizeof(tsa));
  std::memset(&tsb, 0, sizeof(tsb));
  std::memset(&ty, 0, sizeof(ty));
  // A / B: uint8 rows of K* bytes, boxes of [rows, 128 bytes], 128-byte swizzle; a
  // lone CTA with fewer than 128 rows of A loads only those (whole 8-row swizzle
  // atoms), the plain FP4 mode only (its A scale atoms zero the rows past M)
  const int a_box_rows = AROWS < kRowsPerCta ? AROWS
                         : (CG == 1 && FP4 && MODE == kModePlain && p.M < kRowsPerCta)
                             ? static_cast<int>((p.M + 7) / 8 * 8)
                             : kRowsPerCta;
  if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.a, k_bytes, p.M, k_bytes, 128,
                 static_cast<uint32_t>(a_box_rows), CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.b, k_bytes, p.N, k_bytes, 128, Cf::B_ROWS,
                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return cudaErrorInvalidValue;
  const int64_t kg = sf_kgroups(p.K);
  const bool sfb_rm = AROWS < kRowsPerCta && FP4 && MODE == kModePlain && p.w_scale != nullptr;
  if (FP4) {
    // scale atoms as rows of 128 32-bit words; one stage = 4 (A) or 4 * NA (B) atoms
    const int64_t a_atoms = ceil_div64(p.M, kRowsPerCta) * kg;
    const int64_t b_atoms = ceil_div64(p.N, BN) * kg * Cf::NA;
    if (!encode_2d(&tsa, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.sfa, 128, a_atoms, kSfAtomBytes, 128, 4,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
      return cudaErrorInvalidValue;
    if (!sfb_rm &&
        !encode_2d(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.sfb, 128, b_atoms, kSfAtomBytes,
                   128, 4 * Cf::NA, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B)) {
      return cudaErrorInvalidValue;
    }
  }
  const bool tma_store = MODE != kModeGeluQuant && (p.N % 8) == 0 &&
                         (reinterpret_cast<uintptr_t>(p.y) & 15) == 0;
  if (tma_store &&
      !encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.y, p.N, p.M, p.N * 2, Cf::SLAB, 32,
                 Cf::SLAB == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                 CU_TENSOR_MAP_L2_PROMOTION_NONE))
    return cudaErrorInvalidValue;

  const bool lowrank = FP4 && MODE == kModePlain && p.lr_rank > 0;
  if (lowrank) {
    // bf16 [rows, r] with 128-byte boxes of 64 elements: columns r .. 63 read as zeros
    if (p.lr_rank > 64 || p.lr_rank % 8 != 0 || !p.lr_act || !p.lr_up ||
        !encode_2d(&tla, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.lr_act, p.lr_rank, p.M,
                   p.lr_rank * 2, 64, AROWS, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
        !encode_2d(&tlb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.lr_up, p.lr_rank, p.N,
                   p.lr_rank * 2, 64, Cf::B_ROWS, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
      return cudaErrorInvalidValue;
  }

  GemmArgs a{};
  a.a_box_rows = a_box_rows;
  if (sfb_rm) {
    a.sfb_rowmajor = 1;
    a.w_scale = p.w_scale;
    a.ks_bytes = static_cast<int>(p.K / 16);
    a.sfb_vec16 = (p.K % 256 == 0 && (reinterpret_cast<uintptr_t>(p.w_scale) & 15) == 0) ? 1 : 0;
  }
  a.lr_k16 = lowrank ? (p.lr_rank + 15) / 16 : 0;
  a.M = static_cast<int>(p.M);
  a.N = static_cast<int>(p.N);
  a.K = static_cast<int>(p.K);
  a.tiles_m = static_cast<int>(ceil_div64(p.M, Cf::TILE_M));
  a.tiles_n = static_cast<int>(ceil_div64(p.N, BN));
  // a K tile is 128 bytes of every row: 256 E2M1, 128 E4M3 or 64 f16 elements
  a.num_k_tiles = static_cast<int>(ceil_div64(k_bytes, 128));
  a.total_tiles = a.tiles_m * a.tiles_n;
  a.kg = kg;
  a.scale_a = p.scale_a;
  a.scale_b = p.scale_b;
  a.bias = p.bias;
  a.y = static_cast<uint16_t*>(p.y);
  a.status = p.status;
  a.timeout_ns = p.timeout_ns;
  a.inject_fault = p.inject_fault;
  a.wait_prior_grid = p.pdl ? 1 : 0;
  a.b_ready = (MODE == kModePlain && p.b_ready) ? 1 : 0;
  a.use_tma_store = tma_store ? 1 : 0;
  a.raster_n = 0;
  if (MODE == kModeGeluQuant) {
    a.gq_codes = p.gq_codes;
    a.gq_atoms = p.gq_atoms;
    a.gq_scale = p.gq_scale;
  }
  if (FUSED) {
    a.x = static_cast<const uint16_t*>(p.x);
    a.xq = static_cast<uint8_t*>(const_cast<void*>(p.a));
    a.xs = const_cast<uint8_t*>(p.sfa);
    a.w_scale = p.w_scale;
    a.ws_atoms = const_cast<uint8_t*>(p.sfb);
    a.sync = p.sync;
    a.sync_words = 8;  // the whole 64-byte region, so that the call leaves all of it zero
    a.tag = p.tag;
  }

  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(block_threads<MODE, AROWS>());
  cfg.dynamicSmemBytes = Cf::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int nattr = 0;
  if (CG == 2) {
    attr[nattr].id = cudaLaunchAttributeClusterDimension;
    attr[nattr].val.clusterDim.x = 2;
    attr[nattr].val.clusterDim.y = 1;
    attr[nattr].val.clusterDim.z = 1;
    ++nattr;
  }
  // Persistent grid: as many CTA groups as can be resident at once (pairs need two
  // free SMs of one GPC, so fewer than SMs / 2 pairs may fit).
  static std::atomic<int> resident_groups[64] = {};
  int max_groups = sms / CG;
  if (dev < 64 && resident_groups[dev].load(std::memory_order_relaxed) == 0) {
    int n = max_groups;
    if (CG == 2) {
      cfg.gridDim = dim3(static_cast<unsigned>(max_groups * CG));
      cfg.attrs = attr;
      cfg.numAttrs = nattr;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = max_groups;
      }
    }
    resident_groups[dev].store(n < max_groups ? n : max_groups, std::memory_order_relaxed);
  }
  if (dev < 64) max_groups = resident_groups[dev].load(std::memory_order_relaxed);
  const int groups = a.total_tiles < max_groups ? a.total_tiles : max_groups;
  cfg.gridDim = dim3(static_cast<unsigned>(groups * CG));
  if (p.pdl) {
    attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[nattr].val.programmaticStreamSerializationAllowed = 1;
    ++nattr;
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, tsa, tsb, ty, tla, tlb, a);
}

}  // namespace

namespace {
std::atomic<int> g_force_bn{0};
std::atomic<int> g_force_cg{0};
}  // namespace

cudaError_t read_gemm_clock(unsigned long long* cycles, unsigned long long* ns) {
  unsigned long long v[2] = {0, 0};
  const cudaError_t e = cudaMemcpyFromSymbol(v, g_gemm_clock, sizeof(v));
  *cycles = v[0];
  *ns = v[1];
  return e;
}

bool set_tile_override(int bn, int cg) {
  if (bn == 0) {
    g_force_bn.store(0);
    g_force_cg.store(0);
    return true;
  }
  if ((bn != 64 && bn != 96 && bn != 128 && bn != 192 && bn != 224 && bn != 256) ||
      (cg != 1 && cg != 2) || (bn < 128 && cg != 1))
    return false;
  g_force_cg.store(cg);
  g_force_bn.store(bn);
  return true;
}

// Rows of A per pipeline stage of the skinny FP4 kernels for M rows (0: none).
static int skinny_rows(bool fp4, int64_t M, bool whole_buffers) {
  if (!fp4 || whole_buffers || M > 64) return 0;
  return M <= 16 ? 16 : (M <= 32 ? 32 : 64);
}

GemmConfig choose_config(bool fp4, int64_t M, int64_t N, int64_t K, bool whole_buffers,
                         bool allow_skinny) {
  GemmConfig c{};
  const int sk = skinny_rows(fp4, M, whole_buffers || !allow_skinny);
  if (g_force_bn.load() != 0) {
    c.bn = g_force_bn.load();
    c.cg = g_force_cg.load();
    if (whole_buffers && c.bn == 256) c.bn = 224;
    // skinny stages with one CTA per tile of at most 128 columns; narrower tiles
    // exist only as skinny kernels
    c.arows = (c.cg == 1 && c.bn <= 128) ? sk : 0;
    if (c.bn < 128 && c.arows == 0) c.bn = 128;
    return c;
  }
  // Skinny layers (M <= 64, FP4): one CTA per tile with stages holding only 16 / 32 /
  // 64 rows of A, and the narrowest tile width that keeps the tiles in one wave of
  // 148 SMs (the weight streams through as many SMs as possible).
  c.arows = sk;
  if (c.arows > 0) {
    c.cg = 1;
    c.bn = 256;
    for (int bn : {64, 96, 128, 192, 224, 256}) {
      if (ceil_div64(N, bn) <= 148) {
        c.bn = bn;
        break;
      }
    }
    if (c.bn > 128) c.arows = 0;  // wide tiles: the ordinary kernels
    if (c.arows > 0) return c;
  }
  // CTA pairs once there are two 128-row blocks to pair. Tile width from a cost
  // model fitted to B200 measurements: waves over the resident groups x (K steps
  // x operand KB one group loads per K step), plus a fixed per-tile cost for the
  // 256-column FP4 tile, whose TMEM buffers share a slab (the next tile's MMAs
  // wait for the epilogue to drain it; about 1.5 us, worth ~240 KB of loads).
  c.cg = M >= 512 ? 2 : 1;
  const int64_t groups = c.cg == 2 ? 74 : 148;
  const int64_t tiles_m = ceil_div64(M, 128 * c.cg);
  const int64_t ksteps = ceil_div64(K, fp4 ? kKTileFp4 : kKTileFp8);
  double best = 0.0;
  c.bn = 128;
  for (int bn : {128, 192, 224, 256}) {
    if (whole_buffers && fp4 && bn == 256) continue;  // the shared-slab tile
    const int64_t tiles = tiles_m * ceil_div64(N, bn);
    const int64_t waves = ceil_div64(tiles, groups);
    const int na = (bn + 127) / 128;
    const double kb = c.cg * 16.0 + bn * 0.125 + (fp4 ? c.cg * (2.0 + 2.0 * na) : 0.0);
    const double per_tile = static_cast<double>(ksteps) * kb + ((fp4 && bn == 256) ? 240.0 : 0.0);
    const double cost = static_cast<double>(waves) * per_tile;
    if (best == 0.0 || cost < best * 0.999) {
      best = cost;
      c.bn = bn;
    }
  }
  return c;
}

cudaError_t launch_gemm(const GemmProblem& p, cudaStream_t stream) {
  if (p.gelu_quant) {
    if (!p.fp4 || p.fused || !p.gq_codes || !p.gq_atoms || !p.gq_scale || p.N % 256 != 0)
      return cudaErrorInvalidValue;
#define QL_GCASE(BN_, CG_) \
  if (p.bn == BN_ && p.cg == CG_) return launch_typed<true, BN_, CG_, kModeGeluQuant>(p, stream);
    QL_GCASE(128, 1)
    QL_GCASE(192, 1)
    QL_GCASE(224, 1)
    QL_GCASE(128, 2)
    QL_GCASE(192, 2)
    QL_GCASE(224, 2)
#undef QL_GCASE
    return cudaErrorInvalidValue;
  }
  if (p.fused) {
    if (!p.fp4 || !p.x || !p.w_scale || !p.sync || p.K % kKTileFp4 != 0) return cudaErrorInvalidValue;
#define QL_FCASE(BN_, CG_) \
  if (p.bn == BN_ && p.cg == CG_) return launch_typed<true, BN_, CG_, kModeSingleLaunch>(p, stream);
    QL_FCASE(128, 1)
    QL_FCASE(192, 1)
    QL_FCASE(224, 1)
    QL_FCASE(256, 1)
    QL_FCASE(128, 2)
    QL_FCASE(192, 2)
    QL_FCASE(224, 2)
    QL_FCASE(256, 2)
#undef QL_FCASE
    return cudaErrorInvalidValue;
  }
  if (p.arows > 0) {
    if (!p.fp4 || p.cg != 1) return cudaErrorInvalidValue;
#define QL_SCASE(BN_, AR_) \
  if (p.bn == BN_ && p.arows == AR_) return launch_typed<true, BN_, 1, kModePlain, AR_>(p, stream);
    QL_SCASE(64, 16)
    QL_SCASE(64, 32)
    QL_SCASE(64, 64)
    QL_SCASE(96, 16)
    QL_SCASE(96, 32)
    QL_SCASE(96, 64)
    QL_SCASE(128, 16)
    QL_SCASE(128, 32)
    QL_SCASE(128, 64)
#undef QL_SCASE
    return cudaErrorInvalidValue;
  }
  if (p.f16_operands) {
    if (p.fp4) return cudaErrorInvalidValue;
#define QL_HCASE(BN_, CG_) \
  if (p.bn == BN_ && p.cg == CG_)    \
    return launch_typed<false, BN_, CG_, kModePlain, kRowsPerCta, true>(p, stream);
    QL_HCASE(128, 1)
    QL_HCASE(192, 1)
    QL_HCASE(256, 1)
    QL_HCASE(224, 1)
    QL_HCASE(224, 2)
    QL_HCASE(128, 2)
    QL_HCASE(192, 2)
    QL_HCASE(256, 2)
#undef QL_HCASE
    return cudaErrorInvalidValue;
  }
#define QL_CASE(FP4_, BN_, CG_) \
  if (p.fp4 == FP4_ && p.bn == BN_ && p.cg == CG_) return launch_typed<FP4_, BN_, CG_, kModePlain>(p, stream);
  QL_CASE(true, 128, 1)
  QL_CASE(true, 192, 1)
  QL_CASE(true, 256, 1)
  QL_CASE(true, 224, 1)
  QL_CASE(true, 224, 2)
  QL_CASE(true, 128, 2)
  QL_CASE(true, 192, 2)
  QL_CASE(true, 256, 2)
  QL_CASE(false, 128, 1)
  QL_CASE(false, 192, 1)
  QL_CASE(false, 256, 1)
  QL_CASE(false, 224, 1)
  QL_CASE(false, 224, 2)
  QL_CASE(false, 128, 2)
  QL_CASE(false, 192, 2)
  QL_CASE(false, 256, 2)
#undef QL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ql
