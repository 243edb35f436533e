// Prologue of the SVDQuant-style NVFP4 linear ("Bringing Nunchaku 4-bit Diffusion
// Inference to Diffusers", section "Background: SVDQuant and Nunchaku": a small
// 16-bit low-rank branch next to the 4-bit residual, with the low-rank down
// projection sharing its pass over x with the quantization), in one launch that
// reads x once:
//   xs = bf16(RN32(x * smooth))                      (smooth may be absent: xs = x)
//   NVFP4 codes and scale atoms of xs                (the nvfp4_linear prologue's rule)
//   lr_act[m, j] = bf16(D[m, j] / alpha),  D = xs down^T,  alpha = input_scale *
//                                                      weight_scale_2, j < rank
//   weight block scales -> atom layout               (as in the nvfp4_linear prologue)
// lr_act is the form the GEMM's low-rank K step reads (it scales the whole
// accumulator by alpha).
//
// One CTA of 8 warps per 16-row group. The group's x comes in by TMA, in stages of
// 8 boxes of 16 rows x 64 columns (128-byte swizzled), kSvStages stages in flight;
// warp w takes box w of every stage (64-column groups kg = w, w + 8, ...), and the
// last warp to have read a stage slot issues the load that refills it (a counter
// per slot in shared memory), so no warp waits for the others.
// Per box, thread (g = lane / 4, t = lane % 4) holds rows g and g + 8 at columns
// 16t .. 16t + 15, which is one NVFP4 block of each row, and feeds the same
// registers to warp-level bf16 MMAs (m16n8k16, fp32 accumulation) against `down`.
// (Two CTAs of 16 rows per SM hide the encoding latency better than one CTA of 32
// rows that reads the `down` fragments half as often.) The MMA's k slots are permuted in the same way for both operands (slots
// 2t, 2t+1, 2t+8, 2t+9 of MMA q are columns 16t + 4q .. 16t + 4q + 3), which leaves
// the sum over k unchanged. The 8 warps' partial sums are added in a fixed order in
// shared memory, so D does not depend on scheduling.
// The weight-scale tiles (128 rows x 16 groups) of the CTA's layout jobs come in by
// TMA at the start, next to the first stages, and are written out as atoms at the
// end (thread loads instead when the row-major scale rows are not 16-byte multiples).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "layout.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace ql {

namespace {

constexpr int kSvWarps = 8;
constexpr int kSvThreads = 32 * kSvWarps;
constexpr int kSvRows = 16;                                // rows per CTA
constexpr int kSvHalves = kSvRows / 16;                    // 16-row MMA groups per CTA
constexpr int kSvStages = 4;
constexpr int kSvBoxBytes = kSvRows * 128;                 // kSvRows rows x 64 bf16
constexpr int kSvStageBytes = kSvWarps * kSvBoxBytes;
constexpr int kSvWsTiles = 2;                              // weight-scale tiles in flight
constexpr int kSvWsTileBytes = 128 * 64;                   // 128 rows x 64 scale bytes

struct SvdqPrologueArgs {
  int M, K, KG;                  // KG: 64-column groups of the scale atoms (K padded)
  const float* input_scale;      // global scale g of the activations
  const float* weight_scale_2;
  const float* smooth;           // [K] or null
  const uint16_t* down;          // bf16 [rank, K]
  uint8_t* xq;                   // [M, K/2] codes
  uint8_t* xs;                   // activation scale atoms (rows padded to 128)
  uint16_t* lr_act;              // bf16 [M, rank]
  const uint8_t* w_scale;        // E4M3 [N, K/16] row-major
  int64_t N;
  int bn, na;
  int64_t w_jobs;
  bool w_tma;                    // weight-scale tiles by TMA (tmap_ws valid)
  uint8_t* wout;                 // weight scale atoms for tiles of bn rows
  int* status;
  uint64_t timeout_ns;
};

// Shared memory: stages (the partial-sum buffer after the main loop), weight-scale
// tiles, barriers and counters.
constexpr size_t kSvWsOff = static_cast<size_t>(kSvStages) * kSvStageBytes;
constexpr size_t kSvBarOff = kSvWsOff + static_cast<size_t>(kSvWsTiles) * kSvWsTileBytes;
constexpr size_t kSvSmemBytes = 1024 + kSvBarOff + (kSvStages + kSvWsTiles) * sizeof(uint64_t) +
                                kSvStages * sizeof(uint32_t) + sizeof(int);
static_assert(static_cast<size_t>(kSvWarps) * kSvRows * 65 * sizeof(float) <= kSvWsOff,
              "the partial sums of rank 64 fit in the stage buffers");
static_assert(sizeof(WsTile) <= kSvWsOff, "the thread-load weight tile fits in the stage buffers");

__device__ __forceinline__ void sv_record_timeout(int* status) {
  if (status) atomicCAS(status, 0, static_cast<int>(QL_ERR_TIMEOUT_CODE));
}

// Shared-memory counter increment that releases this thread's (and, after a
// __syncwarp, its warp's) earlier reads and acquires the other increments.
__device__ __forceinline__ uint32_t atom_add_acqrel_cta(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "r"(smem_u32(p)), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ uint4 lds16(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&c)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Issues stage load j (boxes 8j .. of the row group) into slot j % kSvStages.
__device__ __forceinline__ void sv_issue_stage(int j, int KG, int row0, uint8_t* stage_buf,
                                               uint64_t* full_bar, int* issued,
                                               const CUtensorMap* tmap_x) {
  const int s = j % kSvStages;
  const int nbox = min(kSvWarps, KG - kSvWarps * j);
  mbar_arrive_expect_tx(&full_bar[s], static_cast<uint32_t>(nbox * kSvBoxBytes));
  for (int b = 0; b < nbox; ++b)
    tma_load_2d(stage_buf + s * kSvStageBytes + b * kSvBoxBytes, tmap_x, &full_bar[s],
                (kSvWarps * j + b) * 64, row0);
  atomicMax(issued, j + 1);
}

// Weight-scale job `job` = (tile t, atom a, 16-group chunk kc) -> its 128 x 64-byte tile
// of the row-major scales (rows t * bn + 128 a .., bytes 64 kc ..) by TMA.
__device__ __forceinline__ void sv_issue_ws_tile(int64_t job, const SvdqPrologueArgs& a,
                                                 uint8_t* tile, uint64_t* bar,
                                                 const CUtensorMap* tmap_ws) {
  const int64_t kg_chunks = ceil_div64(a.KG, kWsGroups);
  const int64_t kc = job % kg_chunks;
  const int at = static_cast<int>((job / kg_chunks) % a.na);
  const int64_t t = job / (kg_chunks * a.na);
  mbar_arrive_expect_tx(bar, kSvWsTileBytes);
  tma_load_2d(tile, tmap_ws, bar, static_cast<int32_t>(kc * 64),
              static_cast<int32_t>(t * a.bn + static_cast<int64_t>(at) * 128));
}

// The atoms of one job from its tile: word w of the atom of group kg holds the 4
// scales of atom row rr = 32 (w % 4) + w / 4; rows outside the bn-row tile or N are 0.
__device__ __forceinline__ void sv_store_ws_tile(int64_t job, int tid, const SvdqPrologueArgs& a,
                                                 const uint8_t* tile) {
  const int64_t kg_chunks = ceil_div64(a.KG, kWsGroups);
  const int64_t kc = job % kg_chunks;
  const int at = static_cast<int>((job / kg_chunks) % a.na);
  const int64_t t = job / (kg_chunks * a.na);
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int idx = tid + kSvThreads * it;  // 0 .. 511: (word w, quad q of groups)
    const int w = idx % 128, q = idx / 128;
    const int rr = (w % 4) * 32 + w / 4;
    const int nn = at * 128 + rr;
    const bool valid = nn < a.bn && t * a.bn + nn < a.N;
    const uint4 v = valid ? lds16(tile + rr * 64 + 16 * q) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int64_t kg = kc * kWsGroups + 4 * q + jj;
      if (kg < a.KG)
        reinterpret_cast<uint32_t*>(
            a.wout + static_cast<size_t>(((t * a.KG) + kg) * a.na + at) * kSfAtomBytes)[w] = vw[jj];
    }
  }
}

template <int NB>
__global__ void __launch_bounds__(kSvThreads, NB <= 4 ? 2 : 1)
svdq_prologue_kernel(const __grid_constant__ CUtensorMap tmap_x,
                     const __grid_constant__ CUtensorMap tmap_ws, const SvdqPrologueArgs a) {
  constexpr int R = 8 * NB;
  constexpr int NBA = NB > 0 ? NB : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stage_buf = smem;  // kSvStages x 8 boxes, 1024-byte aligned (128-byte swizzle)
  uint8_t* ws_buf = smem + kSvWsOff;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kSvBarOff);
  uint64_t* ws_bar = full_bar + kSvStages;
  uint32_t* done = reinterpret_cast<uint32_t*>(ws_bar + kSvWsTiles);  // reads per stage slot
  int* issued = reinterpret_cast<int*>(done + kSvStages);              // stage loads issued
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row0 = blockIdx.x * kSvRows;
  const int loads = (a.KG + kSvWarps - 1) / kSvWarps;  // stage loads of this row group
  // this CTA's weight-scale jobs: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int64_t my_jobs =
      a.w_jobs > blockIdx.x ? (a.w_jobs - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  int64_t ws_issued = 0;  // thread 0 only
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_x);
    for (int s = 0; s < kSvStages; ++s) {
      mbar_init(&full_bar[s], 1);
      done[s] = 0;
    }
    for (int i = 0; i < kSvWsTiles; ++i) mbar_init(&ws_bar[i], 1);
    *issued = 0;
    fence_mbar_init();
    for (int j = 0; j < loads && j < kSvStages; ++j)
      sv_issue_stage(j, a.KG, row0, stage_buf, full_bar, issued, &tmap_x);
    if (a.w_tma) {
      for (; ws_issued < my_jobs && ws_issued < kSvWsTiles; ++ws_issued)
        sv_issue_ws_tile(blockIdx.x + ws_issued * gridDim.x, a,
                         ws_buf + ws_issued * kSvWsTileBytes, &ws_bar[ws_issued], &tmap_ws);
    }
  }
  __syncthreads();
  const uint64_t deadline = globaltimer_ns() + a.timeout_ns;

  const int g = lane / 4, t = lane % 4;
  const int sw = g & 7;  // swizzle phase of box rows g + 8i
  const float gsc = __ldg(a.input_scale);
  const float cq = __frcp_rn(__fmul_rn(6.0f, gsc));
  const int64_t half_k = a.K >> 1;
  float acc[kSvHalves][NBA][4];
#pragma unroll
  for (int h = 0; h < kSvHalves; ++h)
#pragma unroll
    for (int nb = 0; nb < NBA; ++nb) acc[h][nb][0] = acc[h][nb][1] = acc[h][nb][2] = acc[h][nb][3] = 0.0f;
  bool ok = true;
  for (int j = 0; j < loads; ++j) {
    const int kg = kSvWarps * j + warp;
    if (kg >= a.KG) break;  // warp-uniform; only in the last stage
    const int s = j % kSvStages;
    const int k = kg * 64 + 16 * t;
    const bool kin = k < a.K;  // K % 16 == 0: the thread's blocks are inside K or not at all
    // operands that do not come from the stage, in flight while the stage is awaited
    uint4 bf[NBA][2];
    if constexpr (NB > 0) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        if (kin) {
          const uint16_t* dr = a.down + static_cast<int64_t>(8 * nb + g) * a.K + k;
          bf[nb][0] = __ldg(reinterpret_cast<const uint4*>(dr));
          bf[nb][1] = __ldg(reinterpret_cast<const uint4*>(dr + 8));
        } else {
          bf[nb][0] = bf[nb][1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    float4 sm[4];
    const bool smoothing = a.smooth != nullptr && kin;
    if (smoothing) {
#pragma unroll
      for (int i = 0; i < 4; ++i) sm[i] = __ldg(reinterpret_cast<const float4*>(a.smooth + k) + i);
    }
    if (!warp_wait_bounded(&full_bar[s], (j / kSvStages) & 1, deadline)) {
      ok = false;
      break;
    }
    const uint8_t* box = stage_buf + s * kSvStageBytes + warp * kSvBoxBytes;
    uint4 xv[2 * kSvHalves][2];
#pragma unroll
    for (int i = 0; i < 2 * kSvHalves; ++i) {
      xv[i][0] = lds16(box + (g + 8 * i) * 128 + (((2 * t) ^ sw) << 4));
      xv[i][1] = lds16(box + (g + 8 * i) * 128 + (((2 * t + 1) ^ sw) << 4));
    }
    __syncwarp();
    // the last of the 8 warps to have read slot s refills it with stage load j + kSvStages
    if (lane == 0 && atom_add_acqrel_cta(&done[s], 1u) % kSvWarps == kSvWarps - 1 &&
        j + kSvStages < loads)
      sv_issue_stage(j + kSvStages, a.KG, row0, stage_buf, full_bar, issued, &tmap_x);
    if (smoothing) {
#pragma unroll
      for (int i = 0; i < 2 * kSvHalves; ++i) {
        xv[i][0] = smooth8(xv[i][0], sm[0], sm[1]);
        xv[i][1] = smooth8(xv[i][1], sm[2], sm[3]);
      }
    }
    // NVFP4 of the blocks (rows row0 + g + 8i, columns k .. k+15); outside x the values
    // are the TMA's zero fill, which gives zero scales
#pragma unroll
    for (int i = 0; i < 2 * kSvHalves; ++i) {
      const int r = row0 + g + 8 * i;
      uint32_t sc;
      const uint2 cd = nvfp4_block16(xv[i][0], xv[i][1], gsc, cq, sc);
      if (kin && r < a.M) *reinterpret_cast<uint2*>(a.xq + r * half_k + (k >> 1)) = cd;
      a.xs[sf_act_word_offset(r, kg, a.KG) + t] = static_cast<uint8_t>(sc);
    }
    if constexpr (NB > 0) {
      if (kg * 64 < a.K) {  // warp-uniform: groups of K padding add nothing
#pragma unroll
        for (int h = 0; h < kSvHalves; ++h) {
          const uint4 lo0 = xv[2 * h][0], lo1 = xv[2 * h][1];
          const uint4 hi0 = xv[2 * h + 1][0], hi1 = xv[2 * h + 1][1];
          const uint32_t wa8[8] = {lo0.x, lo0.y, lo0.z, lo0.w, lo1.x, lo1.y, lo1.z, lo1.w};
          const uint32_t wb8[8] = {hi0.x, hi0.y, hi0.z, hi0.w, hi1.x, hi1.y, hi1.z, hi1.w};
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const uint32_t wd[8] = {bf[nb][0].x, bf[nb][0].y, bf[nb][0].z, bf[nb][0].w,
                                    bf[nb][1].x, bf[nb][1].y, bf[nb][1].z, bf[nb][1].w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
              mma_m16n8k16_bf16(acc[h][nb], wa8[2 * q], wb8[2 * q], wa8[2 * q + 1],
                                wb8[2 * q + 1], wd[2 * q], wd[2 * q + 1]);
          }
        }
      }
    }
  }

  // every warp is done with the stages (they become the partial-sum buffer)
  const bool failed = barrier1_any<kSvThreads>(!ok);
  if (!ok) sv_record_timeout(a.status);
  if (failed) {
    if (threadIdx.x == 0) {
      // the CTA stays resident until the copies it issued have landed
      const uint64_t drain = globaltimer_ns() + 100000000ull;
      const int n = *issued;
      for (int j = n > kSvStages ? n - kSvStages : 0; j < n; ++j)
        mbar_wait_bounded(&full_bar[j % kSvStages], (j / kSvStages) & 1, drain);
      for (int64_t i = ws_issued > kSvWsTiles ? ws_issued - kSvWsTiles : 0; i < ws_issued; ++i)
        mbar_wait_bounded(&ws_bar[i % kSvWsTiles], (i / kSvWsTiles) & 1, drain);
    }
    return;
  }

  // ------------------------------------ fixed-order sum of the partial D, lr_act
  if constexpr (NB > 0) {
    float(*part)[kSvRows][R + 1] = reinterpret_cast<float(*)[kSvRows][R + 1]>(stage_buf);
#pragma unroll
    for (int h = 0; h < kSvHalves; ++h)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        part[warp][16 * h + g][8 * nb + 2 * t] = acc[h][nb][0];
        part[warp][16 * h + g][8 * nb + 2 * t + 1] = acc[h][nb][1];
        part[warp][16 * h + g + 8][8 * nb + 2 * t] = acc[h][nb][2];
        part[warp][16 * h + g + 8][8 * nb + 2 * t + 1] = acc[h][nb][3];
      }
    barrier1_any<kSvThreads>(false);
    const float alpha = __fmul_rn(__ldg(a.input_scale), __ldg(a.weight_scale_2));
    for (int i = threadIdx.x; i < kSvRows * R; i += kSvThreads) {
      const int rr = i / R, jj = i - (i / R) * R;
      float d = 0.0f;
#pragma unroll
      for (int w = 0; w < kSvWarps; ++w) d = __fadd_rn(d, part[w][rr][jj]);  // fixed order
      if (row0 + rr < a.M) {
        const __nv_bfloat16 hv = __float2bfloat16_rn(__fdiv_rn(d, alpha));
        a.lr_act[static_cast<int64_t>(row0 + rr) * R + jj] = *reinterpret_cast<const uint16_t*>(&hv);
      }
    }
    barrier1_any<kSvThreads>(false);  // the stage buffers may hold the weight tile next
  }

  // -------------------------------------------------- weight-scale layout jobs
  if (a.w_tma) {
    for (int64_t i = 0; i < my_jobs; ++i) {
      const int buf = static_cast<int>(i % kSvWsTiles);
      const bool landed = mbar_wait_bounded(&ws_bar[buf], (i / kSvWsTiles) & 1, deadline);
      if (barrier1_any<kSvThreads>(!landed)) {
        if (threadIdx.x == 0) {
          sv_record_timeout(a.status);
          const uint64_t drain = globaltimer_ns() + 100000000ull;
          for (int64_t m = i; m < ws_issued; ++m)
            mbar_wait_bounded(&ws_bar[m % kSvWsTiles], (m / kSvWsTiles) & 1, drain);
        }
        return;
      }
      sv_store_ws_tile(blockIdx.x + i * gridDim.x, threadIdx.x, a, ws_buf + buf * kSvWsTileBytes);
      barrier1_any<kSvThreads>(false);  // the tile is read before it is refilled
      if (threadIdx.x == 0 && ws_issued < my_jobs) {
        sv_issue_ws_tile(blockIdx.x + ws_issued * gridDim.x, a,
                         ws_buf + (ws_issued % kSvWsTiles) * kSvWsTileBytes,
                         &ws_bar[ws_issued % kSvWsTiles], &tmap_ws);
        ++ws_issued;
      }
    }
  } else {
    WsTile& tile = *reinterpret_cast<WsTile*>(stage_buf);
    for (int64_t job = blockIdx.x; job < a.w_jobs; job += gridDim.x) {
      weight_scale_atoms_load(job, threadIdx.x, a.w_scale, a.N, a.K, a.bn, a.na, a.KG, tile);
      barrier1_any<kSvThreads>(false);
      weight_scale_atoms_store(job, threadIdx.x, a.na, a.KG, a.wout, tile);
      barrier1_any<kSvThreads>(false);
    }
  }
  grid_dependents_launch();
}

template <int NB>
cudaError_t launch_svdq_typed(const CUtensorMap& tx, const CUtensorMap& tws,
                              const SvdqPrologueArgs& args, unsigned grid, cudaStream_t s) {
  // the shared-memory limit is a per-device attribute of the kernel
  static bool attr_set[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(svdq_prologue_kernel<NB>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSvSmemBytes));
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  svdq_prologue_kernel<NB><<<grid, kSvThreads, kSvSmemBytes, s>>>(tx, tws, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_svdq_prologue(const void* x, int64_t M, int64_t K, const float* smooth,
                                 const void* down, int rank, const uint8_t* w_scale, int64_t N,
                                 int bn, const float* input_scale, const float* weight_scale_2,
                                 uint8_t* workspace, void* lr_act, int* status,
                                 uint64_t timeout_ns, cudaStream_t s) {
  if (rank % 8 != 0 || rank < 0 || rank > 64) return cudaErrorInvalidValue;
  CUtensorMap tx, tws;
  if (!encode_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, static_cast<uint64_t>(K),
                 static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, 64, kSvRows,
                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return cudaErrorInvalidValue;
  // row-major weight scales by TMA: rows of K/16 bytes must be 16-byte multiples
  const int64_t nblk = K / 16;
  const bool w_tma = nblk % 16 == 0 && (reinterpret_cast<uintptr_t>(w_scale) & 15) == 0 &&
                     encode_2d(&tws, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_scale,
                               static_cast<uint64_t>(nblk), static_cast<uint64_t>(N),
                               static_cast<uint64_t>(nblk), 64, 128, CU_TENSOR_MAP_SWIZZLE_NONE,
                               CU_TENSOR_MAP_L2_PROMOTION_NONE);
  if (!w_tma) tws = tx;  // unused
  const Nvfp4Workspace L = nvfp4_workspace(M, K, N, bn);
  SvdqPrologueArgs args{};
  args.M = static_cast<int>(M);
  args.K = static_cast<int>(K);
  args.KG = static_cast<int>(sf_kgroups(K));
  args.input_scale = input_scale;
  args.weight_scale_2 = weight_scale_2;
  args.smooth = smooth;
  args.down = static_cast<const uint16_t*>(down);
  args.xq = workspace + L.codes_off;
  args.xs = workspace + L.act_sf_off;
  args.lr_act = static_cast<uint16_t*>(lr_act);
  args.w_scale = w_scale;
  args.N = N;
  args.bn = bn;
  args.na = (bn + 127) / 128;
  args.w_jobs = weight_scale_jobs(N, bn, args.KG);
  args.w_tma = w_tma;
  args.wout = workspace + L.wgt_sf_off;
  args.status = status;
  args.timeout_ns = timeout_ns;
  const unsigned grid = static_cast<unsigned>(ceil_div64(M, 128) * (128 / kSvRows));
  switch (rank / 8) {
    case 0: return launch_svdq_typed<0>(tx, tws, args, grid, s);
    case 1: return launch_svdq_typed<1>(tx, tws, args, grid, s);
    case 2: return launch_svdq_typed<2>(tx, tws, args, grid, s);
    case 3: return launch_svdq_typed<3>(tx, tws, args, grid, s);
    case 4: return launch_svdq_typed<4>(tx, tws, args, grid, s);
    case 5: return launch_svdq_typed<5>(tx, tws, args, grid, s);
    case 6: return launch_svdq_typed<6>(tx, tws, args, grid, s);
    case 7: return launch_svdq_typed<7>(tx, tws, args, grid, s);
    case 8: return launch_svdq_typed<8>(tx, tws, args, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ql
