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
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

#include "internal.h"
#include "layout.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace ql {

namespace {

constexpr int kQuantThreads = 256;

// 16-byte read-only load of 8 bf16 values.
__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// NVFP4 quantization of (row r, 1024-element segment of K) work items. A warp
// handles one item in two 512-element slices: in each slice lane l owns the
// 16-element block l (two 16-byte loads; the warp's loads cover 1 KB
// contiguously), so each block's scale arithmetic runs once. Each lane writes its
// 16 codes as one 8-byte word (256 contiguous bytes per warp and slice); lanes 0,
// 4, ..., 28 gather the scales of four consecutive blocks (one 64-element group)
// and write them as one 32-bit word.
//   x  bf16 [M, K]; xq uint8 [M, K/2]
//   SF_MMA == false: xs uint8 [M, K/16] row-major (only blocks inside K)
//   SF_MMA == true:  xs in the atom layout over rows padded to 128 and KG groups
//                    of 64 (padding written as zero scales)
struct QuantItem {
  uint4 raw[4];
};

__device__ __forceinline__ void nvfp4_load_item(int r, int seg, int lane,
                                                const uint16_t* __restrict__ x, int M, int K,
                                                QuantItem& q) {
  const uint16_t* xr = x + static_cast<int64_t>(r) * K;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int e = seg * 1024 + i * 512 + lane * 16;
    const bool valid = (r < M) && (e < K);  // K % 16 == 0: a block is inside or out as a whole
    q.raw[2 * i] = valid ? ldg16(xr + e) : make_uint4(0u, 0u, 0u, 0u);
    q.raw[2 * i + 1] = valid ? ldg16(xr + e + 8) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <bool SF_MMA>
__device__ __forceinline__ void nvfp4_encode_item(int r, int seg, int lane, const QuantItem& qin,
                                                  int M, int K, const float* inv_of, float c,
                                                  uint8_t* __restrict__ xq,
                                                  uint8_t* __restrict__ xs, int KG) {
  const int nblk = K >> 4;
  uint8_t* qr = xq + static_cast<int64_t>(r) * (K >> 1);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int e = seg * 1024 + i * 512 + lane * 16;
    const bool valid = (r < M) && (e < K);
    const uint4 u = qin.raw[2 * i], v = qin.raw[2 * i + 1];
    uint32_t s;
    const uint2 codes = nvfp4_block16_tab(u, v, c, inv_of, s);
    if (valid) *reinterpret_cast<uint2*>(qr + (e >> 1)) = codes;
    // gather the scales of blocks lane .. lane+3 into lanes 0, 4, ..., 28
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, s, 1);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, s, 2);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, s, 3);
    if ((lane & 3) == 0) {
      const uint32_t word = s | (s1 << 8) | (s2 << 16) | (s3 << 24);
      const int kg = seg * 16 + i * 8 + (lane >> 2);
      if (SF_MMA) {
        if (kg < KG) {
          const int rr = r & 127;
          const int off = ((r >> 7) * KG + kg) * kSfAtomBytes + (rr & 31) * 16 + (rr >> 5) * 4;
          *reinterpret_cast<uint32_t*>(xs + off) = word;
        }
      } else if (r < M && 4 * kg < nblk) {
        uint8_t* sr = xs + static_cast<int64_t>(r) * nblk + kg * 4;
        if (4 * kg + 4 <= nblk && (reinterpret_cast<uintptr_t>(sr) & 3) == 0) {
          *reinterpret_cast<uint32_t*>(sr) = word;
        } else {
#pragma unroll
          for (int b = 0; b < 4; ++b)
            if (4 * kg + b < nblk) sr[b] = static_cast<uint8_t>(word >> (8 * b));
        }
      }
    }
  }
}

// Grid-stride loop of warps over the work items, with the next item's loads in
// flight while the current one is encoded (the grid is one wave of resident
// blocks, so there is no tail wave).
template <bool SF_MMA>
__device__ __forceinline__ void nvfp4_quantize_items(uint32_t warp_id, uint32_t nwarps, int lane,
                                                     const uint16_t* __restrict__ x, int M, int K,
                                                     const float* inv_of, float c,
                                                     uint8_t* __restrict__ xq,
                                                     uint8_t* __restrict__ xs, uint32_t total,
                                                     uint32_t segs, int KG) {
  if (warp_id >= total) return;  // warp-uniform
  // item = r * segs + seg, advanced by nwarps per iteration without dividing
  const uint32_t dr = nwarps / segs, ds = nwarps - (nwarps / segs) * segs;
  uint32_t r = warp_id / segs, seg = warp_id - (warp_id / segs) * segs;
  QuantItem cur;
  nvfp4_load_item(static_cast<int>(r), static_cast<int>(seg), lane, x, M, K, cur);
  for (uint32_t item = warp_id; item < total; item += nwarps) {
    uint32_t rn = r + dr, sn = seg + ds;
    if (sn >= segs) {
      sn -= segs;
      ++rn;
    }
    QuantItem nxt;
    if (item + nwarps < total)
      nvfp4_load_item(static_cast<int>(rn), static_cast<int>(sn), lane, x, M, K, nxt);
    nvfp4_encode_item<SF_MMA>(static_cast<int>(r), static_cast<int>(seg), lane, cur, M, K,
                              inv_of, c, xq, xs, KG);
    cur = nxt;
    r = rn;
    seg = sn;
  }
}

template <bool SF_MMA>
__global__ void __launch_bounds__(kQuantThreads)
nvfp4_quantize_kernel(const uint16_t* __restrict__ x, int M, int K,
                      const float* __restrict__ g_ptr, uint8_t* __restrict__ xq,
                      uint8_t* __restrict__ xs, uint32_t rows_total, uint32_t segs, int KG) {
  __shared__ float inv_of[128];
  const float g = __ldg(g_ptr);
  const float c = __frcp_rn(__fmul_rn(6.0f, g));
  fill_block_reciprocals(inv_of, g, threadIdx.x);
  __syncthreads();
  constexpr uint32_t kWarps = kQuantThreads / 32;
  nvfp4_quantize_items<SF_MMA>(blockIdx.x * kWarps + threadIdx.x / 32, gridDim.x * kWarps,
                               threadIdx.x % 32, x, M, K, inv_of, c, xq, xs, rows_total * segs,
                               segs, KG);
}

// The prologue of nvfp4_linear in one launch, one wave of resident blocks: each
// block's warps first quantize activation items (codes row-major, scales in atom
// layout) in a grid-stride loop, then the block takes weight-scale layout jobs.
// Each block allows the dependent GEMM launch once its own work is issued, so the
// GEMM's set-up overlaps the prologue's tail (the GEMM reads the workspace only
// after this grid has completed); triggering earlier would let resident GEMM CTAs
// take the shared memory the prologue blocks need. EARLY: allow it at the start
// instead (the small activation-only prologue of the skinny GEMMs, which stream
// their weights while it runs; that instantiation asks for the largest shared-memory
// split, so a GEMM CTA can join its blocks on an SM).
template <bool EARLY>
__global__ void __launch_bounds__(kQuantThreads)
nvfp4_prologue_kernel(const uint16_t* __restrict__ x, int M, int K,
                      const float* __restrict__ g_ptr, uint8_t* __restrict__ xq,
                      uint8_t* __restrict__ xs, uint32_t rows_total, uint32_t segs, int KG,
                      const uint8_t* __restrict__ ws, int64_t N, int bn, int na, int64_t n_tiles,
                      int64_t w_jobs, uint8_t* __restrict__ wout) {
  if constexpr (EARLY) grid_dependents_launch();
  // launched as a programmatic dependent of the kernel before it (a skinny GEMM of the
  // previous layer lets it be scheduled at that GEMM's start): nothing is read or
  // written before that kernel has completed and its writes are visible
  grid_dependency_wait();
  __shared__ WsTile tile;
  // the block's first weight-scale job: its loads are in flight during the activation
  // items, so their latency is off the block's critical path
  uint32_t first[8];
  const bool has_job = blockIdx.x < w_jobs;
  if (has_job) weight_scale_words(blockIdx.x, threadIdx.x, ws, N, K, bn, na, KG, first);
  __shared__ float inv_of[128];
  const float g = __ldg(g_ptr);
  const float c = __frcp_rn(__fmul_rn(6.0f, g));
  fill_block_reciprocals(inv_of, g, threadIdx.x);
  __syncthreads();
  constexpr uint32_t kWarps = kQuantThreads / 32;
  nvfp4_quantize_items<true>(blockIdx.x * kWarps + threadIdx.x / 32, gridDim.x * kWarps,
                             threadIdx.x % 32, x, M, K, inv_of, c, xq, xs, rows_total * segs, segs,
                             KG);
  if (has_job) {
    weight_scale_words_to_tile(threadIdx.x, first, tile);
    __syncthreads();
    weight_scale_atoms_store(blockIdx.x, threadIdx.x, na, KG, wout, tile);
    __syncthreads();
  }
  for (int64_t job = blockIdx.x + gridDim.x; job < w_jobs; job += gridDim.x) {
    weight_scale_atoms_load(job, threadIdx.x, ws, N, K, bn, na, KG, tile);
    __syncthreads();
    weight_scale_atoms_store(job, threadIdx.x, na, KG, wout, tile);
    __syncthreads();  // the tile buffer is reused by the next job
  }
  grid_dependents_launch();
}

// FP8 row-wise: one warp per row.
//   scale = amax / 448 (fp32 division); scale == 0 -> zero codes;
//   else codes = E4M3(x * (1/scale)).  Requires K % 8 == 0.
// CACHED: the row is held in registers (K <= 32 * 8 * kFp8Chunks) and read once;
// otherwise a second pass re-reads it (from L1/L2) to encode.
constexpr int kFp8Chunks = 16;

__device__ __forceinline__ uint2 fp8r_encode8(const uint4 u, float inv) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  const uint32_t lo = cvt_e4m3x4(__fmul_rn(bf16_lo(w[0]), inv), __fmul_rn(bf16_hi(w[0]), inv),
                                 __fmul_rn(bf16_lo(w[1]), inv), __fmul_rn(bf16_hi(w[1]), inv));
  const uint32_t hi = cvt_e4m3x4(__fmul_rn(bf16_lo(w[2]), inv), __fmul_rn(bf16_hi(w[2]), inv),
                                 __fmul_rn(bf16_lo(w[3]), inv), __fmul_rn(bf16_hi(w[3]), inv));
  return make_uint2(lo, hi);
}

__device__ __forceinline__ float amax8(const uint4 u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  return m;
}

template <bool CACHED>
__global__ void __launch_bounds__(kQuantThreads)
fp8r_quantize_rows_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                          uint8_t* __restrict__ xq, float* __restrict__ x_scale) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= M) return;
  const uint16_t* xr = x + row * K;
  uint8_t* qr = xq + row * K;
  const int64_t chunks = K / 8;
  float amax = 0.0f;
  uint4 cache[CACHED ? kFp8Chunks : 1];
  if constexpr (CACHED) {
#pragma unroll
    for (int i = 0; i < kFp8Chunks; ++i) {
      const int64_t ch = lane + 32 * i;
      cache[i] = ch < chunks ? ldg16(xr + ch * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kFp8Chunks; ++i) amax = fmaxf(amax, amax8(cache[i]));
  } else {
    for (int64_t ch = lane; ch < chunks; ch += 32) amax = fmaxf(amax, amax8(ldg16(xr + ch * 8)));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = __fdiv_rn(amax, 448.0f);
  if (lane == 0) x_scale[row] = scale;
  const float inv = scale == 0.0f ? 0.0f : __frcp_rn(scale);
  if constexpr (CACHED) {
#pragma unroll
    for (int i = 0; i < kFp8Chunks; ++i) {
      const int64_t ch = lane + 32 * i;
      if (ch < chunks)
        *reinterpret_cast<uint2*>(qr + ch * 8) =
            scale == 0.0f ? make_uint2(0u, 0u) : fp8r_encode8(cache[i], inv);
    }
  } else {
    for (int64_t ch = lane; ch < chunks; ch += 32)
      *reinterpret_cast<uint2*>(qr + ch * 8) =
          scale == 0.0f ? make_uint2(0u, 0u) : fp8r_encode8(ldg16(xr + ch * 8), inv);
  }
  grid_dependents_launch();  // the dependent GEMM may start its set-up
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

// Blocks of `kernel` that fit on the current device at once (one full wave).
template <typename Kernel>
int64_t resident_blocks(Kernel kernel) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQuantThreads, 0) !=
          cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  return static_cast<int64_t>(sms) * per_sm;
}

cudaError_t launch_nvfp4_quantize_rowmajor(const void* x, int64_t M, int64_t K, const float* g,
                                           uint8_t* xq, uint8_t* xs, cudaStream_t s) {
  const int64_t segs = ceil_div64(K, 1024);
  const int64_t items = M * segs;
  static std::atomic<int64_t> wave_cache{0};  // resident blocks of one wave (same on every B200)
  int64_t wave = wave_cache.load(std::memory_order_relaxed);
  if (wave == 0) {
    wave = resident_blocks(nvfp4_quantize_kernel<false>);
    wave_cache.store(wave, std::memory_order_relaxed);
  }
  const int64_t need = ceil_div64(items, kQuantThreads / 32);
  const int64_t blocks = need < wave ? need : wave;
  nvfp4_quantize_kernel<false><<<static_cast<unsigned>(blocks), kQuantThreads, 0, s>>>(
      static_cast<const uint16_t*>(x), static_cast<int>(M), static_cast<int>(K), g, xq, xs,
      static_cast<uint32_t>(M), static_cast<uint32_t>(segs), static_cast<int>(ceil_div64(K, 64)));
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_prologue(const void* x, int64_t M, int64_t K, const uint8_t* w_scale,
                                  int64_t N, int bn, const float* input_scale, uint8_t* workspace,
                                  cudaStream_t s, bool weight_layout, bool early) {
  const bool early_kernel = !weight_layout && early;
  const Nvfp4Workspace L = nvfp4_workspace(M, K, N, bn);
  const int64_t KG = sf_kgroups(K);
  const int64_t rows = ceil_div64(M, 128) * 128;
  const int64_t segs = ceil_div64(KG * 64, 1024);
  const int na = (bn + 127) / 128;
  const int64_t n_tiles = ceil_div64(N, bn);
  const int64_t w_jobs = weight_layout ? n_tiles * na * ceil_div64(KG, kWsGroups) : 0;
  static std::atomic<int64_t> wave_cache{0};  // resident blocks of one wave (same on every B200)
  static std::atomic<int> carveout_set[64] = {};
  int64_t wave = wave_cache.load(std::memory_order_relaxed);
  if (wave == 0) {
    wave = resident_blocks(nvfp4_prologue_kernel<false>);
    wave_cache.store(wave, std::memory_order_relaxed);
  }
  if (early_kernel) {
    // An SM's split between L1 and shared memory follows the kernel whose blocks it
    // runs: with the split chosen for this kernel's 9 KB, a GEMM CTA (about 200 KB)
    // launched early could not join the prologue's blocks on an SM until they left.
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && carveout_set[dev].load(std::memory_order_relaxed) == 0) {
      cudaError_t ce = cudaFuncSetAttribute(nvfp4_prologue_kernel<true>,
                                            cudaFuncAttributePreferredSharedMemoryCarveout,
                                            static_cast<int>(cudaSharedmemCarveoutMaxShared));
      if (ce != cudaSuccess) return ce;
      carveout_set[dev].store(1, std::memory_order_relaxed);
    }
  }
  int64_t need = ceil_div64(rows * segs, kQuantThreads / 32);
  if (need < w_jobs) need = w_jobs;
  const int64_t blocks = need < wave ? need : wave;
  auto kern = early_kernel ? nvfp4_prologue_kernel<true> : nvfp4_prologue_kernel<false>;
  // a programmatic dependent of the kernel before it: its blocks may be resident and
  // waiting while that kernel finishes (the kernel waits before any memory access)
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kQuantThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const uint16_t*>(x), static_cast<int>(M),
                            static_cast<int>(K), input_scale, workspace + L.codes_off,
                            workspace + L.act_sf_off, static_cast<uint32_t>(rows),
                            static_cast<uint32_t>(segs), static_cast<int>(KG), w_scale, N, bn, na,
                            n_tiles, w_jobs, workspace + L.wgt_sf_off);
}

cudaError_t launch_nvfp4_weight_atoms(const uint8_t* w_scale, int64_t K, int64_t N, int bn,
                                      uint8_t* atoms, cudaStream_t s) {
  // the prologue kernel with no activation rows writes only the weight-scale atoms;
  // its scalar input is then unused (read, not applied): the atoms buffer stands in
  const int64_t KG = sf_kgroups(K);
  const int na = (bn + 127) / 128;
  const int64_t n_tiles = ceil_div64(N, bn);
  const int64_t w_jobs = n_tiles * na * ceil_div64(KG, kWsGroups);
  static std::atomic<int64_t> wave_cache{0};  // resident blocks of one wave (same on every B200)
  int64_t wave = wave_cache.load(std::memory_order_relaxed);
  if (wave == 0) {
    wave = resident_blocks(nvfp4_prologue_kernel<false>);
    wave_cache.store(wave, std::memory_order_relaxed);
  }
  const int64_t blocks = w_jobs < wave ? w_jobs : wave;
  nvfp4_prologue_kernel<false><<<static_cast<unsigned>(blocks), kQuantThreads, 0, s>>>(
      nullptr, 0, static_cast<int>(K), reinterpret_cast<const float*>(atoms), atoms, atoms, 0u,
      static_cast<uint32_t>(ceil_div64(KG * 64, 1024)), static_cast<int>(KG), w_scale, N, bn, na,
      n_tiles, w_jobs, atoms);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_weight_layout(const uint8_t* w_scale, int64_t M, int64_t K, int64_t N,
                                       int bn, const float* input_scale, uint8_t* workspace,
                                       cudaStream_t s) {
  // the prologue kernel with no activation rows: only its weight-scale jobs run
  const Nvfp4Workspace L = nvfp4_workspace(M, K, N, bn);
  const int64_t KG = sf_kgroups(K);
  const int na = (bn + 127) / 128;
  const int64_t n_tiles = ceil_div64(N, bn);
  const int64_t w_jobs = n_tiles * na * ceil_div64(KG, kWsGroups);
  static std::atomic<int64_t> wave_cache{0};  // resident blocks of one wave (same on every B200)
  int64_t wave = wave_cache.load(std::memory_order_relaxed);
  if (wave == 0) {
    wave = resident_blocks(nvfp4_prologue_kernel<false>);
    wave_cache.store(wave, std::memory_order_relaxed);
  }
  const int64_t blocks = w_jobs < wave ? w_jobs : wave;
  nvfp4_prologue_kernel<false><<<static_cast<unsigned>(blocks), kQuantThreads, 0, s>>>(
      nullptr, static_cast<int>(M), static_cast<int>(K), input_scale, workspace + L.codes_off,
      workspace + L.act_sf_off, 0u, static_cast<uint32_t>(ceil_div64(KG * 64, 1024)),
      static_cast<int>(KG), w_scale, N, bn, na, n_tiles, w_jobs, workspace + L.wgt_sf_off);
  return cudaGetLastError();
}

cudaError_t launch_fp8r_quantize_rows(const void* x, int64_t M, int64_t K, uint8_t* xq,
                                      float* x_scale, cudaStream_t s) {
  const int rows_per_block = kQuantThreads / 32;
  if (K <= 32 * 8 * kFp8Chunks) {
    fp8r_quantize_rows_kernel<true><<<grid_for(M, rows_per_block), kQuantThreads, 0, s>>>(
        static_cast<const uint16_t*>(x), M, K, xq, x_scale);
  } else {
    fp8r_quantize_rows_kernel<false><<<grid_for(M, rows_per_block), kQuantThreads, 0, s>>>(
        static_cast<const uint16_t*>(x), M, K, xq, x_scale);
  }
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
