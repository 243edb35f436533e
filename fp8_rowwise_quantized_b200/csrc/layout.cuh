// Scale-factor layout read by the block-scaled tensor-core MMA, and the sizes of
// the nvfp4_linear workspace. Host and device code share these definitions.
//
// The MMA (kind::mxf4nvf4, 16-element blocks) takes, per K=64 step, 4 E4M3 scales
// per row. In TMEM they sit as one 32-bit column per group of 32 rows: column c,
// lane l holds the 4 scales of row 32c + l. A tcgen05.cp of shape 32x128b moves
// one "atom" of 128 rows x 4 scales from shared memory: 512 bytes where the scale
// j of row r (r < 128) is byte 16 * (r % 32) + 4 * (r / 32) + j.
//
// Workspace atoms are ordered so that one K tile (256 elements = 4 atoms of a
// 128-row group) is contiguous:
//   activations: atom(row_group, kg)            at ((row_group * KG) + kg) * 512
//   weights:     atom(n_tile, kg, a)             at (((n_tile * KG) + kg) * NA + a) * 512
// where kg counts groups of 64 elements along K (KG = K rounded up to 256, / 64)
// and a counts the 128-row atoms of one BN-wide weight tile (NA = ceil(BN/128)).
// Padding (rows beyond M or N, blocks beyond K/16, rows BN..NA*128 of a tile) is
// written as zero scales.
#pragma once
#include <cstddef>
#include <cstdint>

namespace ql {

constexpr int kSfAtomBytes = 512;
constexpr int kKTileFp4 = 256;  // elements of K per pipeline stage (128 bytes packed)
constexpr int kKTileFp8 = 128;  // elements of K per pipeline stage (128 bytes)

__host__ __device__ constexpr int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// 64-element groups along K, padded to whole K tiles.
__host__ __device__ constexpr int64_t sf_kgroups(int64_t K) {
  return ceil_div64(K, kKTileFp4) * (kKTileFp4 / 64);
}

// Byte offset of the scale word (4 scales j = 0..3 of row r for group kg) inside an
// atom-ordered activation buffer.
__host__ __device__ inline size_t sf_act_word_offset(int64_t r, int64_t kg, int64_t KG) {
  int64_t atom = (r / 128) * KG + kg;
  int64_t rr = r % 128;
  return static_cast<size_t>(atom) * kSfAtomBytes + static_cast<size_t>((rr % 32) * 16 + (rr / 32) * 4);
}

// Same for a weight buffer laid out for tiles of `bn` rows.
__host__ __device__ inline size_t sf_wgt_word_offset(int64_t n_tile, int64_t nn, int64_t kg,
                                                     int64_t KG, int na) {
  int64_t a = nn / 128, rr = nn % 128;
  int64_t atom = (n_tile * KG + kg) * na + a;
  return static_cast<size_t>(atom) * kSfAtomBytes + static_cast<size_t>((rr % 32) * 16 + (rr / 32) * 4);
}

// nvfp4_linear workspace: [packed activation codes M x K/2][activation scale atoms]
// [synchronisation words of the single-launch path: 64 bytes]
// [weight scale atoms for the chosen tile width], each part 1024-byte aligned.
struct Nvfp4Workspace {
  size_t codes_off, act_sf_off, sync_off, wgt_sf_off, total;
};

__host__ __device__ inline Nvfp4Workspace nvfp4_workspace(int64_t M, int64_t K, int64_t N, int bn) {
  Nvfp4Workspace w{};
  const int64_t KG = sf_kgroups(K);
  const int na = static_cast<int>((bn + 127) / 128);
  size_t codes = static_cast<size_t>(M) * static_cast<size_t>(K / 2);
  size_t act_sf = static_cast<size_t>(ceil_div64(M, 128) * KG) * kSfAtomBytes;
  size_t wgt_sf = static_cast<size_t>(ceil_div64(N, bn) * KG * na) * kSfAtomBytes;
  size_t sync = 64;
  w.codes_off = 0;
  w.act_sf_off = align_up(codes, 1024);
  w.sync_off = align_up(w.act_sf_off + act_sf, 1024);
  w.wgt_sf_off = align_up(w.sync_off + sync, 1024);
  w.total = align_up(w.wgt_sf_off + wgt_sf, 1024);
  return w;
}

}  // namespace ql
