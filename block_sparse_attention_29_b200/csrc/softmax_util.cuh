// softmax_util.cuh -- device helpers shared by the prefill kernels: warp
// maxima, the visibility predicate of a row inside a 64-key block, masking,
// row maxima as trees of 3-input maxima, and packed f32x2 arithmetic.
#pragma once
#include <cstdint>
#include <cmath>

#include "common.h"

namespace sa {

// Maximum over the 32 lanes of a warp (one redux instruction on sm_100a).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Bits [lo, hi) of a 64-bit mask, with lo and hi clamped to [0, 64].
__device__ __forceinline__ uint64_t range_bits(int lo, int hi) {
  lo = max(lo, 0);
  hi = min(hi, 64);
  if (hi <= lo) return 0ull;
  const uint64_t upto_hi = hi >= 64 ? ~0ull : ((1ull << hi) - 1ull);
  return upto_hi & ~((1ull << lo) - 1ull);
}

// A row's random key blocks, read once per work unit (the row's random-block
// row does not change inside a unit): up to kRowRandom held in registers,
// longer lists read from global memory.
constexpr int kRowRandom = 3;
struct RowRandom {
  int n;
  int v[kRowRandom];
  const int32_t* row;
};

__device__ __forceinline__ RowRandom load_row_random(const PrefillParams& p, int h, int i) {
  RowRandom rr;
  rr.n = 0;
  rr.row = nullptr;
  if (p.n_random > 0 && i < p.N) {
    const int nrb = (p.N + p.random_block - 1) / p.random_block;
    rr.row = p.rtab + ((int64_t)h * nrb + i / p.random_block) * p.n_random;
    rr.n = p.n_random;
#pragma unroll
    for (int r = 0; r < kRowRandom; ++r) rr.v[r] = r < rr.n ? __ldg(rr.row + r) : -1;
  }
  return rr;
}

// Visible keys of row i inside block kb, as a 64-bit mask (bit c = key
// kb*64 + c).  Every primitive is one index range per row (random blocks cover
// whole 64-key blocks), so the union is built from ranges; the causal cap and
// the sequence end are applied last.  Same predicate as the pattern compiler.
// The per-row part (the global, window and block-local ranges, the cap, the
// row's random blocks as the first 64-key block of their range) is computed
// once per work unit by row_vis, so a block's mask reads no pattern field and
// costs a few compares and range masks, no division.
struct RowVis {
  int all;              // the row sees every key below cap_hi (global row, or no primitive)
  int glob_hi;          // global keys [0, glob_hi) (0 when there are none)
  int win_lo, win_hi;   // window keys [win_lo, win_hi) (empty when there is no window)
  int bl_lo, bl_hi;     // block-local keys [bl_lo, bl_hi) (empty when off)
  int cap_hi;           // causal cap and sequence end: keys < cap_hi (0 for rows past N)
  int rb64;             // 64-key blocks per random block (0 when there are none)
  int rlo[kRowRandom];  // the row's first random blocks, as their first 64-key block
};

__device__ __forceinline__ RowVis row_vis(const PrefillParams& p, const RowRandom& rr, int i) {
  RowVis v;
  const bool any_prim = p.window > 0 || p.n_global > 0 || p.block_local > 0 || p.n_random > 0;
  v.all = (!any_prim || i < p.n_global) ? 1 : 0;
  v.glob_hi = p.n_global;
  if (p.window > 0) {
    v.win_lo = p.causal ? i - p.window + 1 : i - p.window / 2;
    v.win_hi = v.win_lo + (p.causal ? p.window : 2 * (p.window / 2) + 1);
  } else {
    v.win_lo = v.win_hi = 0;
  }
  if (p.block_local > 0) {
    v.bl_lo = (i / p.block_local) * p.block_local;
    v.bl_hi = v.bl_lo + p.block_local;
  } else {
    v.bl_lo = v.bl_hi = 0;
  }
  v.cap_hi = i >= p.N ? 0 : (p.causal ? i + 1 : p.N);
  v.rb64 = p.n_random > 0 ? p.random_block / kTileK : 0;
#pragma unroll
  for (int r = 0; r < kRowRandom; ++r) v.rlo[r] = r < rr.n ? rr.v[r] * v.rb64 : -(1 << 30);
  return v;
}

// Visible keys of row i inside block kb from the row's precomputed ranges:
// random blocks first (a listed random block is visible in full), then the
// union of the global, window and block-local ranges, capped.
__device__ __forceinline__ uint64_t vis_bits(const PrefillParams& p, const RowVis& v, int h,
                                             int i, int kb) {
  const int j0 = kb * kTileK;
  const uint64_t cap = range_bits(0, v.cap_hi - j0);
  if (v.all) return cap;
  const unsigned rb64 = static_cast<unsigned>(v.rb64);
  bool rnd = false;
#pragma unroll
  for (int r = 0; r < kRowRandom; ++r) rnd |= static_cast<unsigned>(kb - v.rlo[r]) < rb64;
  if (p.n_random > kRowRandom && i < p.N) {   // longer lists: read from the table
    const int nrb = (p.N + p.random_block - 1) / p.random_block;
    const int32_t* row = p.rtab + ((int64_t)h * nrb + i / p.random_block) * p.n_random;
    for (int r = kRowRandom; r < p.n_random; ++r)
      rnd |= static_cast<unsigned>(kb - __ldg(row + r) * static_cast<int>(rb64)) < rb64;
  }
  if (rnd) return cap;
  const uint64_t m = range_bits(0, v.glob_hi - j0) | range_bits(v.win_lo - j0, v.win_hi - j0) |
                     range_bits(v.bl_lo - j0, v.bl_hi - j0);
  return m & cap;
}

// x[OFF + c] = -inf where bit c of the visibility mask is clear.
template <int OFF, int NX>
__device__ __forceinline__ void apply_mask_at(uint64_t m, float (&x)[NX]) {
  static_assert(OFF + 64 <= NX, "mask range outside the array");
  const uint32_t lo = static_cast<uint32_t>(m), hi = static_cast<uint32_t>(m >> 32);
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    if (!((lo >> c) & 1u)) x[OFF + c] = -INFINITY;
    if (!((hi >> c) & 1u)) x[OFF + 32 + c] = -INFINITY;
  }
}
__device__ __forceinline__ void apply_mask(uint64_t m, float (&x)[64]) { apply_mask_at<0>(m, x); }

// ---- softmax arithmetic on 64 logits per thread ----
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of x[OFF .. OFF+64) as a tree of 3-input maxima (depth 4 instead
// of a 63-long chain).
template <int OFF, int NX>
__device__ __forceinline__ float row_max64_at(const float (&x)[NX]) {
  static_assert(OFF + 64 <= NX, "max range outside the array");
  float a[22];
#pragma unroll
  for (int k = 0; k < 21; ++k) a[k] = max3(x[OFF + 3 * k], x[OFF + 3 * k + 1], x[OFF + 3 * k + 2]);
  a[21] = x[OFF + 63];
  float b[8];
#pragma unroll
  for (int k = 0; k < 7; ++k) b[k] = max3(a[3 * k], a[3 * k + 1], a[3 * k + 2]);
  b[7] = a[21];
  return max3(max3(b[0], b[1], b[2]), max3(b[3], b[4], b[5]), fmaxf(b[6], b[7]));
}
__device__ __forceinline__ float row_max64(const float (&x)[64]) { return row_max64_at<0>(x); }

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

}  // namespace sa
