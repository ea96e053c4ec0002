// topk_sm100.cu -- decode attention over the top_k keys of each query: the
// dynamic primitive "attend to the top-K dynamic tokens" ("SAS: Sparse
// Attention Synthesizer", Step 5, component 1, primitive C; the dynamic
// patterns of "Sparse Attention Weights Assumption": tokens with the highest
// relevance scores).  For query (s, h) over keys j < len_s of its K/V head:
// score s_j = scale * q . k_j, G = the top_k keys by score (equal scores to
// the smaller j), out = softmax over G of s_j, weighted sum of v_j.
//
// Three launches, each bound by HBM:
//   1. score: one CTA per (chunk of 8192 keys, sequence, group of query heads
//      sharing a K/V head).  Every K row is read once for all the heads of
//      its group (16-byte loads, d/8 lanes per row), each score is written to
//      the workspace (log2-scaled, fp32) and counted in a per-head histogram
//      of the top 11 bits of its order-preserving key, kept in shared memory
//      and added to global memory once per CTA.
//   2. select: one CTA per (sequence, head) -- an exact radix select: the
//      histogram gives the 11-bit bin of the top_k-th largest key; one sweep
//      over the head's scores keeps that bin's keys in shared memory (up to
//      8192; more take a slower path of three sweeps) and counts, per warp
//      segment of the row, the keys above it; the threshold's last 21 bits
//      are resolved in shared memory; a second sweep writes the selected
//      indices in ascending order, equal keys in index order.
//   3. attend: one CTA per (sequence, head) -- online softmax over the stored
//      scores of the selected keys and the weighted sum of their V rows.
#include <cuda_bf16.h>

#include <cmath>

#include "common.h"
#include "ptx.cuh"
#include "softmax_util.cuh"

namespace sa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kSelectThreads = 1024;
constexpr int kAttendThreads = 256;
constexpr int kAttendUnroll = 8;

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

// Order-preserving key of a score: unsigned comparison of keys is the
// comparison of the floats (-0 is taken as +0, so equal floats give equal keys).
__device__ __forceinline__ uint32_t topk_key(float x) {
  const uint32_t u = __float_as_uint(x == 0.f ? 0.f : x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose key is `key` (the inverse of topk_key).
__device__ __forceinline__ float topk_key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Keys of sequence s: lengths[s] clamped to [0, L] (an out-of-range length is
// recorded as SA_ERR_DEVICE_INDEX at `site`).
__device__ __forceinline__ int seq_len(const TopkParams& p, int s, int site) {
  if (!p.lengths) return p.L;
  const int n = __ldg(p.lengths + s);
  if (n < 0 || n > p.L) {
    if (threadIdx.x == 0) record_device_error(p.err, SA_ERR_DEVICE_INDEX, site);
    return n < 0 ? 0 : p.L;
  }
  return n;
}

// ---------------------------------------------------------------- score --
// CTA: 8 warps; a row of D bf16 is read by LPR = D/8 lanes (16 bytes each), so
// a warp step covers 32/LPR rows and a warp takes U steps per iteration (U
// rows' loads in flight per lane).  Each lane ends a step with partial dot
// products for its 8 dimensions, U*G of them per iteration; they are summed
// over the row's LPR lanes by a transposing reduction: at each of the
// log2(LPR) exchange steps a lane keeps half of its values, sends the other
// half to its partner and adds what it receives, so V values cost V-1
// shuffles in all instead of V*log2(LPR), and lane l of a row ends holding
// the totals l*(V/LPR) .. l*(V/LPR) + V/LPR - 1 (value index = u*G + g).
template <int D, int G>
struct ScoreCfg {
  static constexpr int LPR = D / 8;
  static constexpr int RPS = 32 / LPR;                  // rows per warp step
  static constexpr int U = (32 / G) > 16 ? 16 : 32 / G;  // steps per iteration
  static constexpr int V = U * G;                        // partial dots per lane
  static constexpr int HV = V / LPR;                     // totals per lane
  static constexpr int ROWS_WARP = RPS * U;
  static constexpr int ROWS_IT = ROWS_WARP * (kScoreThreads / 32);
  static_assert(V % LPR == 0 && V >= LPR, "reduction needs V a multiple of LPR");
};

template <int D, int G>
__global__ void __launch_bounds__(kScoreThreads, 2) topk_score_kernel(const TopkParams p) {
  using C = ScoreCfg<D, G>;
  extern __shared__ uint32_t hist[];   // [G][kTopkBins1]
  const int nqg = p.H / G;
  const int s = blockIdx.x / nqg, qg = blockIdx.x % nqg;
  const int h0 = qg * G;                      // first query head of the CTA
  const int hkv = h0 / (p.H / p.Hkv);
  const int len = seq_len(p, s, 3);
  const int row_lo = blockIdx.y * p.chunk;
  const int row_hi = min(len, row_lo + p.chunk);
  if (row_lo >= row_hi) return;

  for (int t = threadIdx.x; t < G * kTopkBins1; t += kScoreThreads) hist[t] = 0;
  __syncthreads();

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int l = lane % C::LPR, slot = lane / C::LPR;
  float q[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 qv =
        *reinterpret_cast<const uint4*>(p.Q + ((int64_t)s * p.H + h0 + g) * D + l * 8);
    bf16x8_to_f32(qv, q[g]);
#pragma unroll
    for (int c = 0; c < 8; ++c) q[g][c] *= p.scale_log2;
  }
  const uint16_t* Kb = p.K + ((int64_t)s * p.Hkv + hkv) * p.L * D + l * 8;
  float* Sb = p.scores + ((int64_t)s * p.H + h0) * p.Lp;

  for (int base = row_lo + warp * C::ROWS_WARP; base < row_hi; base += C::ROWS_IT) {
    uint4 kv[C::U];
#pragma unroll
    for (int u = 0; u < C::U; ++u) {
      const int j = base + u * C::RPS + slot;
      kv[u] = j < row_hi ? ld_stream(Kb + (int64_t)j * D) : make_uint4(0, 0, 0, 0);
    }
    float v[C::V];
#pragma unroll
    for (int u = 0; u < C::U; ++u) {
      float kf[8];
      bf16x8_to_f32(kv[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        // packed f32x2 products: even and odd dimensions, summed at the end
        uint64_t d2 = f2_mul(f2_pack(q[g][0], q[g][1]), f2_pack(kf[0], kf[1]));
#pragma unroll
        for (int c = 2; c < 8; c += 2)
          d2 = f2_fma(f2_pack(q[g][c], q[g][c + 1]), f2_pack(kf[c], kf[c + 1]), d2);
        float d0, d1;
        f2_unpack(d2, d0, d1);
        v[u * G + g] = d0 + d1;
      }
    }
    // transposing reduction over the LPR lanes of each row
#pragma unroll
    for (int o = C::LPR / 2, half = C::V / 2; o > 0; o >>= 1, half >>= 1) {
      const bool upper = (l & o) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float keep = upper ? v[half + i] : v[i];
        const float send = upper ? v[i] : v[half + i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
#pragma unroll
    for (int i = 0; i < C::HV; ++i) {
      const int vi = l * C::HV + i;
      const int u = vi / G, g = vi % G;
      const int j = base + u * C::RPS + slot;
      if (j < row_hi) {
        Sb[(int64_t)g * p.Lp + j] = v[i];
        atomicAdd(&hist[g * kTopkBins1 + (topk_key(v[i]) >> 21)], 1u);
      }
    }
  }
  __syncthreads();
  uint32_t* gh = p.hist + ((int64_t)s * p.H + h0) * kTopkBins1;
  for (int t = threadIdx.x; t < G * kTopkBins1; t += kScoreThreads) {
    const uint32_t c = hist[t];
    if (c) atomicAdd(gh + t, c);
  }
}

// --------------------------------------------------------------- select --
// Exclusive prefix sum over the block (kSelectThreads threads); *total gets
// the block's sum.  ws: shared [33].  Every thread must call it.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t* ws, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) ws[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = ws[lane];
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    ws[lane] = wi - w;
    if (lane == 31) ws[32] = wi;
  }
  __syncthreads();
  const uint32_t r = ws[warp] + inc - x;
  *total = ws[32];
  __syncthreads();
  return r;
}

// The bin that holds the r-th largest key (r >= 1) of a histogram of NB bins,
// bins taken from the top: above(b) < r <= above(b) + h[b].  Writes the bin and
// the rank left inside it (r - above(b)) to res[0..1]; res[0] stays -1 when
// the histogram holds fewer than r keys.
template <int NB>
__device__ __forceinline__ void find_bin(const uint32_t* h, uint32_t r, uint32_t* ws, int* res) {
  constexpr int PER = NB / kSelectThreads;
  if (threadIdx.x == 0) res[0] = -1;
  uint32_t c[PER], sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    c[i] = h[NB - 1 - (threadIdx.x * PER + i)];
    sum += c[i];
  }
  uint32_t total;
  uint32_t above = block_excl_scan(sum, ws, &total);   // synchronises (res[0] visible)
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    if (above < r && r <= above + c[i]) {
      res[0] = NB - 1 - (threadIdx.x * PER + i);
      res[1] = int(r - above);
    }
    above += c[i];
  }
  __syncthreads();
}

constexpr int kSelUnroll = 4;      // float4 loads in flight per thread in a sweep
constexpr int kCandCap = 8192;     // keys of the threshold's first-level bin kept in shared memory
constexpr int kSegs = kSelectThreads / 32;   // row segments: one per warp

struct SelectSmem {
  uint32_t h[kTopkBins1];
  uint32_t cand_key[kCandCap];
  int32_t cand_j[kCandCap];
  uint32_t ws[33];
  int res[2];
  uint32_t seg_sel[kSegs], seg_tie[kSegs], seg_off[kSegs], tie_before[kSegs];
  uint32_t seg_cand[kSegs];   // kept keys per segment (each in its warp's region)
  int overflow;               // a segment held more kept keys than its region
};
// kept keys of a warp's segment: region [warp * kRegion, (warp + 1) * kRegion)
constexpr int kRegion = kCandCap / kSegs;

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// One sweep over the scores of a row, j in [0, len): f(j, key) for every key,
// kSelUnroll float4 loads issued per thread before any is used.  Rows are
// padded to a multiple of 4 floats, so a float4 that starts below len is in
// bounds.
template <class F>
__device__ __forceinline__ void sweep(const float* sc, int len, F&& f) {
  constexpr int STEP = kSelectThreads * 4;
  for (int c0 = threadIdx.x * 4; c0 < len; c0 += STEP * kSelUnroll) {
    float4 v[kSelUnroll];
#pragma unroll
    for (int u = 0; u < kSelUnroll; ++u) {
      const int j0 = c0 + u * STEP;
      v[u] = j0 < len ? *reinterpret_cast<const float4*>(sc + j0) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kSelUnroll; ++u) {
      const int j0 = c0 + u * STEP;
      const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (j0 + i < len) f(j0 + i, topk_key(x[i]));
    }
  }
}

__device__ __forceinline__ void select_failed(const TopkParams& p, int sh, int site) {
  if (threadIdx.x == 0) {
    record_device_error(p.err, SA_ERR_DEVICE_INDEX, site);
    p.idx_len[sh] = 0;
  }
}

// Selection when the threshold's first-level bin holds more keys than shared
// memory keeps: two more sweeps resolve bits 20..10 and 9..0 of the
// threshold, and a last one ranks the keys chunk by chunk in index order with
// block-wide prefix sums.
__device__ __noinline__ void select_generic(const TopkParams& p, SelectSmem& sm, const float* sc,
                                            int len, int k, int b1, uint32_t r1, int32_t* out,
                                            float* sel_out, int sh) {
  uint32_t* h = sm.h;
  for (int i = threadIdx.x; i < kTopkBins1; i += kSelectThreads) h[i] = 0;
  __syncthreads();
  sweep(sc, len, [&](int, uint32_t key) {
    if ((key >> 21) == uint32_t(b1)) atomicAdd(&h[(key >> 10) & 2047u], 1u);
  });
  __syncthreads();
  find_bin<kTopkBins1>(h, r1, sm.ws, sm.res);
  const int b2 = sm.res[0];
  const uint32_t r2 = uint32_t(sm.res[1]);
  __syncthreads();
  const uint32_t pre = (uint32_t(b1) << 11) | uint32_t(b2 < 0 ? 0 : b2);
  for (int i = threadIdx.x; i < 1024; i += kSelectThreads) h[i] = 0;
  __syncthreads();
  sweep(sc, len, [&](int, uint32_t key) {
    if ((key >> 10) == pre) atomicAdd(&h[key & 1023u], 1u);
  });
  __syncthreads();
  find_bin<1024>(h, r2, sm.ws, sm.res);
  const int b3 = sm.res[0];
  const uint32_t take_eq = uint32_t(sm.res[1]);
  __syncthreads();
  if (b2 < 0 || b3 < 0) return select_failed(p, sh, 5);
  const uint32_t thr = (pre << 10) | uint32_t(b3);

  constexpr int STEP = kSelectThreads * 4;
  uint32_t n_out = 0, n_eq = 0;
  for (int c0 = 0; c0 < len; c0 += STEP) {
    const int j0 = c0 + threadIdx.x * 4;
    const float4 f = j0 < len ? *reinterpret_cast<const float4*>(sc + j0)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    const float x[4] = {f.x, f.y, f.z, f.w};
    bool gt[4], eq[4];
    uint32_t ce = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t key = topk_key(x[i]);
      const bool in = j0 + i < len;
      gt[i] = in && key > thr;
      eq[i] = in && key == thr;
      ce += eq[i];
    }
    uint32_t eq_total;
    uint32_t eq_rank = n_eq + block_excl_scan(ce, sm.ws, &eq_total);
    bool sel[4];
    uint32_t cs = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sel[i] = gt[i] || (eq[i] && eq_rank < take_eq);
      eq_rank += eq[i];
      cs += sel[i];
    }
    uint32_t sel_total;
    uint32_t pos = n_out + block_excl_scan(cs, sm.ws, &sel_total);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (sel[i] && pos < uint32_t(k)) {
        out[pos] = j0 + i;
        sel_out[pos++] = x[i];
      }
    n_out += sel_total;
    n_eq += eq_total;
  }
  if (threadIdx.x == 0) {
    if (n_out != uint32_t(k)) record_device_error(p.err, SA_ERR_DEVICE_INDEX, 6);
    p.idx_len[sh] = int(min(n_out, uint32_t(k)));
  }
}

// Common case: the row is split into 32 contiguous segments, one per warp.
// Sweep 1 counts, per segment, the keys above the threshold's first-level bin
// and keeps the bin's keys (with their indices) in shared memory; the
// threshold's last 21 bits are resolved there; a 32-entry prefix sum gives
// each segment its first output position; sweep 2 writes each segment's
// selected indices in order, ranked inside the warp by shuffles.
__global__ void __launch_bounds__(kSelectThreads, 1) topk_select_kernel(const TopkParams p) {
  extern __shared__ __align__(16) unsigned char smraw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smraw);
  const int sh = blockIdx.x;
  const int s = sh / p.H;
  const int len = seq_len(p, s, 4);
  const int k = min(p.top_k, len);
  int32_t* out = p.idx + (int64_t)sh * p.top_k;
  float* sel_out = p.sel_scores + (int64_t)sh * p.top_k;
  if (k == len) {   // every key is selected
    const float* scr = p.scores + (int64_t)sh * p.Lp;
    for (int j = threadIdx.x; j < len; j += kSelectThreads) {
      out[j] = j;
      sel_out[j] = scr[j];
    }
    if (threadIdx.x == 0) p.idx_len[sh] = len;
    return;
  }
  const float* sc = p.scores + (int64_t)sh * p.Lp;

  // level 1: top 11 bits, from the score pass's histogram
  for (int i = threadIdx.x; i < kTopkBins1; i += kSelectThreads)
    sm.h[i] = p.hist[(int64_t)sh * kTopkBins1 + i];
  __syncthreads();
  find_bin<kTopkBins1>(sm.h, uint32_t(k), sm.ws, sm.res);
  const int b1 = sm.res[0];
  const uint32_t r1 = uint32_t(sm.res[1]);
  const uint32_t c1 = b1 >= 0 ? sm.h[b1] : 0u;
  // bins 0-3 and 2044-2047 hold the infinities and NaNs
  const uint32_t n_special = sm.h[0] + sm.h[1] + sm.h[2] + sm.h[3] + sm.h[2044] + sm.h[2045] +
                             sm.h[2046] + sm.h[2047];
  __syncthreads();
  if (b1 < 0) return select_failed(p, sh, 5);   // the histogram does not hold len keys
  // The sweeps below compare the floats themselves with the bounds of bin b1
  // and with the threshold (key order is float order, NaN aside); the bounds
  // must be numbers, which holds for bins 4 .. 2043, and the row must hold no
  // infinity or NaN (bins 0-3 and 2044-2047), which the key order ranks but
  // float comparisons do not.
  if (c1 > uint32_t(kCandCap) || b1 < 4 || b1 > 2043 || n_special != 0)
    return select_generic(p, sm, sc, len, k, b1, r1, out, sel_out, sh);
  const float f_lo = topk_key_float(uint32_t(b1) << 21);        // x >= f_lo: bin >= b1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = (((len + kSegs - 1) / kSegs) + 127) & ~127;   // a multiple of 128 keys
  const int lo = warp * seg, hi = min(len, lo + seg);
  if (threadIdx.x == 0) sm.overflow = 0;
  __syncthreads();

  // The one sweep: every key at or above the threshold's bin (the keys above
  // it are all selected, the bin's are resolved below) is kept with its index
  // in the warp's own region of shared memory, in index order, placed by a
  // warp prefix sum -- no shared counter, so no contended atomics.
  uint32_t wc = 0;   // this warp's kept keys so far (warp-uniform)
  uint32_t* ck = sm.cand_key + warp * kRegion;
  int32_t* cj = sm.cand_j + warp * kRegion;
  for (int c0 = lo; c0 < hi; c0 += 128 * kSelUnroll) {
    float4 v[kSelUnroll];
#pragma unroll
    for (int u = 0; u < kSelUnroll; ++u) {
      const int j0 = c0 + u * 128 + lane * 4;
      v[u] = j0 < hi ? *reinterpret_cast<const float4*>(sc + j0) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kSelUnroll; ++u) {
      if (c0 + u * 128 >= hi) break;   // the same for the whole warp
      const int j0 = c0 + u * 128 + lane * 4;
      const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      bool keep[4] = {false, false, false, false};
      uint32_t cl = 0;
      // most scores lie below the bin: one test per float4 skips them
      if (fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3])) >= f_lo) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          keep[i] = j0 + i < hi && x[i] >= f_lo;
          cl += keep[i];
        }
      }
      if (!__any_sync(0xffffffffu, cl != 0)) continue;
      const uint32_t incl = warp_incl_scan(cl);
      uint32_t pos = wc + incl - cl;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (keep[i]) {
          if (pos < uint32_t(kRegion)) {
            ck[pos] = topk_key(x[i]);
            cj[pos] = j0 + i;
          }
          ++pos;
        }
      }
      wc += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (lane == 0) {
    sm.seg_cand[warp] = wc;
    if (wc > uint32_t(kRegion)) sm.overflow = 1;
  }
  for (int i = threadIdx.x; i < kTopkBins1; i += kSelectThreads) sm.h[i] = 0;
  __syncthreads();
  // a segment's kept keys overflowed its region: the generic path (its own sweeps)
  if (sm.overflow) return select_generic(p, sm, sc, len, k, b1, r1, out, sel_out, sh);

  // level 2 and level 3 over the bin's keys
  for (int c = threadIdx.x; c < kCandCap; c += kSelectThreads) {
    if (uint32_t(c % kRegion) >= sm.seg_cand[c / kRegion]) continue;
    const uint32_t key = sm.cand_key[c];
    if ((key >> 21) == uint32_t(b1)) atomicAdd(&sm.h[(key >> 10) & 2047u], 1u);
  }
  __syncthreads();
  find_bin<kTopkBins1>(sm.h, r1, sm.ws, sm.res);
  const int b2 = sm.res[0];
  const uint32_t r2 = uint32_t(sm.res[1]);
  __syncthreads();
  const uint32_t pre = (uint32_t(b1) << 11) | uint32_t(b2 < 0 ? 0 : b2);
  for (int i = threadIdx.x; i < 1024; i += kSelectThreads) sm.h[i] = 0;
  __syncthreads();
  for (int c = threadIdx.x; c < kCandCap; c += kSelectThreads) {
    if (uint32_t(c % kRegion) >= sm.seg_cand[c / kRegion]) continue;
    const uint32_t key = sm.cand_key[c];
    if ((key >> 10) == pre) atomicAdd(&sm.h[key & 1023u], 1u);
  }
  __syncthreads();
  find_bin<1024>(sm.h, r2, sm.ws, sm.res);
  const int b3 = sm.res[0];
  const uint32_t take_eq = uint32_t(sm.res[1]);   // keys equal to the threshold to take
  __syncthreads();
  if (b2 < 0 || b3 < 0) return select_failed(p, sh, 5);
  const uint32_t thr = (pre << 10) | uint32_t(b3);

  // per segment: its kept keys above the threshold and equal to it, and the
  // bin's keys (whose total must be the bin's count)
  {
    uint32_t gt = 0, eq = 0, in_bin = 0;
    for (uint32_t i = lane; i < wc; i += 32) {
      const uint32_t key = ck[i];
      gt += key > thr;
      eq += key == thr;
      in_bin += (key >> 21) == uint32_t(b1);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
      in_bin += __shfl_xor_sync(0xffffffffu, in_bin, o);
    }
    if (lane == 0) {
      sm.seg_sel[warp] = gt;   // above the threshold: the keys above the bin included
      sm.seg_tie[warp] = eq;
      sm.seg_cand[warp] = in_bin;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // equal keys are taken in index order: the first take_eq of them
    const uint32_t tie = sm.seg_tie[lane];
    const uint32_t tie_before = warp_incl_scan(tie) - tie;
    const uint32_t taken = take_eq > tie_before ? min(tie, take_eq - tie_before) : 0u;
    const uint32_t tot = sm.seg_sel[lane] + taken;
    const uint32_t incl = warp_incl_scan(tot);
    sm.seg_off[lane] = incl - tot;
    sm.tie_before[lane] = tie_before;
    const uint32_t nb = warp_incl_scan(sm.seg_cand[lane]);
    if (lane == 31) {
      sm.res[0] = int(incl);
      sm.res[1] = int(nb);
    }
  }
  __syncthreads();
  if (uint32_t(sm.res[1]) != c1) return select_failed(p, sh, 5);   // the bin's count

  // the output: each warp walks its kept keys in index order and writes the
  // selected ones' indices at its segment's offset
  uint32_t run = sm.seg_off[warp];
  uint32_t tie_run = sm.tie_before[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (uint32_t c = 0; c < wc; c += 32) {
    const uint32_t i = c + lane;
    const uint32_t key = i < wc ? ck[i] : 0u;
    const bool gt = i < wc && key > thr;
    const bool eq = i < wc && key == thr;
    const uint32_t eq_b = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && tie_run + __popc(eq_b & lt) < take_eq);
    const uint32_t sel_b = __ballot_sync(0xffffffffu, sel);
    const uint32_t pos = run + __popc(sel_b & lt);
    if (sel && pos < uint32_t(k)) {
      out[pos] = cj[i];
      sel_out[pos] = topk_key_float(key);   // the score itself (the key transform is a bijection)
    }
    run += __popc(sel_b);
    tie_run += __popc(eq_b);
  }
  if (threadIdx.x == 0) {
    const uint32_t total = uint32_t(sm.res[0]);
    if (total != uint32_t(k)) record_device_error(p.err, SA_ERR_DEVICE_INDEX, 6);
    p.idx_len[sh] = int(min(total, uint32_t(k)));
  }
}

// --------------------------------------------------------------- attend --
// One CTA per (sequence, head): rows of the selected set split over row
// groups of D/8 lanes; each group keeps an online softmax over the selected
// keys' scores (already log2-scaled, written contiguously by the select pass)
// and accumulates its V rows; groups merge through shared memory.
template <int D>
__global__ void __launch_bounds__(kAttendThreads) topk_attend_kernel(const TopkParams p) {
  constexpr int LPR = D / 8;
  constexpr int NG = kAttendThreads / LPR;
  __shared__ float sm_m[NG], sm_l[NG];
  __shared__ float sm_acc[NG][D];
  const int sh = blockIdx.x;
  const int s = sh / p.H, h = sh % p.H;
  const int hkv = h / (p.H / p.Hkv);
  const int grp = threadIdx.x / LPR, gl = threadIdx.x % LPR;
  const int len = p.idx_len[sh];
  const int32_t* idx = p.idx + (int64_t)sh * p.top_k;
  const float* sel = p.sel_scores + (int64_t)sh * p.top_k;   // the selected keys' scores
  const uint16_t* Vb = p.V + ((int64_t)s * p.Hkv + hkv) * p.L * D + gl * 8;

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  for (int base = grp; base < len; base += NG * kAttendUnroll) {
    uint4 vv[kAttendUnroll];
    float w[kAttendUnroll];
#pragma unroll
    for (int u = 0; u < kAttendUnroll; ++u) {
      const int r = base + u * NG;
      int j = r < len ? __ldg(idx + r) : -1;
      if (j >= p.L) j = -1;   // cannot happen: the select pass writes indices < len
      vv[u] = j >= 0 ? ld_stream(Vb + (int64_t)j * D) : make_uint4(0, 0, 0, 0);
      w[u] = j >= 0 ? __ldg(sel + r) : -INFINITY;
    }
    float mx = w[0];
#pragma unroll
    for (int u = 1; u < kAttendUnroll; ++u) mx = fmaxf(mx, w[u]);
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;
    const float alpha = ex2(m - m_new);
    l *= alpha;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] *= alpha;
    m = m_new;
#pragma unroll
    for (int u = 0; u < kAttendUnroll; ++u) {
      const float pw = ex2(w[u] - m);
      l += pw;
      float vf[8];
      bf16x8_to_f32(vv[u], vf);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = fmaf(pw, vf[c], acc[c]);
    }
  }
  if (gl == 0) {
    sm_m[grp] = m;
    sm_l[grp] = l;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) sm_acc[grp][gl * 8 + c] = acc[c];
  __syncthreads();
  if (threadIdx.x < D) {
    float M = -INFINITY;
    for (int g = 0; g < NG; ++g) M = fmaxf(M, sm_m[g]);
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int g = 0; g < NG; ++g) {
        const float wg = ex2(sm_m[g] - M);
        L = fmaf(sm_l[g], wg, L);
        o = fmaf(sm_acc[g][threadIdx.x], wg, o);
      }
    }
    const float out = L > 0.f ? o / L : 0.f;
    p.O[(int64_t)sh * D + threadIdx.x] = __bfloat16_as_ushort(__float2bfloat16_rn(out));
    if (threadIdx.x == 0 && p.lse)
      p.lse[sh] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

template <int D, int G>
int launch_score(const TopkParams& p, cudaStream_t stream) {
  const size_t smem = size_t(G) * kTopkBins1 * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_score_kernel<D, G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(topk score)");
  }
  const dim3 grid((unsigned)(p.S * (p.H / G)), (unsigned)((p.L + p.chunk - 1) / p.chunk));
  topk_score_kernel<D, G><<<grid, kScoreThreads, smem, stream>>>(p);
  return SA_OK;
}

}  // namespace

int launch_topk(const TopkParams& p, int d, cudaStream_t stream) {
  const int64_t n = (int64_t)p.S * p.H;
  if (n == 0) return SA_OK;
  if (d != 64 && d != 128) return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  const int group = p.H / p.Hkv;
  // query heads scored together: a whole K/V group when it has 1, 2, 4 or 8
  // heads, else one head per CTA (each CTA then reads its K/V head itself)
  const int G = (group == 1 || group == 2 || group == 4 || group == 8) ? group : 1;
  cudaError_t e = cudaMemsetAsync(p.hist, 0, size_t(n) * kTopkBins1 * sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_error(e, "cudaMemsetAsync(top-k histogram)");
  int rc;
#define SA_SCORE(DD)                                       \
  switch (G) {                                             \
    case 8: rc = launch_score<DD, 8>(p, stream); break;    \
    case 4: rc = launch_score<DD, 4>(p, stream); break;    \
    case 2: rc = launch_score<DD, 2>(p, stream); break;    \
    default: rc = launch_score<DD, 1>(p, stream); break;   \
  }
  if (d == 128) { SA_SCORE(128) } else { SA_SCORE(64) }
#undef SA_SCORE
  if (rc) return rc;
  const int sel_smem = int(sizeof(SelectSmem));
  e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sel_smem);
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(top-k select)");
  topk_select_kernel<<<(unsigned)n, kSelectThreads, sel_smem, stream>>>(p);
  if (d == 128) topk_attend_kernel<128><<<(unsigned)n, kAttendThreads, 0, stream>>>(p);
  else topk_attend_kernel<64><<<(unsigned)n, kAttendThreads, 0, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "top-k launch");
  return SA_OK;
}

}  // namespace sa
