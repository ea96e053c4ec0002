// gather_sm100.cu -- attention of one query per (sequence, head) over an
// explicit, sorted index set of a KV cache (decode over a sparse G; "Sparse
// Attention Weights Assumption": out = sum_{j in G} alpha'_j v_j with the
// softmax taken over G; the KV cache of "SAS: Sparse Attention Synthesizer",
// Step 4 challenge 2), or over the index set of a causal window-plus-globals
// pattern derived from each sequence's position, in a minimum-size cache of
// window + globals slots (the cache SAS's geometric analyzer sizes).
//
// HBM-bound: every selected K and V row is read exactly once.  One CTA per
// (sequence, query head), 256 threads.  A row of d bf16 is split over d/8
// lanes (16 bytes each), so a warp reads 32*16 bytes per load instruction and
// 256/(d/8) row groups run side by side; each group keeps its own online
// softmax state (m, l, 8 accumulators per lane) over the rows r = group,
// group + groups, ... with four rows' K and V loads in flight per lane.  The
// groups are merged through shared memory at the end.
#include <cuda_bf16.h>

#include <cmath>

#include "common.h"
#include "ptx.cuh"
#include "softmax_util.cuh"

namespace sa {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kUnroll = 4;

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

// Row r's slot: the explicit set's entry, or (window decode) the global key r
// or the window key's ring slot.
template <bool WIN>
__device__ __forceinline__ int row_slot(const GatherParams& p, const int32_t* idx, int r, int ng,
                                        int wbase) {
  if (!WIN) return __ldg(idx + r);
  if (r < ng) return r;
  const int w = wbase + (r - ng);   // < 2 * window: the window holds at most W keys
  return p.n_global + (w >= p.window ? w - p.window : w);
}

// The row range of one set: explicit (idx, len) or, for window decode, rows
// 0 .. ng-1 = the global keys and ng .. len-1 = the window keys wlo .. p whose
// ring slots are stepped from wbase (no division per row).
template <bool WIN>
__device__ __forceinline__ void set_rows(const GatherParams& p, int s, int hi, const int32_t*& idx,
                                         int& len, int& ng, int& wbase) {
  idx = nullptr;
  ng = 0;
  wbase = 0;
  if (WIN) {
    const int pos = __ldg(p.positions + s);
    if (pos < 0) {
      if (threadIdx.x == 0) record_device_error(p.err, SA_ERR_DEVICE_INDEX, 2);
      len = 0;
    } else {
      ng = min(p.n_global, pos + 1);
      const int wlo = max(p.n_global, pos - p.window + 1);
      len = ng + max(0, pos - wlo + 1);
      wbase = wlo % p.window;
    }
  } else {
    idx = p.idx + ((int64_t)s * p.H_idx + hi) * p.n_idx;
    len = p.idx_len ? __ldg(p.idx_len + (int64_t)s * p.H_idx + hi) : p.n_idx;
    len = len < 0 ? 0 : (len > p.n_idx ? p.n_idx : len);
  }
}

template <int D, bool WIN>
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const GatherParams p) {
  constexpr int LPR = D / 8;                       // lanes per row
  constexpr int NG = kGatherThreads / LPR;         // row groups per CTA
  __shared__ float sm_m[NG], sm_l[NG];
  __shared__ float sm_acc[NG][D];

  const int sh = blockIdx.x;                       // s * H + h
  const int s = sh / p.H, h = sh % p.H;
  const int hkv = h / (p.H / p.Hkv);
  const int hi = (p.H_idx == p.H) ? h : hkv;
  const int grp = threadIdx.x / LPR, gl = threadIdx.x % LPR;

  const int32_t* idx;
  int len, ng, wbase;
  set_rows<WIN>(p, s, hi, idx, len, ng, wbase);
  const uint16_t* Kb = p.K + ((int64_t)s * p.Hkv + hkv) * p.L * D + gl * 8;
  const uint16_t* Vb = p.V + ((int64_t)s * p.Hkv + hkv) * p.L * D + gl * 8;

  float q[8];
  {
    const uint4 qv = *reinterpret_cast<const uint4*>(p.Q + (int64_t)sh * D + gl * 8);
    bf16x8_to_f32(qv, q);
#pragma unroll
    for (int c = 0; c < 8; ++c) q[c] *= p.scale_log2;
  }

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;

  // The trip count is the same for every thread (shuffles below use full-warp
  // masks); rows past `len` are masked.
  for (int it = 0; it * NG * kUnroll < len; ++it) {
    const int base = grp + it * NG * kUnroll;
    uint4 kv[kUnroll], vv[kUnroll];
    bool valid[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int r = base + u * NG;
      const int j = r < len ? row_slot<WIN>(p, idx, r, ng, wbase) : -1;
      valid[u] = r < len;
      if (valid[u] && (j < 0 || j >= p.L)) {
        if (gl == 0) record_device_error(p.err, SA_ERR_DEVICE_INDEX, 1);
        valid[u] = false;
      }
      if (valid[u]) {
        kv[u] = ld_stream(Kb + (int64_t)j * D);
        vv[u] = ld_stream(Vb + (int64_t)j * D);
      } else {
        kv[u] = make_uint4(0, 0, 0, 0);
        vv[u] = make_uint4(0, 0, 0, 0);
      }
    }
    float sc[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float kf[8];
      bf16x8_to_f32(kv[u], kf);
      // the products in group_rows_update's order (even and odd dimensions
      // in two chains, then their sum), as scalar instructions: the same
      // roundings as its packed f32x2 form, so shared and per-head sets give
      // the same bits; packed here measured slower
      float d0 = q[0] * kf[0], d1 = q[1] * kf[1];
#pragma unroll
      for (int c = 2; c < 8; c += 2) {
        d0 = fmaf(q[c], kf[c], d0);
        d1 = fmaf(q[c + 1], kf[c + 1], d1);
      }
      float d = d0 + d1;
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      sc[u] = valid[u] ? d : -INFINITY;
    }
    float mx = sc[0];
#pragma unroll
    for (int u = 1; u < kUnroll; ++u) mx = fmaxf(mx, sc[u]);
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;      // nothing visible yet in this group
    const float alpha = ex2(m - m_new);    // m = -inf -> 0
    l *= alpha;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] *= alpha;
    m = m_new;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const float pw = ex2(sc[u] - m);
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
        const float w = ex2(sm_m[g] - M);
        L = fmaf(sm_l[g], w, L);
        o = fmaf(sm_acc[g][threadIdx.x], w, o);
      }
    }
    const float out = L > 0.f ? o / L : 0.f;
    p.O[(int64_t)sh * D + threadIdx.x] = __bfloat16_as_ushort(__float2bfloat16_rn(out));
    if (threadIdx.x == 0 && p.lse)
      p.lse[sh] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

// One iteration of the shared-set kernels for the G query heads of a K/V
// head: the K and V rows of this lane's row group (kUnroll of them, 16 bytes
// per lane), scores against the G queries, online softmax per head, weighted
// V accumulation.  Both shared-set kernels call it, so their arithmetic (and
// therefore their results) is the same bit for bit.
template <int D, int G>
__device__ __forceinline__ void group_rows_update(const float (&q)[G][8], float (&m)[G],
                                                  float (&l)[G], float (&acc)[G][8],
                                                  const uint4 (&kv)[kUnroll],
                                                  const uint4 (&vv)[kUnroll],
                                                  const bool (&valid)[kUnroll]) {
  constexpr int LPR = D / 8;
  // Scores: each K row unpacked once, dotted with the G queries.  The
  // products and the V accumulation run in packed f32x2 arithmetic (two
  // lanes of a pair: even and odd dimensions).
  float sc[G][kUnroll];
  constexpr int NV = G * kUnroll;   // partial dots per lane: value u * G + g
  float pv[NV];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    float kf[8];
    bf16x8_to_f32(kv[u], kf);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      uint64_t d2 = f2_mul(f2_pack(q[g][0], q[g][1]), f2_pack(kf[0], kf[1]));
#pragma unroll
      for (int c = 2; c < 8; c += 2)
        d2 = f2_fma(f2_pack(q[g][c], q[g][c + 1]), f2_pack(kf[c], kf[c + 1]), d2);
      float d0, d1;
      f2_unpack(d2, d0, d1);
      pv[u * G + g] = d0 + d1;
    }
  }
  if constexpr (NV >= LPR) {
    // Transposing reduction over the row's LPR lanes: at each level a lane
    // keeps half of its values and adds its partner's copy of them, so lane l
    // ends with the totals of values l*HV .. l*HV + HV - 1 (NV - 1 shuffles
    // instead of NV * log2(LPR)); every total is the same pairwise tree as a
    // butterfly's, so the bits do not change.  Then each total is read from
    // its lane.
    constexpr int HV = NV / LPR;
#pragma unroll
    for (int o = LPR / 2, half = NV / 2; o > 0; o >>= 1, half >>= 1) {
      const bool upper = (threadIdx.x & o) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float keep = upper ? pv[half + i] : pv[i];
        const float send = upper ? pv[i] : pv[half + i];
        pv[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    const int base = (threadIdx.x & 31) & ~(LPR - 1);   // the row group's first lane
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const float d = __shfl_sync(0xffffffffu, pv[v % HV], base + v / HV);
      sc[v % G][v / G] = valid[v / G] ? d : -INFINITY;
    }
  } else {
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      float d = pv[v];
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      sc[v % G][v / G] = valid[v / G] ? d : -INFINITY;
    }
  }
  // Online softmax per head; sc becomes the weights.
  bool live[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float mx = sc[g][0];
#pragma unroll
    for (int u = 1; u < kUnroll; ++u) mx = fmaxf(mx, sc[g][u]);
    const float m_new = fmaxf(m[g], mx);
    live[g] = m_new != -INFINITY;
    if (!live[g]) continue;
    const float alpha = ex2(m[g] - m_new);
    l[g] *= alpha;
    const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      const uint64_t r = f2_mul(f2_pack(acc[g][c], acc[g][c + 1]), a2);
      f2_unpack(r, acc[g][c], acc[g][c + 1]);
    }
    m[g] = m_new;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      sc[g][u] = ex2(sc[g][u] - m[g]);
      l[g] += sc[g][u];
    }
  }
  // Values: each V row unpacked once, accumulated into the G outputs.
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    float vf[8];
    bf16x8_to_f32(vv[u], vf);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (!live[g]) continue;
      const uint64_t s2 = f2_pack(sc[g][u], sc[g][u]);
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        const uint64_t r =
            f2_fma(s2, f2_pack(vf[c], vf[c + 1]), f2_pack(acc[g][c], acc[g][c + 1]));
        f2_unpack(r, acc[g][c], acc[g][c + 1]);
      }
    }
  }
}

// Merge of the row groups' states through shared memory (sm_m, sm_l: [G][NG],
// sm_acc: [G][NG][D]) and the store of the G outputs of sequence s, query
// heads h0 .. h0 + G - 1.  Ends with the whole CTA past a barrier.
template <int D, int G>
__device__ __forceinline__ void group_merge_store(const GatherParams& p, int s, int h0,
                                                  const float (&m)[G], const float (&l)[G],
                                                  const float (&acc)[G][8], float* sm_m,
                                                  float* sm_l, float* sm_acc) {
  constexpr int LPR = D / 8;
  constexpr int NG = kGatherThreads / LPR;
  const int grp = threadIdx.x / LPR, gl = threadIdx.x % LPR;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (gl == 0) {
      sm_m[g * NG + grp] = m[g];
      sm_l[g * NG + grp] = l[g];
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) sm_acc[(g * NG + grp) * D + gl * 8 + c] = acc[g][c];
  }
  __syncthreads();

  for (int t = threadIdx.x; t < G * D; t += kGatherThreads) {
    const int g = t / D, c = t % D;
    float M = -INFINITY;
    for (int k = 0; k < NG; ++k) M = fmaxf(M, sm_m[g * NG + k]);
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int k = 0; k < NG; ++k) {
        const float w = ex2(sm_m[g * NG + k] - M);
        L = fmaf(sm_l[g * NG + k], w, L);
        o = fmaf(sm_acc[(g * NG + k) * D + c], w, o);
      }
    }
    const float out = L > 0.f ? o / L : 0.f;
    const int64_t sh = (int64_t)s * p.H + h0 + g;
    p.O[sh * D + c] = __bfloat16_as_ushort(__float2bfloat16_rn(out));
    if (c == 0 && p.lse) p.lse[sh] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

// Same computation for the G query heads of one K/V head whose explicit index
// set is shared (sets per K/V head): one CTA per (sequence, K/V head) reads
// every selected row once and scores it against the G queries.  Each head's
// arithmetic -- row groups, row order, dot products, online softmax, merge --
// is that of gather_kernel, so the results are the same bits.
template <int D, int G>
__global__ void __launch_bounds__(kGatherThreads, 2) gather_group_kernel(const GatherParams p) {
  constexpr int LPR = D / 8;
  constexpr int NG = kGatherThreads / LPR;
  __shared__ float sm_m[G * NG], sm_l[G * NG];
  __shared__ float sm_acc[G * NG * D];

  const int sk = blockIdx.x;                       // s * H_kv + hkv
  const int s = sk / p.Hkv, hkv = sk % p.Hkv;
  const int grp = threadIdx.x / LPR, gl = threadIdx.x % LPR;

  const int32_t* idx;
  int len, ng, wbase;
  set_rows<false>(p, s, hkv, idx, len, ng, wbase);
  const uint16_t* Kb = p.K + ((int64_t)s * p.Hkv + hkv) * p.L * D + gl * 8;
  const uint16_t* Vb = p.V + ((int64_t)s * p.Hkv + hkv) * p.L * D + gl * 8;

  float q[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 qv = *reinterpret_cast<const uint4*>(
        p.Q + ((int64_t)s * p.H + hkv * G + g) * D + gl * 8);
    bf16x8_to_f32(qv, q[g]);
#pragma unroll
    for (int c = 0; c < 8; ++c) q[g][c] *= p.scale_log2;
  }
  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[g][c] = 0.f;
  }

  for (int it = 0; it * NG * kUnroll < len; ++it) {
    const int base = grp + it * NG * kUnroll;
    uint4 kv[kUnroll], vv[kUnroll];
    bool valid[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int r = base + u * NG;
      const int j = r < len ? row_slot<false>(p, idx, r, ng, wbase) : -1;
      valid[u] = r < len;
      if (valid[u] && (j < 0 || j >= p.L)) {
        if (gl == 0) record_device_error(p.err, SA_ERR_DEVICE_INDEX, 1);
        valid[u] = false;
      }
      if (valid[u]) {
        kv[u] = ld_stream(Kb + (int64_t)j * D);
        vv[u] = ld_stream(Vb + (int64_t)j * D);
      } else {
        kv[u] = make_uint4(0, 0, 0, 0);
        vv[u] = make_uint4(0, 0, 0, 0);
      }
    }
    // Rows of the next iteration: fetched into L2 now (one prefetch per
    // 128-byte line), so that their loads find them there.
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int r = base + NG * kUnroll + u * NG;
      if (r < len && (gl & 7) == 0) {
        const int j = row_slot<false>(p, idx, r, ng, wbase);
        if (j >= 0 && j < p.L) {
          asm volatile("prefetch.global.L2 [%0];" ::"l"(Kb + (int64_t)j * D));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(Vb + (int64_t)j * D));
        }
      }
    }
    group_rows_update<D, G>(q, m, l, acc, kv, vv, valid);
  }
  group_merge_store<D, G>(p, s, hkv * G, m, l, acc, sm_m, sm_l, sm_acc);
}

// Window decode over the minimum-size cache: the set of sequence s is its
// n_global global keys (slots 0 .. ng-1) and its window keys, whose slots run
// contiguously around the ring of window slots.  The rows of an iteration
// (NG * kUnroll of them) are therefore at most three contiguous slot ranges,
// which one thread copies into a shared-memory stage with 1-D bulk copies
// (kWinStages stages in flight, completion on an mbarrier per stage), so the
// loads never wait for the arithmetic.  A CTA scores each row against all
// the K/V head's query heads (G), so every cached row crosses HBM once (CTAs
// holding half the heads each re-read rows that L2 could not keep: measured
// slower).  Rows, row groups and per-head arithmetic are
// those of gather_group_kernel (group_rows_update), so the output equals the
// explicit gather over the same slots bit for bit.
constexpr int kWinStages = 3;
constexpr int kWinWaitSite = 40;   // site code recorded with SA_ERR_TIMEOUT

template <int D>
struct WinCfg {
  static constexpr int LPR = D / 8;
  static constexpr int NG = kGatherThreads / LPR;
  static constexpr int ROWS = NG * kUnroll;                  // rows per iteration
  static constexpr int STAGE_BYTES = ROWS * D * 2 * 2;       // K rows, then V rows
  static constexpr int SMEM = kWinStages * STAGE_BYTES;      // also holds the merge
};

template <int D, int G>   // G: query heads per K/V head
__global__ void __launch_bounds__(kGatherThreads, 2) window_group_kernel(const GatherParams p) {
  using W = WinCfg<D>;
  constexpr int NG = W::NG;
  static_assert(G * NG * (D + 2) * 4 <= W::SMEM, "merge arrays must fit the stages");
  extern __shared__ __align__(128) uint8_t wsm[];
  __shared__ uint64_t full[kWinStages];
  __shared__ int abort_flag;

  const int sk = blockIdx.x;                       // s * H_kv + hkv
  const int s = sk / p.Hkv, hkv = sk % p.Hkv;
  const int h0 = hkv * G;                          // first query head
  const int grp = threadIdx.x / W::LPR, gl = threadIdx.x % W::LPR;
  const int32_t* idx;
  int len, ng, wbase;
  set_rows<true>(p, s, hkv, idx, len, ng, wbase);
  const uint16_t* Kc = p.K + ((int64_t)s * p.Hkv + hkv) * p.L * D;
  const uint16_t* Vc = p.V + ((int64_t)s * p.Hkv + hkv) * p.L * D;
  const int n_it = (len + W::ROWS - 1) / W::ROWS;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kWinStages; ++st) mbar_init(smem_u32(&full[st]), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // Copies the rows of iteration t into stage t % kWinStages (one thread).
  auto issue = [&](int t) {
    const int st = t % kWinStages;
    const uint32_t sK = smem_u32(wsm + st * W::STAGE_BYTES);
    const uint32_t sV = sK + W::ROWS * D * 2;
    const int r0 = t * W::ROWS, r1 = min(len, r0 + W::ROWS);
    mbar_expect_tx(smem_u32(&full[st]), uint32_t(r1 - r0) * D * 2 * 2);
    for (int r = r0; r < r1;) {
      int slot, end;
      if (r < ng) {                                  // global keys: slots 0 .. ng-1
        slot = r;
        end = min(r1, ng);
      } else {                                       // window keys: ring slots
        int w = wbase + (r - ng);
        w = w >= p.window ? w - p.window : w;
        slot = p.n_global + w;
        end = min(r1, r + (p.window - w));
      }
      const uint32_t off = uint32_t(r - r0) * D * 2, bytes = uint32_t(end - r) * D * 2;
      bulk_load(sK + off, Kc + (int64_t)slot * D, bytes, smem_u32(&full[st]));
      bulk_load(sV + off, Vc + (int64_t)slot * D, bytes, smem_u32(&full[st]));
      r = end;
    }
  };
  if (threadIdx.x == 0)
    for (int t = 0; t < kWinStages && t < n_it; ++t) issue(t);

  float q[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 qv = *reinterpret_cast<const uint4*>(p.Q + ((int64_t)s * p.H + h0 + g) * D + gl * 8);
    bf16x8_to_f32(qv, q[g]);
#pragma unroll
    for (int c = 0; c < 8; ++c) q[g][c] *= p.scale_log2;
  }
  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[g][c] = 0.f;
  }

  int done = 0;   // iterations whose stage has been consumed
  for (int it = 0; it < n_it; ++it) {
    const int st = it % kWinStages;
    const bool ok =
        wait_bounded(smem_u32(&full[st]), (it / kWinStages) & 1, &abort_flag, p.err, kWinWaitSite);
    if (__syncthreads_or(!ok)) break;
    const uint16_t* sK = reinterpret_cast<const uint16_t*>(wsm + st * W::STAGE_BYTES);
    const uint16_t* sV = sK + W::ROWS * D;
    uint4 kv[kUnroll], vv[kUnroll];
    bool valid[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int tr = grp + u * NG;                 // row within the iteration
      valid[u] = it * W::ROWS + tr < len;
      if (valid[u]) {
        kv[u] = *reinterpret_cast<const uint4*>(sK + tr * D + gl * 8);
        vv[u] = *reinterpret_cast<const uint4*>(sV + tr * D + gl * 8);
      } else {
        kv[u] = make_uint4(0, 0, 0, 0);
        vv[u] = make_uint4(0, 0, 0, 0);
      }
    }
    group_rows_update<D, G>(q, m, l, acc, kv, vv, valid);
    done = it + 1;
    __syncthreads();                               // every thread is done with this stage
    if (threadIdx.x == 0 && it + kWinStages < n_it) issue(it + kWinStages);
  }
  if (done < n_it) {
    // A stage never completed: let the copies already issued land before the
    // shared memory is reused, and output zeros.
    if (threadIdx.x == 0)
      for (int t = done; t < n_it && t < done + kWinStages; ++t)
        wait_drain(smem_u32(&full[t % kWinStages]), (t / kWinStages) & 1);
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
    }
  }
  float* sm_m = reinterpret_cast<float*>(wsm);
  float* sm_l = sm_m + G * NG;
  float* sm_acc = sm_l + G * NG;
  group_merge_store<D, G>(p, s, h0, m, l, acc, sm_m, sm_l, sm_acc);
}

}  // namespace

int launch_gather(const GatherParams& p, int d, cudaStream_t stream) {
  const int64_t n = (int64_t)p.S * p.H;
  if (n == 0) return SA_OK;
  if (n > INT32_MAX) return set_error(SA_ERR_UNSUPPORTED, "S*H = %lld too large", (long long)n);
  const int G = p.H / p.Hkv;
  // Sets shared by a K/V head's query heads: one CTA per (sequence, K/V head).
  const bool win = p.positions != nullptr;
  const bool shared = win || p.H_idx == p.Hkv;
  const unsigned nk = (unsigned)((int64_t)p.S * p.Hkv);
  if (d != 64 && d != 128) return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  if (win && G != 4 && G != 2) {
    // other group sizes: one CTA per query head, rows read from the cache directly
    if (d == 128) gather_kernel<128, true><<<(unsigned)n, kGatherThreads, 0, stream>>>(p);
    else gather_kernel<64, true><<<(unsigned)n, kGatherThreads, 0, stream>>>(p);
  } else if (win) {
    if (nk == 0) return SA_OK;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
    static bool attr_set[2][2][64] = {};
#define SA_WIN(DD, GG)                                                                        \
  {                                                                                           \
    bool& done = attr_set[DD == 128][GG == 4][dev & 63];                                      \
    if (!done) {                                                                              \
      e = cudaFuncSetAttribute(window_group_kernel<DD, GG>,                                   \
                               cudaFuncAttributeMaxDynamicSharedMemorySize, WinCfg<DD>::SMEM); \
      if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute");                     \
      done = true;                                                                            \
    }                                                                                         \
    window_group_kernel<DD, GG><<<nk, kGatherThreads, WinCfg<DD>::SMEM, stream>>>(p);         \
  }
    if (d == 128 && G == 4) SA_WIN(128, 4)
    else if (d == 128 && G == 2) SA_WIN(128, 2)
    else if (d == 64 && G == 4) SA_WIN(64, 4)
    else SA_WIN(64, 2)
#undef SA_WIN
  } else if (shared && G == 4 && d == 128) {
    gather_group_kernel<128, 4><<<nk, kGatherThreads, 0, stream>>>(p);
  } else if (shared && G == 2 && d == 128) {
    gather_group_kernel<128, 2><<<nk, kGatherThreads, 0, stream>>>(p);
  } else if (shared && G == 4 && d == 64) {
    gather_group_kernel<64, 4><<<nk, kGatherThreads, 0, stream>>>(p);
  } else if (shared && G == 2 && d == 64) {
    gather_group_kernel<64, 2><<<nk, kGatherThreads, 0, stream>>>(p);
  } else if (d == 128) {
    gather_kernel<128, false><<<(unsigned)n, kGatherThreads, 0, stream>>>(p);
  } else {
    gather_kernel<64, false><<<(unsigned)n, kGatherThreads, 0, stream>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "gather launch");
  return SA_OK;
}

}  // namespace sa
