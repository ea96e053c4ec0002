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
      float d = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) d = fmaf(q[c], kf[c], d);
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

// Same computation for the G query heads of one K/V head whose index set is
// shared (window decode, or explicit sets per K/V head): one CTA per
// (sequence, K/V head) reads every selected row once and scores it against
// the G queries.  Each head's arithmetic -- row groups, row order, dot
// products, online softmax, merge -- is that of gather_kernel, so the results
// are the same bits.
template <int D, int G, bool WIN>
__global__ void __launch_bounds__(kGatherThreads, 2) gather_group_kernel(const GatherParams p) {
  constexpr int LPR = D / 8;
  constexpr int NG = kGatherThreads / LPR;
  __shared__ float sm_m[G][NG], sm_l[G][NG];
  __shared__ float sm_acc[G][NG][D];

  const int sk = blockIdx.x;                       // s * H_kv + hkv
  const int s = sk / p.Hkv, hkv = sk % p.Hkv;
  const int grp = threadIdx.x / LPR, gl = threadIdx.x % LPR;

  const int32_t* idx;
  int len, ng, wbase;
  set_rows<WIN>(p, s, hkv, idx, len, ng, wbase);
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
    // Rows of the next iteration: fetched into L2 now (one prefetch per
    // 128-byte line), so that their loads find them there.
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int r = base + NG * kUnroll + u * NG;
      if (r < len && (gl & 7) == 0) {
        const int j = row_slot<WIN>(p, idx, r, ng, wbase);
        if (j >= 0 && j < p.L) {
          asm volatile("prefetch.global.L2 [%0];" ::"l"(Kb + (int64_t)j * D));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(Vb + (int64_t)j * D));
        }
      }
    }
    // Scores: each K row unpacked once, dotted with the G queries.
    float sc[G][kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float kf[8];
      bf16x8_to_f32(kv[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float d = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) d = fmaf(q[g][c], kf[c], d);
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        sc[g][u] = valid[u] ? d : -INFINITY;
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
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[g][c] *= alpha;
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
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[g][c] = fmaf(sc[g][u], vf[c], acc[g][c]);
      }
    }
  }

#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (gl == 0) {
      sm_m[g][grp] = m[g];
      sm_l[g][grp] = l[g];
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) sm_acc[g][grp][gl * 8 + c] = acc[g][c];
  }
  __syncthreads();

  for (int t = threadIdx.x; t < G * D; t += kGatherThreads) {
    const int g = t / D, c = t % D;
    float M = -INFINITY;
    for (int k = 0; k < NG; ++k) M = fmaxf(M, sm_m[g][k]);
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int k = 0; k < NG; ++k) {
        const float w = ex2(sm_m[g][k] - M);
        L = fmaf(sm_l[g][k], w, L);
        o = fmaf(sm_acc[g][k][c], w, o);
      }
    }
    const float out = L > 0.f ? o / L : 0.f;
    const int64_t sh = (int64_t)s * p.H + hkv * G + g;
    p.O[sh * D + c] = __bfloat16_as_ushort(__float2bfloat16_rn(out));
    if (c == 0 && p.lse) p.lse[sh] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
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
#define SA_GROUP(DD, GG)                                                                    \
  if (win) gather_group_kernel<DD, GG, true><<<nk, kGatherThreads, 0, stream>>>(p);       \
  else gather_group_kernel<DD, GG, false><<<nk, kGatherThreads, 0, stream>>>(p);
#define SA_SINGLE(DD)                                                                       \
  if (win) gather_kernel<DD, true><<<(unsigned)n, kGatherThreads, 0, stream>>>(p);        \
  else gather_kernel<DD, false><<<(unsigned)n, kGatherThreads, 0, stream>>>(p);
  if (d != 64 && d != 128) return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  if (shared && G == 4 && d == 128) { SA_GROUP(128, 4) }
  else if (shared && G == 2 && d == 128) { SA_GROUP(128, 2) }
  else if (shared && G == 4 && d == 64) { SA_GROUP(64, 4) }
  else if (shared && G == 2 && d == 64) { SA_GROUP(64, 2) }
  else if (d == 128) { SA_SINGLE(128) }
  else { SA_SINGLE(64) }
#undef SA_GROUP
#undef SA_SINGLE
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "gather launch");
  return SA_OK;
}

}  // namespace sa
