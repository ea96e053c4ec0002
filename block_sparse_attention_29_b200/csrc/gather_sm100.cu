// gather_sm100.cu -- attention of one query per (sequence, head) over an
// explicit, sorted index set of a KV cache (decode over a sparse G; "Sparse
// Attention Weights Assumption": out = sum_{j in G} alpha'_j v_j with the
// softmax taken over G; the KV cache of "SAS: Sparse Attention Synthesizer",
// Step 4 challenge 2).
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

template <int D>
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

  const int32_t* idx = p.idx + ((int64_t)s * p.H_idx + hi) * p.n_idx;
  int len = p.idx_len ? __ldg(p.idx_len + (int64_t)s * p.H_idx + hi) : p.n_idx;
  len = len < 0 ? 0 : (len > p.n_idx ? p.n_idx : len);
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
      int j = r < len ? __ldg(idx + r) : -1;
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

}  // namespace

int launch_gather(const GatherParams& p, int d, cudaStream_t stream) {
  const int64_t n = (int64_t)p.S * p.H;
  if (n == 0) return SA_OK;
  if (n > INT32_MAX) return set_error(SA_ERR_UNSUPPORTED, "S*H = %lld too large", (long long)n);
  if (d == 128) gather_kernel<128><<<(unsigned)n, kGatherThreads, 0, stream>>>(p);
  else if (d == 64) gather_kernel<64><<<(unsigned)n, kGatherThreads, 0, stream>>>(p);
  else return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "gather launch");
  return SA_OK;
}

}  // namespace sa
