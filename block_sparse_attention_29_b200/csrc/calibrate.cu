// calibrate.cu -- per-head threshold calibration of the block-skip rule.
//
// "Block Sparse Flash Attention" (AI Radio episode, improvements): the
// thresholds are learned once per layer and head from a small calibration
// set.  Here: tau_h = the statistic of rank floor((n_h - 1) * q) (ascending,
// 0-based) among head h's full blocks of a statistics pass, n_h their number;
// q = 0.5 gives the lower median.  Exact selection by a 4-pass radix select
// (8 bits per pass) on order-preserving integer keys; one CTA per head.
#include <cmath>

#include "common.h"

namespace sa {
namespace {

constexpr int kCalThreads = 512;

__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

__global__ void __launch_bounds__(kCalThreads) calibrate_kernel(
    const float* __restrict__ stat, const int32_t* __restrict__ row_ptr,
    const int32_t* __restrict__ entries, int head_pat, int B, int H, int T, int n_kb, double q,
    float* __restrict__ out) {
  __shared__ uint32_t hist[256];
  __shared__ unsigned long long s_count;
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ unsigned long long s_rank;
  const int h = blockIdx.x;
  const int hp = head_pat ? h : 0;
  const int32_t* rp = row_ptr + (int64_t)hp * T;

  if (threadIdx.x == 0) s_count = 0;
  __syncthreads();
  unsigned long long local = 0;
  for (int t = 0; t < T; ++t)
    for (int e = rp[t] + threadIdx.x; e < rp[t + 1]; e += kCalThreads)
      if (!(entries[e] & 1)) local += B;
  atomicAdd(&s_count, local);
  __syncthreads();
  const unsigned long long n = s_count;
  if (n == 0) {
    if (threadIdx.x == 0) out[h] = -INFINITY;
    return;
  }
  if (threadIdx.x == 0) {
    s_rank = (unsigned long long)floor((double)(n - 1) * q);
    if (s_rank > n - 1) s_rank = n - 1;
    s_prefix = 0;
    s_mask = 0;
  }
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int k = threadIdx.x; k < 256; k += kCalThreads) hist[k] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int t = 0; t < T; ++t) {
      const int len = rp[t + 1] - rp[t];
      for (int w = threadIdx.x; w < B * len; w += kCalThreads) {
        const int b = w / len, e = rp[t] + w % len;
        const int32_t ent = entries[e];
        if (ent & 1) continue;   // partial blocks are never skipped
        const float v = stat[(((int64_t)b * H + h) * T + t) * n_kb + (ent >> 1)];
        const uint32_t key = float_key(v);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long r = s_rank, cum = 0;
      int digit = 255;
      for (int dgt = 0; dgt < 256; ++dgt) {
        if (cum + hist[dgt] > r) {
          digit = dgt;
          break;
        }
        cum += hist[dgt];
      }
      s_rank = r - cum;
      s_prefix = prefix | (uint32_t(digit) << shift);
      s_mask = mask | (255u << shift);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) out[h] = key_float(s_prefix);
}

}  // namespace

int launch_calibrate(const float* stat, const int32_t* row_ptr, const int32_t* entries,
                     int head_pat, int B, int H, int T, int n_kb, double q, float* out,
                     cudaStream_t stream) {
  if (H <= 0) return SA_OK;
  calibrate_kernel<<<H, kCalThreads, 0, stream>>>(stat, row_ptr, entries, head_pat, B, H, T, n_kb,
                                                  q, out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "calibrate launch");
  return SA_OK;
}

}  // namespace sa
