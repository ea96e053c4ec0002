// noalloc.cu -- sparse_attn_prefill_noalloc: a prefill entry point that
// allocates no device memory.
//
// The regular entry points keep each compiled pattern (per-tile block lists,
// the work order and a copy of the random table) in device memory obtained
// with cudaMalloc.  Some callers cannot allocate device memory at call time --
// for example code running under a memory pool or allocator that owns the
// whole device, or a runtime that forbids allocation on its inference path.
// This entry point compiles the pattern on the host and copies the result into
// a fixed, file-scope device array instead, then launches the same prefill
// kernel.  The array is static device memory of kNoAllocScratchBytes.  CUDA
// loads the library's device code lazily, so the array is reserved on a device
// when the library's code is first used there (for a caller that only uses
// this entry point: its first call) and held until the process exits.  A
// caller whose device memory is about to be handed to an external pool should
// make one call (a warm-up) before the pool takes the device.
//
// Set-up: the first call on a device, with that device current, looks up the
// array's device address with cudaGetSymbolAddress (the array's name in host
// code is only a host-side stand-in, not a device address).  Make that first
// call before any stream capture begins.
//
// Every argument and size check, the size limit included, runs on the host
// before the first CUDA call, so a rejected call queues no device work.
//
// Sharing: every call uses the same array and leaves the last call's contents
// in it.  The plan data is rewritten in full by each call; the two work-queue
// counters at the start of the array must start at zero and are cleared by
// each call before its launch.  Calls whose copies and kernels may overlap on
// the GPU (for example on two streams without ordering between them) race on
// the array.
#include <algorithm>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "common.h"

namespace sa {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDev = 64;
unsigned char* g_scratch_ptr[kMaxDev] = {nullptr};
std::mutex g_scratch_mu;

int scratch_address(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDev) return set_error(SA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_scratch_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_scratch_ptr[dev];
  return SA_OK;
}

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }
}  // namespace

}  // namespace sa

using namespace sa;

extern "C" int sparse_attn_prefill_noalloc(const void* Q, const void* K, const void* V, void* O,
                                           int B, int H, int H_kv, int N, int d,
                                           const sa_pattern_t* pat, float* lse_out,
                                           sa_stream_t stream) {
  if (!pat) return set_error(SA_ERR_INVALID_ARG, "pattern descriptor is NULL");
  if (!Q || !K || !V || !O) return set_error(SA_ERR_INVALID_ARG, "Q, K, V and O must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
       reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(O)) & 15u)
    return set_error(SA_ERR_INVALID_ARG, "Q, K, V and O must be 16-byte aligned");
  int rc = check_shapes(pat, B, H, H_kv, N, d);
  if (rc) return rc;
  if (pat->thresholds && pat->block_q != kTileQ)
    return set_error(SA_ERR_UNSUPPORTED, "the block-skip rule needs block_q = 128");
  const bool rnd = pat->n_random > 0 && pat->random_table != nullptr;

  // Host compile (host memory only).
  CompiledPattern cp;
  rc = compile_pattern(pat, H, N, kTileQ, kTileK, &cp);
  if (rc) return rc;
  const int T = cp.T;
  const int dil = pat->dilation > 1 ? pat->dilation : 1;
  if (dil > 1 && pat->thresholds)
    return set_error(SA_ERR_UNSUPPORTED, "a dilated window takes no block-skip thresholds");
  const int64_t n_units = int64_t(B) * dil * H * T;
  const int nrb = rnd ? (N + pat->random_block - 1) / pat->random_block : 0;
  const size_t b_row = round256(cp.row_ptr.size() * 4);
  const size_t b_ent = round256(std::max<size_t>(cp.kb.size(), 1) * 4);
  const size_t b_units = round256(size_t(n_units) * 4);
  const size_t b_rtab = rnd ? round256(size_t(H) * nrb * pat->n_random * 4) : 0;
  const size_t b_sched = 256;   // work-queue counters
  const size_t need = b_sched + b_row + b_ent + b_units + b_rtab;
  if (need > kNoAllocScratchBytes)
    return set_error(SA_ERR_INVALID_ARG,
                     "pattern needs %zu bytes of plan data; the no-alloc entry point holds at most "
                     "%zu (use sparse_attn_plan_create)",
                     need, kNoAllocScratchBytes);

  std::vector<int32_t> entries(cp.kb.size());
  for (size_t e = 0; e < cp.kb.size(); ++e) entries[e] = entry_pack(cp.kb[e], !cp.full[e]);
  // No tile is split here: the pieces' workspace would not fit the scratch.
  UnitOrder order;
  build_units(cp, B * dil, H, H_kv, N / dil, d, -1, &order);
  const std::vector<int32_t>& units = order.units;

  unsigned char* base = nullptr;
  rc = scratch_address(&base);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* d_sched = reinterpret_cast<int32_t*>(base);
  int32_t* d_row = reinterpret_cast<int32_t*>(base + b_sched);
  int32_t* d_ent = reinterpret_cast<int32_t*>(base + b_sched + b_row);
  int32_t* d_units = reinterpret_cast<int32_t*>(base + b_sched + b_row + b_ent);
  int32_t* d_rtab =
      rnd ? reinterpret_cast<int32_t*>(base + b_sched + b_row + b_ent + b_units) : nullptr;
  cudaError_t e = cudaMemsetAsync(d_sched, 0, 2 * sizeof(int32_t), st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(d_row, cp.row_ptr.data(), cp.row_ptr.size() * 4, cudaMemcpyHostToDevice,
                        st);
  if (e == cudaSuccess && !entries.empty())
    e = cudaMemcpyAsync(d_ent, entries.data(), entries.size() * 4, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(d_units, units.data(), units.size() * 4, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && rnd)
    e = cudaMemcpyAsync(d_rtab, pat->random_table, size_t(H) * nrb * pat->n_random * 4,
                        cudaMemcpyHostToDevice, st);
  // Copies from pageable host memory are staged before cudaMemcpyAsync
  // returns, so the host vectors may be released when this function returns.
  if (e != cudaSuccess) return cuda_error(e, "cudaMemcpyAsync(no-alloc scratch)");

  PrefillParams p;
  std::memset(&p, 0, sizeof p);
  rc = make_tmap(&p.tm_q, Q, d, N, B * H, kTileQ, dil);
  if (!rc) rc = make_tmap(&p.tm_k, K, d, N, B * H_kv, kTileK, dil);
  if (!rc) rc = make_tmap(&p.tm_v, V, d, N, B * H_kv, kTileK, dil);
  if (rc) return rc;
  p.O = static_cast<uint16_t*>(O);
  p.lse = lse_out;
  p.row_ptr = d_row;
  p.entries = d_ent;
  p.units = d_units;
  p.sched = d_sched;
  p.rtab = d_rtab;
  p.thresholds = pat->thresholds;
  p.n_units = int(n_units);
  p.B = B;
  p.H = H;
  p.Hkv = H_kv;
  p.N = N / dil;
  p.dil = dil;
  p.T = T;
  p.n_kb = cp.n_kb;
  p.head_pat = cp.H_pat > 1 ? 1 : 0;
  p.causal = pat->causal;
  p.window = pat->window;
  p.n_global = pat->n_global;
  p.block_local = pat->block_local;
  p.random_block = pat->random_block;
  p.n_random = rnd ? pat->n_random : 0;
  p.skip_denominator = pat->skipped_in_denominator ? 1 : 0;
  p.row_level = pat->row_level_skip ? 1 : 0;
  const float scale = pat->scale != 0.f ? pat->scale : 1.0f / sqrtf(float(d));
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.gate = pat->thresholds ? 1 : 0;
  p.want_stats = p.gate;
  p.err = device_error_word();
  if (!p.err) return set_error(SA_ERR_CUDA, "device error word unavailable");
  return launch_prefill(p, d, st);
}
