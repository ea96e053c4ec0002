// api.cu -- the C ABI declared in include/sparse_attn.h: argument checks,
// plans (compiled pattern + work order in device memory), TMA tensor maps,
// launches, the per-process plan cache and the device error word.
#include <algorithm>
#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <numeric>
#include <string>
#include <vector>

#include "common.h"

namespace sa {

// ------------------------------------------------------------- errors --
namespace {
thread_local char g_msg[512] = "";
}

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return code;
}

int cuda_error(cudaError_t e, const char* what) {
  if (e == cudaErrorMemoryAllocation)
    return set_error(SA_ERR_NO_MEMORY, "%s: %s", what, cudaGetErrorString(e));
  return set_error(SA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// -------------------------------------------------- device error word --
__device__ int g_device_error_word = 0;

namespace {
constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {nullptr};
std::mutex g_err_mu;
}  // namespace

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  return g_err_ptr[dev];
}

// -------------------------------------------------------- tensor maps --
namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_current_device(int want) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev != want)
    return set_error(SA_ERR_INVALID_ARG, "plan was created on device %d, current device is %d",
                     want, dev);
  return SA_OK;
}
}  // namespace

// 4-D bf16 map over a [BH][N][d] tensor seen as [BH][N/dil][dil][d]:
// coordinates (x, residue r, position m within the residue class, slice) address
// row m*dil + r; box {64, 1, rows, 1}, 128-byte swizzle, so a box is `rows`
// rows of one class, dil rows apart (dil = 1: plain consecutive rows).  Rows
// past N/dil read as zero.  N % dil == 0 is checked by the caller, so no
// in-bounds coordinate reaches past row N - 1 of its slice.
int make_tmap(CUtensorMap* m, const void* base, int d, int N, int BH, int rows, int dil) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(SA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  if (dil < 1 || N % dil != 0) return set_error(SA_ERR_INVALID_ARG, "dilation %d, N = %d", dil, N);
  const cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(dil), cuuint64_t(N / dil), cuuint64_t(BH)};
  const cuuint64_t strides[3] = {cuuint64_t(d) * 2, cuuint64_t(dil) * d * 2,
                                 cuuint64_t(N) * d * 2};
  const cuuint32_t box[4] = {64, 1, cuuint32_t(rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return SA_OK;
}

// Shape and descriptor checks shared by every prefill entry point.
int check_shapes(const sa_pattern_t* pat, int B, int H, int Hkv, int N, int d) {
  if (!pat) return set_error(SA_ERR_INVALID_ARG, "pattern descriptor is NULL");
  if (B <= 0 || H <= 0 || Hkv <= 0 || N <= 0)
    return set_error(SA_ERR_INVALID_ARG, "B, H, H_kv and N must be positive");
  if (H % Hkv != 0) return set_error(SA_ERR_INVALID_ARG, "H = %d is not a multiple of H_kv = %d", H, Hkv);
  if (d != 64 && d != 128) return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  if (pat->block_k != kTileK)
    return set_error(SA_ERR_UNSUPPORTED, "block_k = %d (the kernels use 64-key blocks)", pat->block_k);
  if (pat->block_q != 64 && pat->block_q != 128)
    return set_error(SA_ERR_UNSUPPORTED, "block_q = %d (64 or 128 supported)", pat->block_q);
  if (pat->n_random > 0 && pat->random_table && (pat->random_block <= 0 || pat->random_block % kTileK))
    return set_error(SA_ERR_UNSUPPORTED, "random_block = %d must be a positive multiple of 64",
                     pat->random_block);
  if (pat->row_level_skip && pat->skipped_in_denominator)
    return set_error(SA_ERR_UNSUPPORTED,
                     "the row-level block-skip reading is not combined with skipped keys kept "
                     "in the denominator");
  if (N >= (1 << 28)) return set_error(SA_ERR_UNSUPPORTED, "N = %d too large", N);
  const int dil = pat->dilation > 1 ? pat->dilation : 1;
  const int64_t units = int64_t(B) * dil * H * ((N / dil + kTileQ - 1) / kTileQ);
  if (units > INT32_MAX) return set_error(SA_ERR_UNSUPPORTED, "B*H*tiles too large");
  if (int64_t(B) * H > 65535 || int64_t(B) * Hkv > 65535)
    return set_error(SA_ERR_UNSUPPORTED, "B*H must not exceed 65535");
  return SA_OK;
}

}  // namespace sa

// ================================================================= plans ==
struct sa_plan {
  sa_pattern_t pat{};
  int B = 0, H = 0, Hkv = 0, N = 0, d = 0, device = 0;
  int T = 0, n_kb = 0, H_pat = 0;
  int dil = 1;                 // dilation: the plan's lists cover one of dil residue classes
  int n_units = 0;
  int32_t* d_row_ptr = nullptr;
  int32_t* d_entries = nullptr;
  int32_t* d_units = nullptr;
  int4* d_pieces = nullptr;    // split-tile pieces (two int4 each, see PrefillParams)
  int* d_split_cnt = nullptr;  // pieces finished per split tile, zero between launches
  float* d_part = nullptr;     // pieces' partial results [slot][d + 2][128]
  int n_split = 0;
  int32_t* d_rtab = nullptr;
  int* d_sched = nullptr;      // work-queue counters, zero between launches
  sa_plan_info_t info{};
};

using namespace sa;

namespace {

void plan_free(sa_plan_t* p) {
  if (!p) return;
  int prev = -1;
  cudaGetDevice(&prev);
  if (prev != p->device) cudaSetDevice(p->device);
  cudaDeviceSynchronize();
  cudaFree(p->d_row_ptr);
  cudaFree(p->d_entries);
  cudaFree(p->d_units);
  cudaFree(p->d_pieces);
  cudaFree(p->d_split_cnt);
  cudaFree(p->d_part);
  cudaFree(p->d_rtab);
  cudaFree(p->d_sched);
  if (prev >= 0 && prev != p->device) cudaSetDevice(prev);
  delete p;
}

template <typename T>
int upload(T** dst, const T* src, size_t n) {
  *dst = nullptr;
  if (n == 0) n = 1;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(dst), n * sizeof(T));
  if (e != cudaSuccess) return cuda_error(e, "cudaMalloc");
  if (src) {
    e = cudaMemcpy(*dst, src, n * sizeof(T), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_error(e, "cudaMemcpy");
  }
  return SA_OK;
}

// Key of the one-shot plan cache: every descriptor field but the pointers,
// the random table's contents, the shapes and the device.
std::string cache_key(const sa_pattern_t* p, int B, int H, int Hkv, int N, int d, int dev) {
  std::string k;
  auto put = [&k](const void* src, size_t n) { k.append(static_cast<const char*>(src), n); };
  const int32_t f[] = {p->causal, p->window, p->n_global, p->block_local, p->block_q,
                       p->block_k, p->random_block, p->n_random, p->dilation > 1 ? p->dilation : 1,
                       p->skipped_in_denominator ? 1 : 0, p->row_level_skip ? 1 : 0,
                       B, H, Hkv, N, d, dev};
  put(f, sizeof f);
  put(&p->scale, sizeof p->scale);
  if (p->n_random > 0 && p->random_table && p->random_block > 0) {
    const int nrb = (N + p->random_block - 1) / p->random_block;
    put(p->random_table, size_t(H) * nrb * p->n_random * sizeof(int32_t));
  } else {
    const char none = 0;
    put(&none, 1);
  }
  return k;
}

std::mutex g_cache_mu;
std::map<std::string, sa_plan_t*>* g_cache = nullptr;

int fill_prefill_params(const sa_plan_t* plan, const void* Q, const void* K, const void* V,
                        void* O, const float* thresholds, float* lse, uint8_t* mask,
                        float* stat, PrefillParams* p) {
  std::memset(p, 0, sizeof *p);
  const int dil = plan->dil;
  int rc = make_tmap(&p->tm_q, Q, plan->d, plan->N, plan->B * plan->H, kTileQ, dil);
  if (!rc) rc = make_tmap(&p->tm_k, K, plan->d, plan->N, plan->B * plan->Hkv, kTileK, dil);
  if (!rc) rc = make_tmap(&p->tm_v, V, plan->d, plan->N, plan->B * plan->Hkv, kTileK, dil);
  if (rc) return rc;
  p->O = static_cast<uint16_t*>(O);
  p->lse = lse;
  p->mask_out = mask;
  p->stat_out = stat;
  p->row_ptr = plan->d_row_ptr;
  p->entries = plan->d_entries;
  p->units = plan->d_units;
  p->pieces = plan->d_pieces;
  p->part = plan->d_part;
  p->split_cnt = plan->d_split_cnt;
  p->n_split = plan->n_split;
  p->sched = plan->d_sched;
  p->rtab = plan->d_rtab;
  p->thresholds = thresholds;
  p->n_units = plan->n_units;
  p->B = plan->B;
  p->H = plan->H;
  p->Hkv = plan->Hkv;
  p->N = plan->N / dil;
  p->dil = dil;
  p->T = plan->T;
  p->n_kb = plan->n_kb;
  p->head_pat = plan->H_pat > 1 ? 1 : 0;
  p->causal = plan->pat.causal;
  p->window = plan->pat.window;
  p->n_global = plan->pat.n_global;
  p->block_local = plan->pat.block_local;
  p->random_block = plan->pat.random_block;
  p->n_random = plan->d_rtab ? plan->pat.n_random : 0;
  p->skip_denominator = plan->pat.skipped_in_denominator ? 1 : 0;
  p->row_level = plan->pat.row_level_skip ? 1 : 0;
  const float scale = plan->pat.scale != 0.f ? plan->pat.scale : 1.0f / sqrtf(float(plan->d));
  p->scale = scale;
  p->scale_log2 = scale * 1.4426950408889634f;
  p->err = device_error_word();
  if (!p->err) return set_error(SA_ERR_CUDA, "device error word unavailable");
  return SA_OK;
}

}  // namespace

extern "C" {

const char* sparse_attn_last_error(void) { return sa::g_msg; }

int sparse_attn_work_order(const sa_pattern_t* pat, int B, int H, int H_kv, int N, int d,
                           int max_unit_blocks, int64_t* n_units_out, int64_t* n_pieces_out,
                           int64_t* n_split_out, int32_t* units, int32_t* pieces,
                           int32_t* split) {
  int rc = check_shapes(pat, B, H, H_kv, N, d);
  if (rc) return rc;
  CompiledPattern cp;
  rc = compile_pattern(pat, H, N, kTileQ, kTileK, &cp);
  if (rc) return rc;
  const int dil = pat->dilation > 1 ? pat->dilation : 1;
  UnitOrder order;
  build_units(cp, B * dil, H, H_kv, N / dil, d, max_unit_blocks, &order);
  if (n_units_out) *n_units_out = int64_t(order.units.size());
  if (n_pieces_out) *n_pieces_out = int64_t(order.pieces.size());
  if (n_split_out) *n_split_out = int64_t(order.split.size());
  if (units) {
    if ((!pieces && !order.pieces.empty()) || (!split && !order.split.empty()))
      return set_error(SA_ERR_INVALID_ARG, "pieces and split must be given with units");
    std::copy(order.units.begin(), order.units.end(), units);
    for (size_t k = 0; k < order.pieces.size(); ++k) {
      const Piece& pc = order.pieces[k];
      pieces[4 * k + 0] = pc.id;
      pieces[4 * k + 1] = pc.k0;
      pieces[4 * k + 2] = pc.n;
      pieces[4 * k + 3] = pc.slot;
    }
    for (size_t k = 0; k < order.split.size(); ++k) {
      const SplitTile& st = order.split[k];
      split[4 * k + 0] = st.id;
      split[4 * k + 1] = st.first_slot;
      split[4 * k + 2] = st.n_pieces;
      split[4 * k + 3] = 0;
    }
  }
  return SA_OK;
}

int sparse_attn_compile_pattern(const sa_pattern_t* pat, int H, int N, int tile_q, int tile_k,
                                int* H_pat_out, int* T_out, int64_t* n_entries_out,
                                int32_t* row_ptr, int32_t* kb, uint8_t* full, int64_t* cnt) {
  CompiledPattern cp;
  int rc = compile_pattern(pat, H, N, tile_q, tile_k, &cp);
  if (rc) return rc;
  if (H_pat_out) *H_pat_out = cp.H_pat;
  if (T_out) *T_out = cp.T;
  if (n_entries_out) *n_entries_out = int64_t(cp.kb.size());
  if (row_ptr) {
    if (!kb || !full) return set_error(SA_ERR_INVALID_ARG, "kb and full must be given with row_ptr");
    std::copy(cp.row_ptr.begin(), cp.row_ptr.end(), row_ptr);
    std::copy(cp.kb.begin(), cp.kb.end(), kb);
    std::copy(cp.full.begin(), cp.full.end(), full);
    if (cnt) std::copy(cp.cnt.begin(), cp.cnt.end(), cnt);
  }
  return SA_OK;
}

int sparse_attn_plan_create(const sa_pattern_t* pat, int B, int H, int H_kv, int N, int d,
                            sa_plan_t** out) {
  return sparse_attn_plan_create_ex(pat, B, H, H_kv, N, d, SA_KERNEL_AUTO, out);
}

int sparse_attn_plan_create_ex(const sa_pattern_t* pat, int B, int H, int H_kv, int N, int d,
                               int kernel, sa_plan_t** out) {
  sa_plan_options_t o;
  o.kernel = kernel;
  o.max_unit_blocks = 0;
  return sparse_attn_plan_create_opts(pat, B, H, H_kv, N, d, &o, out);
}

int sparse_attn_plan_create_opts(const sa_pattern_t* pat, int B, int H, int H_kv, int N, int d,
                                 const sa_plan_options_t* opts, sa_plan_t** out) {
  if (!out) return set_error(SA_ERR_INVALID_ARG, "out is NULL");
  const int kernel = opts ? opts->kernel : SA_KERNEL_AUTO;
  const int max_unit_blocks = opts ? opts->max_unit_blocks : 0;
  if (kernel != SA_KERNEL_AUTO && kernel != SA_KERNEL_SINGLE_HEAD)
    return set_error(SA_ERR_INVALID_ARG, "kernel = %d (not an SA_KERNEL_* value)", kernel);
  *out = nullptr;
  int rc = check_shapes(pat, B, H, H_kv, N, d);
  if (rc) return rc;
  const auto t0 = std::chrono::steady_clock::now();
  CompiledPattern cp;
  rc = compile_pattern(pat, H, N, kTileQ, kTileK, &cp);
  if (rc) return rc;
  const int dil = pat->dilation > 1 ? pat->dilation : 1;
  sa_plan_t* plan = new sa_plan_t;
  plan->pat = *pat;
  plan->pat.random_table = nullptr;
  plan->pat.thresholds = nullptr;
  plan->B = B;
  plan->H = H;
  plan->Hkv = H_kv;
  plan->N = N;
  plan->d = d;
  plan->T = cp.T;
  plan->n_kb = cp.n_kb;
  plan->H_pat = cp.H_pat;
  plan->dil = dil;
  cudaGetDevice(&plan->device);

  // Block lists as packed entries; accounting over all (b, h).
  std::vector<int32_t> entries(cp.kb.size());
  int64_t per_pat_blocks = 0, per_pat_full = 0, per_pat_pairs = 0;
  for (size_t e = 0; e < cp.kb.size(); ++e) {
    entries[e] = entry_pack(cp.kb[e], !cp.full[e]);
    per_pat_full += cp.full[e];
    per_pat_pairs += cp.cnt[e];
  }
  per_pat_blocks = int64_t(cp.kb.size());
  // B*dil independent sequences: each residue class of a dilated window runs the lists
  const int Bd = B * dil;
  const int64_t rep = int64_t(Bd) * (cp.H_pat == 1 ? H : 1);
  plan->info.T_q = cp.T;
  plan->info.n_kb = cp.n_kb;
  plan->info.n_units = int64_t(Bd) * H * cp.T;
  plan->info.blocks = per_pat_blocks * rep;
  plan->info.blocks_full = per_pat_full * rep;
  plan->info.pairs = per_pat_pairs * rep;
  if (pat->block_q == kTileQ) {
    plan->info.blocks_desc = plan->info.blocks;
  } else {
    CompiledPattern cd;
    rc = compile_pattern(pat, H, N, pat->block_q, pat->block_k, &cd);
    if (rc) {
      delete plan;
      return rc;
    }
    plan->info.blocks_desc = int64_t(cd.kb.size()) * int64_t(Bd) * (cd.H_pat == 1 ? H : 1);
  }

  UnitOrder order;
  build_units(cp, Bd, H, H_kv, N / dil, d, max_unit_blocks, &order);
  const std::vector<int32_t>& units = order.units;
  plan->n_units = int(units.size());
  plan->n_split = int(order.split.size());
  plan->info.split_tiles = int64_t(order.split.size());
  plan->info.queue_units = int64_t(units.size());
  plan->info.workspace_bytes = order.n_slots * piece_slot_floats(d) * int64_t(sizeof(float));

  rc = upload(&plan->d_row_ptr, cp.row_ptr.data(), cp.row_ptr.size());
  if (!rc) rc = upload(&plan->d_entries, entries.data(), entries.size());
  if (!rc) rc = upload(&plan->d_units, units.data(), units.size());
  if (!rc && !order.pieces.empty()) {
    static_assert(sizeof(Piece) == 2 * sizeof(int4), "a piece is two int4");
    rc = upload(&plan->d_pieces, reinterpret_cast<const int4*>(order.pieces.data()),
                2 * order.pieces.size());
    if (!rc) {
      const std::vector<int32_t> zeros(order.split.size(), 0);
      rc = upload(&plan->d_split_cnt, zeros.data(), zeros.size());
    }
    if (!rc)
      rc = upload(&plan->d_part, static_cast<const float*>(nullptr),
                  size_t(order.n_slots * piece_slot_floats(d)));
  }
  if (!rc) {
    const int zeros[2] = {0, 0};
    rc = upload(&plan->d_sched, zeros, 2);
  }
  if (!rc && pat->n_random > 0 && pat->random_table) {
    const int nrb = (N + pat->random_block - 1) / pat->random_block;
    rc = upload(&plan->d_rtab, pat->random_table, size_t(H) * nrb * pat->n_random);
  }
  if (rc) {
    plan_free(plan);
    return rc;
  }
  plan->info.compile_ms =
      std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
  *out = plan;
  return SA_OK;
}

int sparse_attn_plan_info(const sa_plan_t* plan, sa_plan_info_t* info) {
  if (!plan || !info) return set_error(SA_ERR_INVALID_ARG, "plan or info is NULL");
  *info = plan->info;
  return SA_OK;
}

void sparse_attn_plan_destroy(sa_plan_t* plan) { plan_free(plan); }

int sparse_attn_prefill_plan(const sa_plan_t* plan, const void* Q, const void* K, const void* V,
                             void* O, const float* thresholds, float* lse_out,
                             uint8_t* block_mask_out, float* block_stat_out, sa_stream_t stream) {
  if (!plan) return set_error(SA_ERR_INVALID_ARG, "plan is NULL");
  if (!Q || !K || !V || !O) return set_error(SA_ERR_INVALID_ARG, "Q, K, V and O must be non-NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return set_error(SA_ERR_INVALID_ARG, "Q, K, V and O must be 16-byte aligned");
  if (thresholds && plan->pat.block_q != kTileQ)
    return set_error(SA_ERR_UNSUPPORTED, "the block-skip rule needs block_q = 128");
  if (plan->dil > 1 && (thresholds || block_mask_out || block_stat_out))
    return set_error(SA_ERR_UNSUPPORTED,
                     "a dilated plan takes no thresholds, block mask or block statistics");
  int rc = check_current_device(plan->device);
  if (rc) return rc;
  PrefillParams p;
  rc = fill_prefill_params(plan, Q, K, V, O, thresholds, lse_out, block_mask_out, block_stat_out, &p);
  if (rc) return rc;
  p.gate = thresholds ? 1 : 0;
  p.stats_only = 0;
  p.want_stats = (thresholds || block_stat_out) ? 1 : 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (block_mask_out) {
    cudaError_t e = cudaMemsetAsync(block_mask_out, 0,
                                    size_t(plan->B) * plan->H * plan->T * plan->n_kb, st);
    if (e != cudaSuccess) return cuda_error(e, "cudaMemsetAsync");
  }
  return launch_prefill(p, plan->d, st);
}

int sparse_attn_block_stats(const sa_plan_t* plan, const void* Q, const void* K,
                            float* block_stat_out, uint8_t* block_mask_out, sa_stream_t stream) {
  if (!plan) return set_error(SA_ERR_INVALID_ARG, "plan is NULL");
  if (!Q || !K || !block_stat_out)
    return set_error(SA_ERR_INVALID_ARG, "Q, K and block_stat_out must be non-NULL");
  if (!aligned16(Q) || !aligned16(K)) return set_error(SA_ERR_INVALID_ARG, "Q and K must be 16-byte aligned");
  if (plan->pat.block_q != kTileQ)
    return set_error(SA_ERR_UNSUPPORTED, "the block-skip rule needs block_q = 128");
  if (plan->dil > 1) return set_error(SA_ERR_UNSUPPORTED, "no block statistics for a dilated plan");
  int rc = check_current_device(plan->device);
  if (rc) return rc;
  PrefillParams p;
  // V is never read in this pass; its map points at K so the descriptor is valid.
  rc = fill_prefill_params(plan, Q, K, K, nullptr, nullptr, nullptr, block_mask_out,
                           block_stat_out, &p);
  if (rc) return rc;
  p.gate = 1;
  p.stats_only = 1;
  p.want_stats = 1;
  p.skip_denominator = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (block_mask_out) {
    cudaError_t e = cudaMemsetAsync(block_mask_out, 0,
                                    size_t(plan->B) * plan->H * plan->T * plan->n_kb, st);
    if (e != cudaSuccess) return cuda_error(e, "cudaMemsetAsync");
  }
  return launch_prefill(p, plan->d, st);
}

int sparse_attn_calibrate(const sa_plan_t* plan, const float* block_stat, double q,
                          float* thresholds_out, sa_stream_t stream) {
  if (!plan || !block_stat || !thresholds_out)
    return set_error(SA_ERR_INVALID_ARG, "plan, block_stat and thresholds_out must be non-NULL");
  if (!(q >= 0.0 && q <= 1.0)) return set_error(SA_ERR_INVALID_ARG, "q = %g outside [0, 1]", q);
  if (plan->dil > 1) return set_error(SA_ERR_UNSUPPORTED, "no calibration for a dilated plan");
  int rc = check_current_device(plan->device);
  if (rc) return rc;
  return launch_calibrate(block_stat, plan->d_row_ptr, plan->d_entries, plan->H_pat > 1 ? 1 : 0,
                          plan->B, plan->H, plan->T, plan->n_kb, q, thresholds_out,
                          reinterpret_cast<cudaStream_t>(stream));
}

int sparse_attn_prefill(const void* Q, const void* K, const void* V, void* O, int B, int H, int H_kv,
                        int N, int d, const sa_pattern_t* pat, float* lse_out,
                        uint8_t* block_mask_out, sa_stream_t stream) {
  int rc = check_shapes(pat, B, H, H_kv, N, d);
  if (rc) return rc;
  rc = validate_pattern(pat, H, N);
  if (rc) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  const std::string key = cache_key(pat, B, H, H_kv, N, d, dev);
  sa_plan_t* plan = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    if (!g_cache) g_cache = new std::map<std::string, sa_plan_t*>();
    auto it = g_cache->find(key);
    if (it != g_cache->end()) {
      plan = it->second;
    } else {
      rc = sparse_attn_plan_create(pat, B, H, H_kv, N, d, &plan);
      if (rc) return rc;
      (*g_cache)[key] = plan;
    }
  }
  return sparse_attn_prefill_plan(plan, Q, K, V, O, pat->thresholds, lse_out, block_mask_out,
                                  nullptr, stream);
}

int sparse_attn_gather(const void* Q, const void* K, const void* V, const int32_t* idx,
                       const int32_t* idx_len, void* O, int S, int H, int H_kv, int H_idx, int L,
                       int n_idx, int d, float scale, float* lse_out, sa_stream_t stream) {
  if (!Q || !K || !V || !idx || !O)
    return set_error(SA_ERR_INVALID_ARG, "Q, K, V, idx and O must be non-NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return set_error(SA_ERR_INVALID_ARG, "Q, K, V and O must be 16-byte aligned");
  if (S < 0 || H <= 0 || H_kv <= 0 || L <= 0 || n_idx < 0)
    return set_error(SA_ERR_INVALID_ARG, "bad shape (S=%d H=%d H_kv=%d L=%d n_idx=%d)", S, H, H_kv,
                     L, n_idx);
  if (H % H_kv != 0) return set_error(SA_ERR_INVALID_ARG, "H = %d is not a multiple of H_kv = %d", H, H_kv);
  if (H_idx != H && H_idx != H_kv)
    return set_error(SA_ERR_INVALID_ARG, "H_idx = %d must be H (%d) or H_kv (%d)", H_idx, H, H_kv);
  if (d != 64 && d != 128) return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  GatherParams p;
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.idx = idx;
  p.idx_len = idx_len;
  p.O = static_cast<uint16_t*>(O);
  p.lse = lse_out;
  p.S = S;
  p.H = H;
  p.Hkv = H_kv;
  p.H_idx = H_idx;
  p.L = L;
  p.n_idx = n_idx;
  p.positions = nullptr;
  p.window = p.n_global = 0;
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf(float(d));
  p.scale_log2 = sc * 1.4426950408889634f;
  p.err = device_error_word();
  if (!p.err) return set_error(SA_ERR_CUDA, "device error word unavailable");
  return launch_gather(p, d, reinterpret_cast<cudaStream_t>(stream));
}

int sparse_attn_decode_window(const void* Q, const void* K, const void* V,
                              const int32_t* positions, void* O, int S, int H, int H_kv, int d,
                              const sa_pattern_t* pat, float* lse_out, sa_stream_t stream) {
  if (!Q || !K || !V || !positions || !O || !pat)
    return set_error(SA_ERR_INVALID_ARG, "Q, K, V, positions, O and pat must be non-NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return set_error(SA_ERR_INVALID_ARG, "Q, K, V and O must be 16-byte aligned");
  if (S < 0 || H <= 0 || H_kv <= 0)
    return set_error(SA_ERR_INVALID_ARG, "bad shape (S=%d H=%d H_kv=%d)", S, H, H_kv);
  if (H % H_kv != 0) return set_error(SA_ERR_INVALID_ARG, "H = %d is not a multiple of H_kv = %d", H, H_kv);
  if (d != 64 && d != 128) return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  if (!pat->causal || pat->window < 1 || pat->n_global < 0)
    return set_error(SA_ERR_UNSUPPORTED,
                     "window decode needs a causal pattern with window >= 1 and n_global >= 0");
  if (pat->block_local > 0 || (pat->n_random > 0 && pat->random_table) || pat->thresholds ||
      pat->dilation > 1)
    return set_error(SA_ERR_UNSUPPORTED,
                     "window decode covers the window and global tokens only (no block_local, "
                     "random blocks, dilation or thresholds)");
  const int64_t C = int64_t(pat->window) + pat->n_global;
  if (C > INT32_MAX) return set_error(SA_ERR_UNSUPPORTED, "cache of %lld slots too large", (long long)C);
  GatherParams p;
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.idx = nullptr;
  p.idx_len = nullptr;
  p.O = static_cast<uint16_t*>(O);
  p.lse = lse_out;
  p.S = S;
  p.H = H;
  p.Hkv = H_kv;
  p.H_idx = H;
  p.L = int(C);
  p.n_idx = 0;
  p.positions = positions;
  p.window = pat->window;
  p.n_global = pat->n_global;
  const float sc = pat->scale != 0.f ? pat->scale : 1.0f / sqrtf(float(d));
  p.scale_log2 = sc * 1.4426950408889634f;
  p.err = device_error_word();
  if (!p.err) return set_error(SA_ERR_CUDA, "device error word unavailable");
  return launch_gather(p, d, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
// Workspace of the top-k decode: scores [S*H][Lp] fp32, first-level
// histograms [S*H][kTopkBins1], selected keys [S*H][top_k], counts [S*H] and
// the selected keys' scores [S*H][top_k] fp32; each region starts on a
// 256-byte boundary.
struct TopkLayout {
  size_t scores = 0, hist = 0, idx = 0, idx_len = 0, sel = 0, total = 0;
};
size_t round_up256(size_t n) { return (n + 255) & ~size_t(255); }
bool topk_layout(int S, int H, int L, int top_k, TopkLayout* t) {
  if (S < 0 || H <= 0 || L <= 0 || top_k <= 0) return false;
  const size_t sh = size_t(S) * size_t(H);
  const size_t Lp = (size_t(L) + 3) & ~size_t(3);
  t->scores = 0;
  t->hist = round_up256(sh * Lp * 4);
  t->idx = t->hist + round_up256(sh * kTopkBins1 * 4);
  t->idx_len = t->idx + round_up256(sh * size_t(top_k) * 4);
  t->sel = t->idx_len + round_up256(sh * 4);
  t->total = t->sel + round_up256(sh * size_t(top_k) * 4);
  return true;
}
}  // namespace

extern "C" {

size_t sparse_attn_decode_topk_workspace(int S, int H, int L, int top_k) {
  TopkLayout t;
  return topk_layout(S, H, L, top_k, &t) ? t.total : 0;
}

int sparse_attn_decode_topk(const void* Q, const void* K, const void* V, const int32_t* lengths,
                            void* O, int S, int H, int H_kv, int L, int d, int top_k, float scale,
                            int32_t* idx_out, int32_t* idx_len_out, float* lse_out,
                            void* workspace, size_t workspace_bytes, sa_stream_t stream) {
  if (!Q || !K || !V || !O || !workspace)
    return set_error(SA_ERR_INVALID_ARG, "Q, K, V, O and workspace must be non-NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(workspace))
    return set_error(SA_ERR_INVALID_ARG, "Q, K, V, O and workspace must be 16-byte aligned");
  if (S < 0 || H <= 0 || H_kv <= 0 || L <= 0)
    return set_error(SA_ERR_INVALID_ARG, "bad shape (S=%d H=%d H_kv=%d L=%d)", S, H, H_kv, L);
  if (H % H_kv != 0) return set_error(SA_ERR_INVALID_ARG, "H = %d is not a multiple of H_kv = %d", H, H_kv);
  if (top_k < 1) return set_error(SA_ERR_INVALID_ARG, "top_k = %d (must be >= 1)", top_k);
  if (d != 64 && d != 128) return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  // grids: (S*H) CTAs in x for the select and attention passes; the score pass
  // puts its 8192-key chunks in y (at most 65535 of them)
  if (int64_t(S) * H > INT32_MAX || int64_t(L) > int64_t(65535) * kTopkChunk)
    return set_error(SA_ERR_UNSUPPORTED, "S*H or L too large for the launch grids");
  TopkLayout t;
  topk_layout(S, H, L, top_k, &t);
  if (workspace_bytes < t.total)
    return set_error(SA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes,
                     t.total);
  if (S == 0) return SA_OK;
  unsigned char* w = static_cast<unsigned char*>(workspace);
  TopkParams p;
  std::memset(&p, 0, sizeof p);
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.lengths = lengths;
  p.O = static_cast<uint16_t*>(O);
  p.lse = lse_out;
  p.scores = reinterpret_cast<float*>(w + t.scores);
  p.hist = reinterpret_cast<uint32_t*>(w + t.hist);
  p.idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + t.idx);
  p.idx_len = idx_len_out ? idx_len_out : reinterpret_cast<int32_t*>(w + t.idx_len);
  p.sel_scores = reinterpret_cast<float*>(w + t.sel);
  p.S = S;
  p.H = H;
  p.Hkv = H_kv;
  p.L = L;
  p.Lp = (L + 3) & ~3;
  p.top_k = top_k;
  p.chunk = kTopkChunk;
  const float sc = scale != 0.f ? scale : 1.0f / sqrtf(float(d));
  p.scale_log2 = sc * 1.4426950408889634f;
  p.err = device_error_word();
  if (!p.err) return set_error(SA_ERR_CUDA, "device error word unavailable");
  return launch_topk(p, d, reinterpret_cast<cudaStream_t>(stream));
}

int64_t sparse_attn_window_slot(int64_t j, int window, int n_global) {
  if (j < 0 || window < 1 || n_global < 0) return -1;
  return j < n_global ? j : n_global + (j % window);
}

int sparse_attn_check_device_error(sa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_error(e, "cudaStreamSynchronize");
  int* w = device_error_word();
  if (!w) return set_error(SA_ERR_CUDA, "device error word unavailable");
  int v = 0;
  e = cudaMemcpy(&v, w, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_error(e, "cudaMemcpy");
  if (v == 0) return SA_OK;
  e = cudaMemset(w, 0, sizeof v);
  if (e != cudaSuccess) return cuda_error(e, "cudaMemset");
  const int code = v & 0xFF, where = v >> 8;
  if (code == SA_ERR_TIMEOUT)
    return set_error(SA_ERR_TIMEOUT, "a kernel pipeline wait ran out of time (site %d)", where);
  if (code == SA_ERR_DEVICE_INDEX)
    return set_error(SA_ERR_DEVICE_INDEX, "a gather index was outside [0, L)");
  return set_error(code, "device error %d (site %d)", code, where);
}

}  // extern "C"
