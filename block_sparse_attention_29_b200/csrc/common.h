// common.h -- internal declarations shared by the library's translation units:
// error reporting (host message + device error word), kernel parameter blocks
// and launcher prototypes.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <vector>

#include "../../include/sparse_attn.h"

namespace sa {

// ---------------------------------------------------------------- errors --
// Host: set the thread-local message returned by sparse_attn_last_error().
int set_error(int code, const char* fmt, ...);
int cuda_error(cudaError_t e, const char* what);

// Device error word (one per device, owned by the API translation unit and
// passed to every kernel): 0 = none; otherwise (where << 8) | code of the
// first error recorded since the last sparse_attn_check_device_error().
int* device_error_word();   // host: address for the current device, or null

__device__ __forceinline__ void record_device_error(int* err, int code, int where) {
  atomicCAS(err, 0, (where << 8) | code);
}

// ---------------------------------------------------------------- prefill --
constexpr int kTileQ = 128;   // query rows per tile (UMMA M)
constexpr int kTileK = 64;    // keys per block (UMMA N of Q K^T)

// Block-list entry: (kb << 1) | partial.
__host__ __device__ inline int32_t entry_pack(int32_t kb, bool partial) {
  return (kb << 1) | (partial ? 1 : 0);
}

struct PrefillParams {
  CUtensorMap tm_q;   // 4-D {d, dil, N/dil, B*H}    box {64, 1, 128, 1}, 128-B swizzle
  CUtensorMap tm_k;   // 4-D {d, dil, N/dil, B*H_kv} box {64, 1, 64, 1},  128-B swizzle
  CUtensorMap tm_v;   // same as tm_k over V
  uint16_t* O;        // [B][H][N][d] bf16
  float* lse;         // [B][H][N] or null
  uint8_t* mask_out;  // [B][H][T][n_kb] or null
  float* stat_out;    // [B][H][T][n_kb] or null
  const int32_t* row_ptr;   // [H_pat*T + 1]
  const int32_t* entries;   // block lists
  const int32_t* units;     // work order: unit = (b'*H + h)*T + t with
                            // b' = b*dil + residue class (b' = b without dilation);
                            // a negative entry u is the piece ~u of a split tile
  const int4* pieces;       // split-tile pieces, two int4 each: {id, k0, n, slot},
                            // {split tile, its first slot, its pieces, 0}; or null
  float* part;              // piece workspace [slot][d + 2][128] or null
  int* split_cnt;           // [n_split] pieces finished per split tile; zero between
                            // launches (the last CTA of a launch resets them)
  int n_split;              // split tiles
  int* sched;               // [2] work-queue counters (next unit, CTAs done); zero
                            // between launches (the last CTA of a launch resets them)
  const int32_t* rtab;      // random table [H][n_rb][n_random] or null
  const float* thresholds;  // [H] or null
  int n_units;
  int B, H, Hkv, N, T, n_kb, head_pat;   // head_pat: 1 when lists are per head;
                                         // N: positions per residue class (N/dil)
  int dil;         // dilation: query/key position m of class r is row m*dil + r
  int causal, window, n_global, block_local, random_block, n_random;
  int gate;        // 1: statistics + decision per block (rule or stats pass)
  int stats_only;  // 1: no PV, no output (statistics pass)
  int skip_denominator;  // 1: a skipped block's exp terms still enter m and l
  int row_level;   // 1: rows also drop full blocks whose own maximum is below the threshold
  int want_stats;  // 1: block statistics needed (stat_out or gate)
  float scale;       // logit scale
  float scale_log2;  // scale * log2(e)
  int* err;          // device error word
};

int launch_prefill(const PrefillParams& p, int d, cudaStream_t stream);

// 4-D bf16 TMA map over a [BH][N][d] tensor seen as [BH][N/dil][dil][d]:
// coordinates (x, r, m, slice) address row m*dil + r; box {64, 1, rows, 1},
// 128-byte swizzle; positions m past N/dil read as zero.  N % dil == 0.
int make_tmap(CUtensorMap* m, const void* base, int d, int N, int BH, int rows, int dil);

// ----------------------------------------------------------------- gather --
struct GatherParams {
  const uint16_t* Q;   // [S][H][d]
  const uint16_t* K;   // [S][H_kv][L][d]
  const uint16_t* V;
  const int32_t* idx;  // [S][H_idx][n_idx]
  const int32_t* idx_len;  // [S][H_idx] or null
  uint16_t* O;         // [S][H][d]
  float* lse;          // [S][H] or null
  int S, H, Hkv, H_idx, L, n_idx;
  // Window decode (positions != null): the index set of sequence s is
  // [0, min(n_global, p+1)) u [max(n_global, p-window+1), p], p = positions[s],
  // key j in cache slot j (j < n_global) or n_global + (j mod window).
  const int32_t* positions;
  int window, n_global;
  float scale_log2;
  int* err;            // device error word
};

int launch_gather(const GatherParams& p, int d, cudaStream_t stream);

// ------------------------------------------------------------------ top-k --
constexpr int kTopkBins1 = 2048;   // first-level histogram: the top 11 bits of a score's key
constexpr int kTopkChunk = 8192;   // keys per CTA of the score pass

struct TopkParams {
  const uint16_t* Q;         // [S][H][d]
  const uint16_t* K;         // [S][H_kv][L][d]
  const uint16_t* V;
  const int32_t* lengths;    // [S] keys per sequence, or null (all L)
  uint16_t* O;               // [S][H][d]
  float* lse;                // [S][H] or null
  float* scores;             // workspace [S][H][Lp]: log2-scaled scores
  uint32_t* hist;            // workspace [S][H][kTopkBins1]
  int32_t* idx;              // [S][H][top_k] selected keys, ascending
  int32_t* idx_len;          // [S][H] selected count
  float* sel_scores;         // workspace [S][H][top_k]: the selected keys' scores
  int S, H, Hkv, L, Lp, top_k, chunk;   // Lp: L rounded up to a multiple of 4
  float scale_log2;
  int* err;                  // device error word
};

// Score pass, radix select and attention over the selected keys.
int launch_topk(const TopkParams& p, int d, cudaStream_t stream);

// ------------------------------------------------------------ calibration --
// Per-head rank selection over the statistics of full blocks (plan lists).
int launch_calibrate(const float* stat, const int32_t* row_ptr, const int32_t* entries,
                     int head_pat, int B, int H, int T, int n_kb, double q, float* out,
                     cudaStream_t stream);

// ------------------------------------------------------ pattern compiler --
struct CompiledPattern {
  int H_pat = 0, T = 0, n_kb = 0;
  std::vector<int32_t> row_ptr;   // [H_pat*T + 1]
  std::vector<int32_t> kb;        // listed key blocks, ascending per list
  std::vector<uint8_t> full;      // every pair of the block is in G
  std::vector<int64_t> cnt;       // visible pairs per listed block
};
// Returns SA_OK or an error code (message set).
int compile_pattern(const sa_pattern_t* pat, int H, int N, int tile_q, int tile_k,
                    CompiledPattern* out);
// Validates the descriptor fields that do not depend on the kernel.
int validate_pattern(const sa_pattern_t* pat, int H, int N);
// Shapes and the descriptor fields the kernels constrain (head dim, block
// sizes, random-block granularity, grid and index limits); SA_OK or an error.
int check_shapes(const sa_pattern_t* pat, int B, int H, int Hkv, int N, int d);
// A piece of a split tile: blocks [k0, k0 + n) of tile `id`'s list, whose
// unnormalised partial result goes to workspace slot `slot`; the tile is split
// tile `split`, whose n_pieces pieces hold slots [first_slot, first_slot + n_pieces).
struct Piece {
  int32_t id, k0, n, slot;
  int32_t split, first_slot, n_pieces, pad;
};
// A split tile: its pieces hold slots [first_slot, first_slot + n_pieces).
struct SplitTile {
  int32_t id, first_slot, n_pieces, pad;
};
// Work order of a prefill launch.  units[k] >= 0 is a whole tile
// ((b*H + h)*T + t); units[k] < 0 is pieces[~units[k]].
struct UnitOrder {
  std::vector<int32_t> units;
  std::vector<Piece> pieces;
  std::vector<SplitTile> split;
  int64_t n_slots = 0;
};
// Work order of the B*H*T tiles: tiles longer than a CTA's share of the work
// split into pieces (max_unit_blocks: 0 automatic, > 0 the longest list a unit
// may have, < 0 never; slot_bytes: workspace bytes per piece), units longer than half a
// CTA's share first (longest first), the rest tile-major or K/V-group-major
// (see kv_bytes), the query heads of a group adjacent.  kv_bytes: size of K
// plus V; above 64 MiB (half of L2) the order is K/V-group-major, below
// tile-major.  ctas is the number of CTAs that share the queue.
void order_units(const CompiledPattern& cp, int B, int H, int H_kv, int64_t kv_bytes, int ctas,
                 int max_unit_blocks, int64_t slot_bytes, UnitOrder* out);

// Partial-result workspace of one piece: d O columns, then the row maximum
// (log2 domain) and the row sum, each as 128 consecutive floats (one per row).
inline int64_t piece_slot_floats(int d) { return int64_t(d + 2) * kTileQ; }

// Work units of a prefill launch in queue order (two CTAs per SM share the queue).
inline void build_units(const CompiledPattern& cp, int B, int H, int H_kv, int N, int d,
                        int max_unit_blocks, UnitOrder* order) {
  const int64_t kv_bytes = int64_t(B) * H_kv * N * d * 2 * 2;
  order_units(cp, B, H, H_kv, kv_bytes, 296, max_unit_blocks, piece_slot_floats(d) * 4, order);
}

}  // namespace sa
