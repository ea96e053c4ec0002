// prefill_sm100.cu -- block-sparse attention prefill for B200 (sm_100a).
//
// Computes out_i = sum_{j in G_i} softmax_G(s_ij) v_j ("Sparse Attention
// Weights Assumption", sparse attention output formula) for every query row,
// where G_i is given by per-(head, 128-row tile) lists of 64-key blocks built
// by the host pattern compiler, optionally pruned by the Block-Sparse-
// FlashAttention rule ("Block Sparse Flash Attention", paper summary and
// improvements): the exact QK^T tile of a block is computed first, its
// maximum scaled logit is compared with the head's calibrated threshold, and
// below it the block's V tile is never loaded and its PV product never issued.
//
// One CTA = 6 warps, persistent, two CTAs per SM (each owns 256 TMEM columns):
//   warp 0      TMA producer: lane 0 loads the Q tile once per work unit and
//               the K blocks into a ring; lane 1 loads the V tiles of kept
//               blocks (when the rule is on, after deciding from the softmax
//               warps' four maxima of the block).
//   warp 1      TMEM owner and single-thread tcgen05 issuer: S = Q K^T into
//               TMEM, O += P V with P read from TMEM, as an event loop that
//               issues whichever step is ready.
//   warps 2..5  softmax warpgroup, one query row per thread (TMEM lane):
//               mask of partial blocks, row max, the warp's maximum published
//               for the gate (a warp waits for the other three only when its
//               own does not keep the block), online softmax statistics
//               (m, l) in fp32, P (bf16) written to TMEM, lazy rescale of O,
//               epilogue O / l.
// Work units (b, h, tile) -- or pieces of a split tile's block list, whose
// partial results the CTA finishing the last piece merges -- come from a
// launch-wide queue: the host orders them
// (very long units first; then tile-major when all of K/V fits in L2, else
// K/V-group-major so a K/V head's blocks stay in L2 while its query heads use
// them) and each CTA's producer claims the next one with an atomic counter
// when it has room, so CTAs that get cheap units take more of them.
//
// TMEM columns: NS S buffers of 64 columns at [0, 64 NS) (NS = 2 at d = 128,
// 3 at d = 64, where O is half as wide), O at [64 NS, 64 NS + d).  Block k
// uses S buffer k % NS; its P (bf16 pairs) is written over the first 32
// columns of that buffer once the logits are in registers, and the PV of block
// k reads it there.  The QK^T of the next NS - 1 blocks runs while the softmax
// works on block k, also when block k is skipped by the rule, so a run of
// skipped blocks costs the softmax's statistic alone per block.
#include <cuda_bf16.h>

#include <cmath>

#include "common.h"
#include "ptx.cuh"
#include "softmax_util.cuh"

namespace sa {
namespace {

constexpr int kThreads = 192;
constexpr int kTmemCols = 256;
constexpr int kTmemS = 0;     // S buffers of 64 fp32 columns, at kTmemS + 64 b
constexpr uint32_t kSoftmaxBar = 1;    // named barrier of the softmax warpgroup
constexpr uint32_t kSoftmaxWarps = 4;
constexpr float kRescaleLog2 = 8.0f;   // lazy rescale: keep a stale max up to 2^8
constexpr uint32_t kUnitRing = 4;       // depth of the work-unit ring
// consumers of a ring slot: the MMA thread, the V loader and one lane of
// each softmax warp
constexpr uint32_t kUnitConsumers = 1 + 1 + 4;
// The block-skip gate: each softmax warp publishes its warp maximum of a
// block in a ring of kRedRing slots (an mbarrier per slot counts the four
// warps); the V loader reads the four and decides, and frees the slot.
constexpr uint32_t kRedRing = 8;
// PV completions are tracked on a ring of kODone barriers (PV number n on
// barrier n % kODone, phase n / kODone).  A softmax warp waits on PV number L
// only after the S of its current block has landed, and S(k) is issued after
// block k - NS is handled, so every PV older than L - NS + 1 is complete: the
// parity wait on L's barrier cannot mistake an older phase for L's while
// kODone >= NS + 1.
constexpr uint32_t kODone = 4;

// where-codes recorded with SA_ERR_TIMEOUT
enum { W_PROD_Q = 1, W_PROD_K, W_MMA_Q, W_MMA_SFREE, W_MMA_K, W_MMA_VEMPTY, W_MMA_DEC,
       W_MMA_P, W_MMA_VFULL, W_SM_S, W_SM_O, W_SM_EPI, W_PROD_UNIT, W_MMA_UNIT, W_SM_UNIT,
       W_SM_P, W_VL_UNIT, W_VL_DEC, W_VL_EMPTY, W_MMA_LOOP, W_SM_DEC };

template <int D>
struct Cfg {
  static constexpr int KS = D == 128 ? 2 : 3;   // K ring depth
  static constexpr int VS = D == 128 ? 2 : 3;   // V ring depth
  static constexpr int CH = D / 64;             // 64-column (128-byte) chunks per row
  static constexpr int NS = D == 128 ? 2 : 3;   // S buffers in TMEM
  // d = 64 (BigBird-style patterns): warps whose rows see no key of a random
  // block skip it; at d = 128 the plain loop is kept (measured faster there)
  static constexpr bool kSkipInvisible = D == 64;
  static_assert(kODone >= NS + 1, "PV-completion ring too shallow for NS S buffers");
  static constexpr int TMEM_O = kTmemS + 64 * NS;   // O accumulator: d fp32 columns
  static_assert(TMEM_O + D <= kTmemCols, "TMEM budget");
  static constexpr int Q_BYTES = kTileQ * D * 2;
  static constexpr int KV_BYTES = kTileK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VS * KV_BYTES;
  static constexpr int BAR_BYTES = 1024;
  // At least 80 KB so that no third CTA fits on an SM: two CTAs use all 512
  // TMEM columns, a third would block in tcgen05.alloc.
  static constexpr int SMEM_USED = OFF_BAR + BAR_BYTES;
  static constexpr int SMEM = (SMEM_USED > 80 * 1024 ? SMEM_USED : 80 * 1024) + 1024;
};

struct Unit {
  int b, r, h, hkv, t, beg, n;   // r: residue class of a dilated window (0 otherwise)
  int slot;                      // piece of a split tile: its workspace slot; -1 otherwise
  int split, first_slot, n_pieces;   // piece: its split tile and that tile's slots
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[3], v_empty[3];
  uint64_t s_full[3];                   // per S buffer: S of the block written
  uint64_t p_ready[3];                  // per S buffer: P written (or block skipped)
  uint64_t red_full[kRedRing], red_empty[kRedRing];   // warp maxima: softmax -> V loader
  uint64_t o_done[4];
  uint64_t drain;
  uint64_t u_full[4], u_empty[4];   // work-unit ring (producer -> MMA + softmax)
  uint32_t tmem_base;
  int abort;
  uint32_t flags[3];   // per S buffer: 1 = block kept, 0 = skipped
  float red[kRedRing][4];   // per ring slot: the four warp maxima of a block
  Unit unit_slot[4];   // decoded work unit; n = -1 once the queue is exhausted
  int merge_last;      // the piece just finished was its split tile's last
};
static_assert(sizeof(Bars) <= 1024, "barrier block too large");


template <bool SPLIT>
__device__ __forceinline__ Unit get_unit(const PrefillParams& p, int ui) {
  Unit u;
  int id = __ldg(p.units + ui), k0 = 0, n = -1;
  u.slot = u.split = u.first_slot = u.n_pieces = -1;
  if (SPLIT && id < 0) {   // a piece of a split tile
    const int4 pc = __ldg(p.pieces + 2 * ~id);
    const int4 st = __ldg(p.pieces + 2 * ~id + 1);
    id = pc.x;
    k0 = pc.y;
    n = pc.z;
    u.slot = pc.w;
    u.split = st.x;
    u.first_slot = st.y;
    u.n_pieces = st.z;
  }
  u.t = id % p.T;
  const int bh = id / p.T;
  u.h = bh % p.H;
  const int bd = bh / p.H;   // b*dil + r
  u.b = bd / p.dil;
  u.r = bd - u.b * p.dil;
  u.hkv = u.h / (p.H / p.Hkv);
  const int row = (p.head_pat ? u.h : 0) * p.T + u.t;
  u.beg = __ldg(p.row_ptr + row) + k0;
  u.n = n >= 0 ? n : __ldg(p.row_ptr + row + 1) - u.beg;
  return u;
}

// Work queue.  The producer thread claims unit indices from the launch-wide
// counter p.sched[0] (atomicAdd, longest-first order), decodes each unit and
// publishes it in a shared-memory ring; the MMA thread, the V loader and the
// softmax warps take the decoded units from the ring in the same order (so
// they need no dependent global loads at unit boundaries).  n = -1 marks the
// end of the queue.
template <bool SPLIT>
__device__ __forceinline__ bool publish_unit(const PrefillParams& p, Bars* bars, uint32_t n,
                                             Unit* out) {
  const uint32_t slot = n % kUnitRing;
  if (!wait_bounded(smem_u32(&bars->u_empty[slot]), ((n / kUnitRing) & 1) ^ 1, &bars->abort,
                    p.err, W_PROD_UNIT))
    return false;
  const int v = atomicAdd(p.sched, 1);
  Unit u;
  if (v < p.n_units) {
    u = get_unit<SPLIT>(p, v);
  } else {
    u.b = u.r = u.h = u.hkv = u.t = u.beg = 0;
    u.n = -1;
    u.slot = u.split = u.first_slot = u.n_pieces = -1;
  }
  volatile int* d = reinterpret_cast<volatile int*>(&bars->unit_slot[slot]);
  d[0] = u.b; d[1] = u.h; d[2] = u.hkv; d[3] = u.t; d[4] = u.beg; d[5] = u.n; d[6] = u.r;
  if (SPLIT) { d[7] = u.slot; d[8] = u.split; d[9] = u.first_slot; d[10] = u.n_pieces; }
  mbar_arrive(smem_u32(&bars->u_full[slot]));
  *out = u;
  return true;
}

// Consumer side: one thread (MMA, V loader) or every lane of a softmax warp
// calls it; the slot is released once per caller group (the warp's lane 0
// after the whole warp has read it).
template <bool SPLIT>
__device__ __forceinline__ bool take_unit(const PrefillParams& p, Bars* bars, uint32_t n, Unit* out,
                                          int where, bool whole_warp) {
  const uint32_t slot = n % kUnitRing;
  if (!wait_bounded(smem_u32(&bars->u_full[slot]), (n / kUnitRing) & 1, &bars->abort, p.err,
                    where))
    return false;
  const volatile int* d = reinterpret_cast<const volatile int*>(&bars->unit_slot[slot]);
  out->b = d[0]; out->h = d[1]; out->hkv = d[2]; out->t = d[3]; out->beg = d[4]; out->n = d[5];
  out->r = d[6];
  if (SPLIT) {
    out->slot = d[7];
    out->split = d[8];
    out->first_slot = d[9];
    out->n_pieces = d[10];
  } else {
    out->slot = out->split = out->first_slot = out->n_pieces = -1;
  }
  if (whole_warp) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&bars->u_empty[slot]));
  } else {
    mbar_arrive(smem_u32(&bars->u_empty[slot]));
  }
  return true;
}

// ------------------------------------------------------------ producer --
template <int D, bool SPLIT>
__device__ void producer_role(const PrefillParams& p, uint8_t* smem, Bars* bars) {
  using C = Cfg<D>;
  volatile int* abort_flag = &bars->abort;
  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sK = smem_u32(smem + C::OFF_K);
  uint32_t qc = 0, kc = 0;
  for (uint32_t n = 0;; ++n) {
    Unit u;
    if (!publish_unit<SPLIT>(p, bars, n, &u)) goto drain;
    if (u.n < 0) break;
    if (u.n == 0) continue;
    if (!wait_bounded(smem_u32(&bars->q_empty), (qc & 1) ^ 1, abort_flag, p.err, W_PROD_Q))
      goto drain;
    mbar_expect_tx(smem_u32(&bars->q_full), C::Q_BYTES);
    for (int c = 0; c < C::CH; ++c)
      tma_load_4d(sQ + c * (kTileQ * 128), &p.tm_q, smem_u32(&bars->q_full), c * 64, u.r,
                  u.t * kTileQ, u.b * p.H + u.h);
    ++qc;
    for (int k = 0; k < u.n; ++k) {
      const int kb = __ldg(p.entries + u.beg + k) >> 1;
      const int st = kc % C::KS;
      if (!wait_bounded(smem_u32(&bars->k_empty[st]), ((kc / C::KS) & 1) ^ 1, abort_flag, p.err,
                        W_PROD_K))
        goto drain;
      const uint32_t dst = sK + st * C::KV_BYTES;
      mbar_expect_tx(smem_u32(&bars->k_full[st]), C::KV_BYTES);
      for (int c = 0; c < C::CH; ++c)
        tma_load_4d(dst + c * (kTileK * 128), &p.tm_k, smem_u32(&bars->k_full[st]), c * 64,
                    u.r, kb * kTileK, u.b * p.Hkv + u.hkv);
      ++kc;
    }
  }
  return;
drain:
  // Let the loads already issued land before the CTA's shared memory is released.
  if (qc > 0) wait_drain(smem_u32(&bars->q_full), (qc - 1) & 1);
  for (uint32_t s = 0; s < C::KS && s < kc; ++s) {
    const uint32_t last = kc - 1 - ((kc - 1 - s) % C::KS);
    wait_drain(smem_u32(&bars->k_full[s]), (last / C::KS) & 1);
  }
}

// ------------------------------------------------------------- V loader --
// Producer warp, lane 1: loads the V tile of every kept block, in block order,
// as soon as a V stage is free.  With the rule on it first takes the block's
// decision from its four warp maxima (skipped blocks load nothing).
template <int D, bool SPLIT>
__device__ void vloader_role(const PrefillParams& p, uint8_t* smem, Bars* bars) {
  using C = Cfg<D>;
  volatile int* abort_flag = &bars->abort;
  const uint32_t sV = smem_u32(smem + C::OFF_V);
  uint32_t vc = 0, g = 0;
  for (uint32_t n = 0;; ++n) {
    Unit u;
    if (!take_unit<SPLIT>(p, bars, n, &u, W_VL_UNIT, false)) goto drain;
    if (u.n < 0) break;
    for (int k = 0; k < u.n; ++k, ++g) {
      const int e = __ldg(p.entries + u.beg + k);
      const int kb = e >> 1;
      bool keep = true;
      if (p.gate) {
        // the rule's decision, from the four warp maxima (as the softmax warps take it)
        const uint32_t rs = g % kRedRing;
        if (!wait_bounded(smem_u32(&bars->red_full[rs]), (g / kRedRing) & 1, abort_flag, p.err,
                          W_VL_DEC))
          goto drain;
        const volatile float* r = bars->red[rs];
        const float tmax = fmaxf(fmaxf(r[0], r[1]), fmaxf(r[2], r[3]));
        mbar_arrive(smem_u32(&bars->red_empty[rs]));
        keep = !p.stats_only && ((e & 1) || !(tmax * p.scale < __ldg(p.thresholds + u.h)));
      }
      if (!keep) continue;
      const uint32_t vs = vc % C::VS;
      if (!wait_bounded(smem_u32(&bars->v_empty[vs]), ((vc / C::VS) & 1) ^ 1, abort_flag, p.err,
                        W_VL_EMPTY))
        goto drain;
      const uint32_t dst = sV + vs * C::KV_BYTES;
      mbar_expect_tx(smem_u32(&bars->v_full[vs]), C::KV_BYTES);
      for (int c = 0; c < C::CH; ++c)
        tma_load_4d(dst + c * (kTileK * 128), &p.tm_v, smem_u32(&bars->v_full[vs]), c * 64,
                    u.r, kb * kTileK, u.b * p.Hkv + u.hkv);
      ++vc;
    }
  }
  return;
drain:
  for (uint32_t s = 0; s < C::VS && s < vc; ++s) {
    const uint32_t last = vc - 1 - ((vc - 1 - s) % C::VS);
    wait_drain(smem_u32(&bars->v_full[s]), (last / C::VS) & 1);
  }
}

// ----------------------------------------------------------- MMA issuer --
// One thread, an event loop per work unit that never blocks on one condition
// while another step is ready.  Steps, each issued in block order:
//   S  : S_k = Q K_k^T into S buffer k % 2 once K_k is in shared memory and
//        block k-2, the buffer's previous user, is done: its hand-off taken
//        and, if kept, its PV issued (the PV reads P_{k-2} from that buffer
//        and is issued first; tcgen05.mma operations of one thread execute
//        in issue order);
//   P  : take block k's P hand-off (kept or skipped) from the softmax;
//   PV : O += P_k V_k for a kept block once V_k has landed.
template <int D, bool SPLIT>
__device__ void mma_role(const PrefillParams& p, uint8_t* smem, Bars* bars, uint32_t tmem) {
  using C = Cfg<D>;
  volatile int* abort_flag = &bars->abort;
  volatile uint32_t* flags = bars->flags;
  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sK = smem_u32(smem + C::OFF_K);
  const uint32_t sV = smem_u32(smem + C::OFF_V);
  constexpr uint32_t idesc_s = make_idesc_bf16(kTileQ, kTileK, 0);
  constexpr uint32_t idesc_o = make_idesc_bf16(kTileQ, D, 1);
  uint32_t qc = 0, kc = 0, g = 0, pvc = 0;
  bool ok = true;

  for (uint32_t n = 0; ok; ++n) {
    Unit u;
    if (!take_unit<SPLIT>(p, bars, n, &u, W_MMA_UNIT, false)) {
      ok = false;
      break;
    }
    if (u.n < 0) break;
    if (u.n == 0) continue;
    if (!wait_bounded(smem_u32(&bars->q_full), qc & 1, abort_flag, p.err, W_MMA_Q)) {
      ok = false;
      break;
    }
    ++qc;
    tc_fence_after();
    const uint32_t g0 = g;
    int ns = 0, nr = 0, npv = 0;   // S issued, P hand-offs taken, PVs handled
    uint32_t keep_bits = 0;        // keep flags of blocks nr-? .. nr-1 (bit = block % 32)
    bool first_pv = true;
    uint64_t t_last = 0;
    uint32_t idle = 0;
    while (npv < u.n) {
      bool progress = false;
      // S for block ns (its buffer's previous block, ns - NS, handled).
      if (ns < u.n && ns <= npv + C::NS - 1) {
        const uint32_t st = kc % C::KS;
        if (mbar_try_wait(smem_u32(&bars->k_full[st]), (kc / C::KS) & 1)) {
          const uint32_t sb = (g0 + ns) % C::NS;
          const uint32_t kbase = sK + st * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t da = make_sdesc(sQ + (kk >> 2) * (kTileQ * 128) + off, 16, 1024);
            const uint64_t db = make_sdesc(kbase + (kk >> 2) * (kTileK * 128) + off, 16, 1024);
            umma_ss(tmem + kTmemS + 64 * sb, da, db, idesc_s, kk > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&bars->k_empty[st]));
          tc_commit(smem_u32(&bars->s_full[sb]));
          if (ns == u.n - 1) tc_commit(smem_u32(&bars->q_empty));
          ++kc;
          ++g;
          ++ns;
          progress = true;
        }
      }
      // P hand-off of block nr.
      if (nr < ns) {
        const uint32_t gk = g0 + nr, fb = gk % C::NS;
        if (mbar_try_wait(smem_u32(&bars->p_ready[fb]), (gk / C::NS) & 1)) {
          tc_fence_after();
          if (flags[fb]) keep_bits |= 1u << (nr & 31);
          else keep_bits &= ~(1u << (nr & 31));
          ++nr;
          progress = true;
        }
      }
      // PV of block npv.
      if (npv < nr) {
        if (!((keep_bits >> (npv & 31)) & 1u)) {
          ++npv;
          progress = true;
        } else {
          const uint32_t vs = pvc % C::VS;
          if (mbar_try_wait(smem_u32(&bars->v_full[vs]), (pvc / C::VS) & 1)) {
            tc_fence_after();
            const uint32_t vbase = sV + vs * C::KV_BYTES;
            const uint32_t pcol = kTmemS + 64 * ((g0 + npv) % C::NS);   // P over block npv's S
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
              const uint64_t db = make_sdesc(vbase + kk * (16 * 128), kTileK * 128, 1024);
              umma_ts(tmem + C::TMEM_O, tmem + pcol + kk * 8, db, idesc_o,
                      (first_pv && kk == 0) ? 0u : 1u);
            }
            tc_commit(smem_u32(&bars->v_empty[vs]));
            tc_commit(smem_u32(&bars->o_done[pvc % kODone]));
            ++pvc;
            ++npv;
            first_pv = false;
            progress = true;
          }
        }
      }
      if (progress) {
        idle = 0;
      } else if ((++idle & 255u) == 0) {
        // Bounded: no step became ready for the whole wait budget -> abort.
        if (*abort_flag) {
          ok = false;
          break;
        }
        const uint64_t now = globaltimer_ns();
        if (idle == 256) t_last = now;
        else if (now - t_last > kWaitBudgetNs) {
          record_device_error(p.err, SA_ERR_TIMEOUT, W_MMA_LOOP);
          *abort_flag = 1;
          ok = false;
          break;
        }
      }
    }
  }
  if (!ok) {
    // Let every MMA already issued finish before TMEM and shared memory go away.
    tc_commit(smem_u32(&bars->drain));
    wait_drain(smem_u32(&bars->drain), 0);
  }
}

// Merge of a split tile's pieces for one row: the pieces' partial results
// (O in the piece's scale m_j, row sum l_j; read past L1, they were written by
// other CTAs) are brought to the largest m_j and summed; O / L -> bf16 and the
// log-sum-exp as in the epilogue.  Pieces whose row saw no key (l_j = 0) are
// left out.
template <int D>
__device__ __forceinline__ void merge_pieces(const PrefillParams& p, int first_slot, int n_pieces, int row,
                             uint16_t* orow_ptr, float* lse_ptr) {
  if (!orow_ptr) return;
  const int64_t stride = int64_t(D + 2) * kTileQ;
  const float* base = p.part + int64_t(first_slot) * stride + row;
  // Loads are unconditional (a piece's O is finite, zero where its row saw no
  // key) so that those of several pieces are in flight together.
  float M = -INFINITY, L = 0.f;
#pragma unroll 4
  for (int j = 0; j < n_pieces; ++j) {
    const float* pj = base + j * stride;
    const float mj = __ldcg(pj + D * kTileQ), lj = __ldcg(pj + (D + 1) * kTileQ);
    if (lj > 0.f) {   // online merge of (M, L) with (m_j, l_j)
      const float mn = fmaxf(M, mj);
      L = L * ex2(M - mn) + lj * ex2(mj - mn);
      M = mn;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    float acc[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) acc[q] = 0.f;
#pragma unroll 2
    for (int j = 0; j < n_pieces; ++j) {
      const float* pj = base + j * stride;
      const float mj = __ldcg(pj + D * kTileQ), lj = __ldcg(pj + (D + 1) * kTileQ);
      float o[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) o[q] = __ldcg(pj + (c0 + q) * kTileQ);
      const float w = lj > 0.f ? ex2(mj - M) : 0.f;
#pragma unroll
      for (int q = 0; q < 32; ++q) acc[q] = fmaf(w, o[q], acc[q]);
    }
    uint4* dst = reinterpret_cast<uint4*>(orow_ptr + c0);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint4 o;
      o.x = pack_bf16x2(acc[8 * v + 0] * inv, acc[8 * v + 1] * inv);
      o.y = pack_bf16x2(acc[8 * v + 2] * inv, acc[8 * v + 3] * inv);
      o.z = pack_bf16x2(acc[8 * v + 4] * inv, acc[8 * v + 5] * inv);
      o.w = pack_bf16x2(acc[8 * v + 6] * inv, acc[8 * v + 7] * inv);
      dst[v] = o;
    }
  }
  if (lse_ptr) *lse_ptr = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

// Epilogue of a piece of a split tile (all four softmax warps): O
// unnormalised (fp32), the row's scale reference m and its sum l go to the
// piece's workspace slot, each column as 128 consecutive floats (one per row);
// a piece with no kept block leaves O = 0.  The CTA that finishes the tile's
// last piece (counted on a device-wide counter after a fence) merges them.
// Kept out of line: it runs once per piece, and inlined it would take
// registers from the block loop.  Returns false on a timed-out wait.
template <int D>
__device__ __noinline__ bool piece_epilogue(const PrefillParams& p, Bars* bars, uint32_t tmem_row,
                                            const Unit& u, uint32_t kept, uint32_t pv_total,
                                            float m, float l, int row, bool leader,
                                            uint16_t* orow_ptr, float* lse_ptr) {
  using C = Cfg<D>;
  float* part = p.part + int64_t(u.slot) * (D + 2) * kTileQ + row;
  if (kept > 0) {
    const uint32_t last = pv_total - 1;
    if (!wait_bounded(smem_u32(&bars->o_done[last % kODone]), (last / kODone) & 1, &bars->abort,
                      p.err, W_SM_EPI))
      return false;
    tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(tmem_row + C::TMEM_O + c * 32, o);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 32; ++q) __stcg(part + (c * 32 + q) * kTileQ, __uint_as_float(o[q]));
    }
    tc_fence_before();
  } else {
    for (int c = 0; c < D; ++c) __stcg(part + c * kTileQ, 0.f);
  }
  __stcg(part + D * kTileQ, m);
  __stcg(part + (D + 1) * kTileQ, l);
  __threadfence();
  named_bar_sync(kSoftmaxBar, 128);
  if (leader)
    reinterpret_cast<volatile int*>(&bars->merge_last)[0] =
        atomicAdd(p.split_cnt + u.split, 1) == u.n_pieces - 1;
  named_bar_sync(kSoftmaxBar, 128);
  if (reinterpret_cast<volatile int*>(&bars->merge_last)[0]) {
    __threadfence();
    merge_pieces<D>(p, u.first_slot, u.n_pieces, row, orow_ptr, lse_ptr);
  }
  return true;
}

template <int D, bool SPLIT>
__device__ void softmax_role(const PrefillParams& p, Bars* bars, uint32_t tmem, int warp,
                             int lane) {
  using C = Cfg<D>;
  volatile int* abort_flag = &bars->abort;
  volatile uint32_t* flags = bars->flags;
  const int q4 = warp & 3;              // TMEM lane quadrant of this warp
  const int row = q4 * 32 + lane;       // query row within the tile
  const bool leader = (warp == 2 && lane == 0);
  const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
  uint32_t g = 0, pv_total = 0;

  for (uint32_t n = 0;; ++n) {
    Unit u;
    if (!take_unit<SPLIT>(p, bars, n, &u, W_SM_UNIT, true)) return;
    if (u.n < 0) break;
    const int i = u.t * kTileQ + row;
    const bool row_ok = i < p.N;
    // output row: position i of residue class u.r is row i*dil + r of the slice
    const int64_t orow = (int64_t)(u.b * p.H + u.h) * p.N * p.dil + (int64_t)i * p.dil + u.r;
    const int64_t tile_base = ((int64_t)(u.b * p.H + u.h) * p.T + u.t) * p.n_kb;
    const float tau = (p.gate && !p.stats_only) ? __ldg(p.thresholds + u.h) : 0.f;
    float m = -INFINITY, l = 0.f;
    uint32_t kept = 0;
    // Block entries are read one block ahead so the load overlaps the S wait.
    int e_next = u.n > 0 ? __ldg(p.entries + u.beg) : 0;
    const RowVis rv = row_vis(p, load_row_random(p, u.h, i), i);

    for (int k = 0; k < u.n; ++k) {
      const uint32_t fb = g % C::NS;   // this block's S buffer (and flag / statistic slot)
      const int e = e_next;
      if (k + 1 < u.n) e_next = __ldg(p.entries + u.beg + k + 1);
      const int kb = e >> 1;
      const bool partial = e & 1;
      uint64_t vis = ~0ull;
      if (partial) vis = vis_bits(p, rv, u.h, i, kb);
      // A warp none of whose rows sees a key of this (partial) block -- the
      // other half of the tile of a random block drawn for 64 query rows --
      // neither reads S nor computes exponentials: its rows' P is zero.
      const bool none =
          C::kSkipInvisible && p.n_random > 0 && partial && __all_sync(0xffffffffu, vis == 0ull);
      // This block's slot of the maxima ring, claimed now while S is still
      // being computed (the V loader frees slots as it reads them).
      const uint32_t rs = g % kRedRing;
      if (p.want_stats && p.gate &&
          !wait_bounded(smem_u32(&bars->red_empty[rs]), ((g / kRedRing) & 1) ^ 1, abort_flag,
                        p.err, W_SM_DEC))
        return;
      // S of this block is in S buffer fb; the MMA thread computes the next
      // block's S into the other buffer meanwhile.
      const uint32_t tS = tmem + lane_base + kTmemS + 64 * fb;
      if (!wait_bounded(smem_u32(&bars->s_full[fb]), (g / C::NS) & 1, abort_flag, p.err, W_SM_S))
        return;
      tc_fence_after();
      float x[64];
      float mx = -INFINITY;
      if (!none) {
        uint32_t r0[32], r1[32];
        tmem_ld32(tS, r0);
        tmem_ld32(tS + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = __uint_as_float(r0[c]);
          x[32 + c] = __uint_as_float(r1[c]);
        }
        if (partial && vis != ~0ull) apply_mask(vis, x);
        mx = row_max64(x);
      }

      bool keep = true;
      if (p.want_stats) {
        // The tile maximum is the largest of the four warp maxima: each warp
        // publishes its own; a warp whose own maximum keeps the block (a
        // tile maximum is at least as large) needs nobody else's, the others
        // wait for all four.  No barrier between the warps.
        const float wm = warp_max(mx);
        if (lane == 0) reinterpret_cast<volatile float*>(bars->red[rs])[q4] = wm;
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->red_full[rs]));
        const bool own_keep = p.gate && !p.stats_only && (partial || !(wm * p.scale < tau));
        const bool need_all = (warp == 2 && (p.stat_out || p.mask_out)) || (p.gate && !own_keep);
        float tmax = wm;
        if (need_all) {
          if (!wait_bounded(smem_u32(&bars->red_full[rs]), (g / kRedRing) & 1, abort_flag, p.err,
                            W_SM_P))
            return;
          const volatile float* r = bars->red[rs];
          tmax = fmaxf(fmaxf(r[0], r[1]), fmaxf(r[2], r[3]));
        }
        const float stat = tmax * p.scale;
        if (p.gate) keep = !p.stats_only && (partial || !(stat < tau));
        if (leader) {
          if (p.stat_out) p.stat_out[tile_base + kb] = stat;
          if (p.mask_out) p.mask_out[tile_base + kb] = keep || p.stats_only ? 1 : 2;
        }
        if (p.gate && lane == 0) flags[fb] = keep ? 1u : 0u;   // every warp: the same value
      } else if (leader && p.mask_out) {
        p.mask_out[tile_base + kb] = 1;
      }
      if (!keep) {
        // each warp hands back its rows of the S buffer, already read
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_ready[fb]));
        // Default rule: the block's keys leave G.  Variant: they stay in the
        // denominator -- the max and the row sum below take them, no P is
        // written (the S buffer is already handed back) and no PV runs.
        if (!p.skip_denominator) {
          ++g;
          continue;
        }
      }

      // Row-level reading of the rule: a row whose own maximum over a full
      // block is below the threshold drops the block (P = 0 in its row, no
      // contribution to its max or sum) while the tile keeps it for other rows.
      const bool row_drop = p.row_level && p.gate && keep && !partial && (mx * p.scale < tau);
      // Online softmax in the log2 domain with a lazily updated max.
      const float mx2 = row_drop ? -INFINITY : mx * p.scale_log2;
      const float m_new = fmaxf(m, mx2);
      const bool need = m_new > m + kRescaleLog2 || (m == -INFINITY && m_new != -INFINITY);
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m - m_new);   // m = -inf -> 0
        l *= alpha;
        m = m_new;
      }
      if (kept > 0 && __any_sync(0xffffffffu, need)) {
        // O += P V of the previous kept block must be complete before O is rescaled.
        const uint32_t last = pv_total - 1;
        if (!wait_bounded(smem_u32(&bars->o_done[last % kODone]), (last / kODone) & 1, abort_flag,
                          p.err, W_SM_O))
          return;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          const uint32_t ta = tmem + lane_base + C::TMEM_O + c * 32;
          tmem_ld32(ta, o);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st32(ta, o);
        }
      }
      const float mb = (m == -INFINITY) ? 0.f : m;
      // p = 2^(s*scale*log2e - m): the argument and the row sum in packed
      // f32x2 arithmetic, the exponentials on MUFU (ex2.approx).  Moving part
      // of them to an FMA-pipe polynomial was measured slower: this loop is
      // bound by instruction issue, not by the MUFU pipe.
      const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
      // a dropped row's exponent arguments are all -inf: p = 0
      const uint64_t nmb = row_drop ? f2_pack(-INFINITY, -INFINITY) : f2_pack(-mb, -mb);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[32];
      if (none) {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float a0, a1, p0, p1;
          f2_unpack(f2_fma(f2_pack(x[2 * c], x[2 * c + 1]), sl2, nmb), a0, a1);
          p0 = ex2(a0);
          p1 = ex2(a1);
          acc[c & 3] = f2_add(acc[c & 3], f2_pack(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
        float s0, s1;
        f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), s0, s1);
        l += s0 + s1;
      }
      if (!keep) {   // skipped, kept in the denominator only
        ++g;
        continue;
      }
      // P (bf16 pairs) over the first 32 columns of this block's S buffer,
      // whose logits are in registers.
      tmem_st32(tS, pk);
      tmem_wait_st();
      tc_fence_before();
      // Each warp signals its own 32 rows of P; the MMA warp waits for all four.
      if (leader) flags[fb] = 1u;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_ready[fb]));
      ++kept;
      ++pv_total;
      ++g;
    }

    if (p.stats_only) continue;
    if (SPLIT && u.slot >= 0) {
      if (!piece_epilogue<D>(p, bars, tmem + lane_base, u, kept, pv_total, m, l, row, leader,
                             row_ok ? p.O + orow * D : nullptr,
                             row_ok && p.lse ? p.lse + orow : nullptr))
        return;
      continue;
    }
    // Epilogue: O / l -> bf16, one row per thread.
    uint16_t* orow_ptr = p.O + orow * D;
    if (kept > 0) {
      const uint32_t last = pv_total - 1;
      if (!wait_bounded(smem_u32(&bars->o_done[last % kODone]), (last / kODone) & 1, abort_flag,
                        p.err, W_SM_EPI))
        return;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + C::TMEM_O + c * 32, o);
        tmem_wait_ld();
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow_ptr + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
            dst[v] = w;
          }
        }
      }
      tc_fence_before();
    } else if (row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(orow_ptr);
      for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0, 0, 0, 0);
    }
    if (row_ok && p.lse)
      p.lse[orow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
}

template <int D, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 2) prefill_kernel(const __grid_constant__ PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + Cfg<D>::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(smem_u32(&bars->k_full[s]), 1);
      mbar_init(smem_u32(&bars->k_empty[s]), 1);
      mbar_init(smem_u32(&bars->v_full[s]), 1);
      mbar_init(smem_u32(&bars->v_empty[s]), 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(smem_u32(&bars->s_full[b]), 1);
      mbar_init(smem_u32(&bars->p_ready[b]), kSoftmaxWarps);
    }
    for (uint32_t b = 0; b < kODone; ++b) mbar_init(smem_u32(&bars->o_done[b]), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    for (uint32_t r = 0; r < kRedRing; ++r) {
      mbar_init(smem_u32(&bars->red_full[r]), kSoftmaxWarps);
      mbar_init(smem_u32(&bars->red_empty[r]), 1);
    }
    for (uint32_t r = 0; r < kUnitRing; ++r) {
      mbar_init(smem_u32(&bars->u_full[r]), 1);
      mbar_init(smem_u32(&bars->u_empty[r]), kUnitConsumers);
    }
    bars->abort = 0;
    bars->flags[0] = bars->flags[1] = bars->flags[2] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) producer_role<D, SPLIT>(p, smem, bars);
    else if (lane == 1) vloader_role<D, SPLIT>(p, smem, bars);
  } else if (warp == 1) {
    if (lane == 0) mma_role<D, SPLIT>(p, smem, bars, tmem);
  } else {
    softmax_role<D, SPLIT>(p, bars, tmem, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  // The last CTA to finish resets the work-queue counters for the next launch
  // (every CTA has claimed past the end of the queue before it gets here).
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sched + 1, 1) == int(gridDim.x) - 1) {
      atomicExch(p.sched, 0);
      atomicExch(p.sched + 1, 0);
      if (SPLIT)
        for (int k = 0; k < p.n_split; ++k) atomicExch(p.split_cnt + k, 0);
    }
  }
}

int g_num_sms[64] = {0};
bool g_attr_set[2][2][64] = {};

}  // namespace

int launch_prefill(const PrefillParams& p, int d, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return set_error(SA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  if (g_num_sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_error(e, "cudaDeviceGetAttribute");
  }
  if (p.n_units == 0) return SA_OK;
  const int grid = p.n_units < 2 * g_num_sms[dev] ? p.n_units : 2 * g_num_sms[dev];
  if (d != 128 && d != 64)
    return set_error(SA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  // Plans without split tiles run the instantiation that has no piece code.
  const bool split = p.n_split > 0;
  bool& attr = g_attr_set[d == 128][split][dev];
  const int smem = d == 128 ? Cfg<128>::SMEM : Cfg<64>::SMEM;
  auto* kern = d == 128 ? (split ? prefill_kernel<128, true> : prefill_kernel<128, false>)
                        : (split ? prefill_kernel<64, true> : prefill_kernel<64, false>);
  if (!attr) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute");
    attr = true;
  }
  kern<<<grid, kThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "prefill launch");
  return SA_OK;
}

}  // namespace sa
