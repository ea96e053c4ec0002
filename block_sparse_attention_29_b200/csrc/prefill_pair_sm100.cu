// prefill_pair_sm100.cu -- paired-head block-sparse attention prefill for B200
// (sm_100a), head dimension 128.
//
// Computes the same result as the single-head kernel (prefill_sm100.cu): for
// every query row out_i = sum_{j in G_i} softmax_G(s_ij) v_j ("Sparse Attention
// Weights Assumption", sparse attention output formula) over per-(128-row
// tile) lists of 64-key blocks, optionally pruned by the Block-Sparse-
// FlashAttention rule ("Block Sparse Flash Attention", paper summary and
// improvements: a block whose maximum scaled logit is below the head's
// calibrated threshold has its V tile never loaded and its PV never issued).
//
// A work unit is one 128-row query tile of TWO query heads of the same K/V
// head (grouped-query attention), whose block lists are the same; every K and
// V tile is loaded once for both heads.  Key blocks are taken two at a time:
// one QK^T of a pair is a single M=128 x N=128 x K=128 tcgen05 MMA, which runs
// at the full tensor rate (an N=64 MMA chain on one accumulator does not).
// The gate decision stays per 64-key block and per head.
//
// One CTA per SM, 12 warps (three warpgroups), persistent:
//   warp 0      TMA producer of the two Q tiles of a unit and of the K pairs
//               (one 32 KB ring stage per pair).
//   warp 1      TMEM owner (all 512 columns); lane 0 issues the tcgen05 MMAs
//               of head slot 0.
//   warp 2      V loader (one 32 KB stage per pair, one barrier per 64-key
//               half; under the rule a half is loaded when either head keeps
//               its block).
//   warp 3      lane 0 issues the tcgen05 MMAs of head slot 1.
//   warps 4..7  softmax of head slot 0, warps 8..11 softmax of head slot 1:
//               one query row per thread, 128 logits per pair.
// Warpgroup 0 hands registers to the softmax warpgroups (setmaxnreg).
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).  The
// softmax of head x writes P_x (bf16 pairs) of each block over the first half
// of that block's own S columns once it has read them.
//
// Each head slot has its own MMA issuer: S_x(j), PV_x(j), S_x(j+1), ...; the
// two heads proceed independently and share the tensor pipe, so one head's
// softmax overlaps the other head's MMAs.  S_x(j+1) is issued after PV_x(j),
// which reads P_x(j) from the columns S_x(j+1) overwrites: this relies on the
// tcgen05.mma operations of one thread executing in issue order, as the
// Blackwell attention kernels of CUTLASS do.  A tcgen05.commit tracks all
// earlier MMAs of its thread, so when the softmax sees S_x(j) complete, every
// PV_x before it has completed too, and O_x may be rescaled in place.
#include <cuda_bf16.h>

#include <cmath>

#include "common.h"
#include "ptx.cuh"
#include "softmax_util.cuh"

namespace sa {
namespace {

constexpr int kD = 128;
constexpr int kThreads2 = 384;
// Register split (setmaxnreg): the launch gives every thread kRegLaunch
// registers; warpgroup 0 (producer, MMA issuer, V loader) gives some up and
// the two softmax warpgroups take them.  The split uses exactly the launch's
// registers, and the host launches only when ptxas allocated kRegLaunch per
// thread, so no increase can wait for registers that are not there.
constexpr int kRegLaunch = 168;
constexpr int kRegControl = 72;
constexpr int kRegSoftmax = 216;
static_assert(kRegControl * 128 + kRegSoftmax * 256 == kRegLaunch * kThreads2,
              "register split must use exactly the launch's registers");
static_assert((kRegControl + 2 * kRegSoftmax) * 32 <= 16384,
              "one SM sub-partition holds a control warp and two softmax warps");
constexpr uint32_t kTmemCols2 = 512;
constexpr uint32_t kColS = 0;     // S_x at kColS + 128 x
constexpr uint32_t kColO = 256;   // O_x at kColO + 128 x
constexpr uint32_t kUnitRing2 = 4;
// consumers of a unit-ring slot: the two MMA issuers, the V loader and one
// lane of each of the eight softmax warps
constexpr uint32_t kUnitConsumers2 = 2 + 1 + 8;
constexpr uint32_t kDecRing2 = 4;
constexpr float kRescaleLog2b = 8.0f;   // lazy rescale: keep a stale max up to 2^8

constexpr int KS2 = 2;                       // K ring depth (pairs)
constexpr int VS2 = 2;                       // V ring depth (pairs)
constexpr int Q_BYTES = kTileQ * kD * 2;     // one 128-row Q tile: 32 KB
constexpr int HALF_BYTES = kTileK * kD * 2;  // one 64-key block of K or V: 16 KB
constexpr int PAIR_BYTES = 2 * HALF_BYTES;
constexpr int OFF_Q = 0;                     // Q of head slot x at OFF_Q + x * Q_BYTES
constexpr int OFF_K = 2 * Q_BYTES;
constexpr int OFF_V = OFF_K + KS2 * PAIR_BYTES;
constexpr int OFF_BAR = OFF_V + VS2 * PAIR_BYTES;
constexpr int BAR_BYTES = 1024;
constexpr int SMEM2 = OFF_BAR + BAR_BYTES + 1024;
static_assert(SMEM2 <= 227 * 1024, "shared memory budget");

// where-codes recorded with SA_ERR_TIMEOUT (offset so they differ from the
// single-head kernel's)
enum { X_PROD_UNIT = 40, X_PROD_Q, X_PROD_K, X_VL_UNIT, X_VL_EMPTY, X_VL_DEC0, X_VL_DEC1,
       X_MMA_UNIT, X_MMA_Q, X_MMA_K, X_MMA_P, X_MMA_OFREE, X_MMA_V, X_SM_UNIT, X_SM_DEC, X_SM_S,
       X_SM_O };

struct Unit2 {
  int b, hp, hkv, t, beg, n;
};

struct Bars2 {
  uint64_t q_full, q_empty;
  uint64_t k_full[KS2], k_empty[KS2];
  uint64_t v_full[VS2][2], v_empty[VS2];   // one full barrier per 64-key half
  uint64_t s_full[2];                       // per head slot: S_x of the pair written
  uint64_t p_ready[2];                      // per head slot: P_x written or blocks skipped
  uint64_t o_full[2];                       // per head slot: last PV_x of the unit done
  uint64_t o_free[2];                       // per head slot: epilogue has read O_x
  uint64_t dec_full[2][kDecRing2], dec_empty[2][kDecRing2];
  uint64_t u_full[kUnitRing2], u_empty[kUnitRing2];
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
  uint32_t flags[2];                 // per head slot: keep bits of the current pair
  uint32_t dec_val[2][kDecRing2];    // decision ring: keep bits per pair
  float red[2][2][2][4];             // [head slot][pair parity][block of pair][warp]
  Unit2 unit_slot[kUnitRing2];
};
static_assert(sizeof(Bars2) <= BAR_BYTES, "barrier block too large");

__device__ __forceinline__ Unit2 get_unit2(const PrefillParams& p, int ui) {
  Unit2 u;
  const int id = __ldg(p.units + ui);
  const int hpairs = p.H >> 1;
  u.t = id % p.T;
  const int bhp = id / p.T;
  u.hp = bhp % hpairs;
  u.b = bhp / hpairs;
  u.hkv = (2 * u.hp) / (p.H / p.Hkv);
  u.beg = __ldg(p.row_ptr + u.t);
  u.n = __ldg(p.row_ptr + u.t + 1) - u.beg;
  return u;
}

// Work queue: the producer claims unit indices from the launch-wide counter,
// decodes them and publishes them in a shared-memory ring that every other
// role reads in the same order; n = -1 marks the end of the queue.
__device__ __forceinline__ bool publish_unit2(const PrefillParams& p, Bars2* bars, uint32_t n,
                                              Unit2* out) {
  const uint32_t slot = n % kUnitRing2;
  if (!wait_bounded(smem_u32(&bars->u_empty[slot]), ((n / kUnitRing2) & 1) ^ 1, &bars->abort,
                    p.err, X_PROD_UNIT))
    return false;
  const int v = atomicAdd(p.sched, 1);
  Unit2 u;
  if (v < p.n_units) {
    u = get_unit2(p, v);
  } else {
    u.b = u.hp = u.hkv = u.t = u.beg = 0;
    u.n = -1;
  }
  volatile int* d = reinterpret_cast<volatile int*>(&bars->unit_slot[slot]);
  d[0] = u.b; d[1] = u.hp; d[2] = u.hkv; d[3] = u.t; d[4] = u.beg; d[5] = u.n;
  mbar_arrive(smem_u32(&bars->u_full[slot]));
  *out = u;
  return true;
}

__device__ __forceinline__ bool take_unit2(const PrefillParams& p, Bars2* bars, uint32_t n,
                                           Unit2* out, int where, bool whole_warp) {
  const uint32_t slot = n % kUnitRing2;
  if (!wait_bounded(smem_u32(&bars->u_full[slot]), (n / kUnitRing2) & 1, &bars->abort, p.err,
                    where))
    return false;
  const volatile int* d = reinterpret_cast<const volatile int*>(&bars->unit_slot[slot]);
  out->b = d[0]; out->hp = d[1]; out->hkv = d[2]; out->t = d[3]; out->beg = d[4]; out->n = d[5];
  if (whole_warp) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&bars->u_empty[slot]));
  } else {
    mbar_arrive(smem_u32(&bars->u_empty[slot]));
  }
  return true;
}

// ------------------------------------------------------------ producer --
// K pair stage layout (K-major, 128-byte swizzle): 64-column chunk c of the
// head dimension at + c * 16 KB, holding 128 key rows of 128 bytes; the first
// block of the pair fills rows 0..63, the second rows 64..127.
__device__ void producer2(const PrefillParams& p, uint8_t* smem, Bars2* bars) {
  volatile int* abort_flag = &bars->abort;
  const uint32_t sQ = smem_u32(smem + OFF_Q);
  const uint32_t sK = smem_u32(smem + OFF_K);
  uint32_t qc = 0, kc = 0;
  for (uint32_t n = 0;; ++n) {
    Unit2 u;
    if (!publish_unit2(p, bars, n, &u)) goto drain;
    if (u.n < 0) break;
    if (u.n == 0) continue;
    if (!wait_bounded(smem_u32(&bars->q_empty), (qc & 1) ^ 1, abort_flag, p.err, X_PROD_Q))
      goto drain;
    mbar_expect_tx(smem_u32(&bars->q_full), 2 * Q_BYTES);
    for (int x = 0; x < 2; ++x)
      for (int c = 0; c < 2; ++c)
        tma_load_4d(sQ + x * Q_BYTES + c * (kTileQ * 128), &p.tm_q, smem_u32(&bars->q_full),
                    c * 64, 0, u.t * kTileQ, u.b * p.H + 2 * u.hp + x);
    ++qc;
    for (int j = 0; j < u.n; j += 2) {
      const int nb = min(2, u.n - j);
      const int st = kc % KS2;
      if (!wait_bounded(smem_u32(&bars->k_empty[st]), ((kc / KS2) & 1) ^ 1, abort_flag, p.err,
                        X_PROD_K))
        goto drain;
      const uint32_t dst = sK + st * PAIR_BYTES;
      mbar_expect_tx(smem_u32(&bars->k_full[st]), nb * HALF_BYTES);
      for (int hb = 0; hb < nb; ++hb) {
        const int kb = __ldg(p.entries + u.beg + j + hb) >> 1;
        for (int c = 0; c < 2; ++c)
          tma_load_4d(dst + c * (2 * kTileK * 128) + hb * (kTileK * 128), &p.tm_k,
                      smem_u32(&bars->k_full[st]), c * 64, 0, kb * kTileK, u.b * p.Hkv + u.hkv);
      }
      ++kc;
    }
  }
  return;
drain:
  if (qc > 0) wait_drain(smem_u32(&bars->q_full), (qc - 1) & 1);
  for (uint32_t s = 0; s < uint32_t(KS2) && s < kc; ++s) {
    const uint32_t last = kc - 1 - ((kc - 1 - s) % KS2);
    wait_drain(smem_u32(&bars->k_full[s]), (last / KS2) & 1);
  }
}

// ------------------------------------------------------------- V loader --
// V pair stage layout (MN-major, 128-byte swizzle): half hb (block hb of the
// pair) at + hb * 16 KB, inside it chunk c of the head dimension at + c * 8 KB
// (64 key rows of 128 bytes).  Each half has its own full barrier, which
// completes either by the half's TMA bytes or, when no head needs the block,
// by a plain arrival.
__device__ __forceinline__ void load_v_half(const PrefillParams& p, Bars2* bars, uint32_t base,
                                            uint32_t st, int hb, int kb, const Unit2& u) {
  const uint32_t bar = smem_u32(&bars->v_full[st][hb]);
  mbar_expect_tx(bar, HALF_BYTES);
  for (int c = 0; c < 2; ++c)
    tma_load_4d(base + hb * HALF_BYTES + c * (kTileK * 128), &p.tm_v, bar, c * 64, 0, kb * kTileK,
                u.b * p.Hkv + u.hkv);
}

__device__ void vloader2(const PrefillParams& p, uint8_t* smem, Bars2* bars) {
  volatile int* abort_flag = &bars->abort;
  const uint32_t sV = smem_u32(smem + OFF_V);
  uint32_t vc = 0, g = 0;
  uint32_t pending = 0;   // halves of the current pair with loads in flight
  for (uint32_t n = 0;; ++n) {
    Unit2 u;
    if (!take_unit2(p, bars, n, &u, X_VL_UNIT, false)) goto drain;
    if (u.n < 0) break;
    if (p.stats_only) continue;
    for (int j = 0; j < u.n; j += 2, ++g) {
      const int nb = min(2, u.n - j);
      const uint32_t st = vc % VS2;
      if (!wait_bounded(smem_u32(&bars->v_empty[st]), ((vc / VS2) & 1) ^ 1, abort_flag, p.err,
                        X_VL_EMPTY))
        goto drain;
      const uint32_t base = sV + st * PAIR_BYTES;
      uint32_t done = 0;
      uint32_t need = (1u << nb) - 1u;
      if (p.gate) {
        const uint32_t slot = g % kDecRing2, ph = (g / kDecRing2) & 1;
        // Head slot 0 decides first (its S is computed first): its kept
        // blocks start loading before head slot 1 has decided.
        if (!wait_bounded(smem_u32(&bars->dec_full[0][slot]), ph, abort_flag, p.err, X_VL_DEC0))
          goto drain;
        const uint32_t d0 = reinterpret_cast<volatile uint32_t*>(bars->dec_val[0])[slot];
        mbar_arrive(smem_u32(&bars->dec_empty[0][slot]));
        for (int hb = 0; hb < nb; ++hb)
          if ((d0 >> hb) & 1u) {
            load_v_half(p, bars, base, st, hb, __ldg(p.entries + u.beg + j + hb) >> 1, u);
            done |= 1u << hb;
            pending = done;
          }
        if (!wait_bounded(smem_u32(&bars->dec_full[1][slot]), ph, abort_flag, p.err, X_VL_DEC1))
          goto drain;
        const uint32_t d1 = reinterpret_cast<volatile uint32_t*>(bars->dec_val[1])[slot];
        mbar_arrive(smem_u32(&bars->dec_empty[1][slot]));
        need = (d0 | d1) & need;
      }
      for (int hb = 0; hb < 2; ++hb) {
        if ((done >> hb) & 1u) continue;
        if ((need >> hb) & 1u) {
          load_v_half(p, bars, base, st, hb, __ldg(p.entries + u.beg + j + hb) >> 1, u);
          done |= 1u << hb;
          pending = done;
        } else {
          mbar_arrive(smem_u32(&bars->v_full[st][hb]));
        }
      }
      pending = 0;
      ++vc;
    }
  }
  return;
drain:
  // Halves of the interrupted pair whose loads were issued.
  for (int hb = 0; hb < 2; ++hb)
    if ((pending >> hb) & 1u) wait_drain(smem_u32(&bars->v_full[vc % VS2][hb]), (vc / VS2) & 1);
  // Every half of a completed pair got one arrival, so its last phase ends.
  for (uint32_t s = 0; s < uint32_t(VS2) && s < vc; ++s) {
    const uint32_t last = vc - 1 - ((vc - 1 - s) % VS2);
    for (int hb = 0; hb < 2; ++hb) wait_drain(smem_u32(&bars->v_full[s][hb]), (last / VS2) & 1);
  }
}

// ---------------------------------------------------------- MMA issuers --
// Two issuing threads, one per head slot, on different SM sub-partitions.  A
// shared-memory access (a barrier wait included) by a thread that has MMAs
// queued stalls that thread until its queue drains, so one thread alone
// leaves the tensor pipe idle at every wait; with two issuers, one keeps the
// pipe fed while the other waits.  Issuer X handles head slot X only: S_X of
// every pair and O_X += P_X V of its kept blocks, in the order
// S_X(j), PV_X(j), S_X(j+1), ...  The K and V stages and the Q tiles are
// released by both issuers (barrier counts of 2).
//
// Descriptors are built once and stepped with one add per MMA.
constexpr uint32_t kDescHi = sdesc_hi(1024);   // 8-row groups 1024 bytes apart

template <int X>
__device__ void mma_issuer(const PrefillParams& p, uint8_t* smem, Bars2* bars, uint32_t tmem) {
  volatile int* abort_flag = &bars->abort;
  volatile uint32_t* flags = bars->flags;
  constexpr uint32_t idesc_s2 = make_idesc_bf16(kTileQ, 2 * kTileK, 0);
  constexpr uint32_t idesc_s1 = make_idesc_bf16(kTileQ, kTileK, 0);
  constexpr uint32_t idesc_o = make_idesc_bf16(kTileQ, kD, 1);
  const uint32_t q_lo = sdesc_lo(smem_u32(smem + OFF_Q), 16) + X * (Q_BYTES >> 4);
  const uint32_t k_lo = sdesc_lo(smem_u32(smem + OFF_K), 16);
  const uint32_t v_lo = sdesc_lo(smem_u32(smem + OFF_V), kTileK * 128);
  const uint32_t tS = tmem + kColS + 128 * X;
  const uint32_t tO = tmem + kColO + 128 * X;
  const bool pv_on = !p.stats_only;
  uint32_t qc = 0, kc = 0, vc = 0, pc = 0, uc = 0;
  // V halves of the previous pair that this head did not use: waited for (so
  // the issuer stays in step with the V loader's phases) after the next S is
  // issued, then the pair's V stage is released.
  bool pend = false;
  uint32_t pend_st = 0, pend_ph = 0, pend_mask = 0;
  bool ok = true;

  auto release_pending = [&]() -> bool {
    if (!pend) return true;
#pragma unroll
    for (int hb = 0; hb < 2; ++hb)
      if ((pend_mask >> hb) & 1u)
        if (!wait_bounded(smem_u32(&bars->v_full[pend_st][hb]), pend_ph, abort_flag, p.err,
                          X_MMA_V))
          return false;
    tc_commit(smem_u32(&bars->v_empty[pend_st]));
    pend = false;
    return true;
  };

  for (uint32_t n = 0; ok; ++n) {
    Unit2 u;
    if (!take_unit2(p, bars, n, &u, X_MMA_UNIT, false)) {
      ok = false;
      break;
    }
    if (u.n < 0) break;
    if (u.n == 0) continue;
    if (!wait_bounded(smem_u32(&bars->q_full), qc & 1, abort_flag, p.err, X_MMA_Q)) {
      ok = false;
      break;
    }
    ++qc;
    const int np = (u.n + 1) >> 1;
    bool first = true;
    for (int j = 0; j < np && ok; ++j) {
      // S_X(j) = Q_X K_pair^T.  K-major operands: K-step kk reads 64-column
      // chunk kk / 4 at byte offset (kk % 4) * 32.
      const int nb = min(2, u.n - 2 * j);
      const uint32_t st = kc % KS2;
      if (!wait_bounded(smem_u32(&bars->k_full[st]), (kc / KS2) & 1, abort_flag, p.err, X_MMA_K)) {
        ok = false;
        break;
      }
      {
        const uint32_t b0 = k_lo + st * (PAIR_BYTES >> 4);
        const uint32_t idesc = nb == 2 ? idesc_s2 : idesc_s1;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t qa = ((kk >> 2) * (kTileQ * 128) + (kk & 3) * 32) >> 4;
          const uint32_t kb = ((kk >> 2) * (2 * kTileK * 128) + (kk & 3) * 32) >> 4;
          umma_ss_w(tS, q_lo + qa, kDescHi, b0 + kb, kDescHi, idesc, kk > 0 ? 1u : 0u);
        }
      }
      tc_commit(smem_u32(&bars->s_full[X]));
      tc_commit(smem_u32(&bars->k_empty[st]));
      if (j == np - 1) tc_commit(smem_u32(&bars->q_empty));
      ++kc;
      if (!release_pending()) {
        ok = false;
        break;
      }

      // Hand-off of pair j from this head's softmax (P in TMEM, keep bits).
      if (!wait_bounded(smem_u32(&bars->p_ready[X]), pc & 1, abort_flag, p.err, X_MMA_P)) {
        ok = false;
        break;
      }
      ++pc;
      tc_fence_after();
      if (!pv_on) continue;
      const uint32_t f = flags[X];
      if (j == 0 && uc > 0) {
        // The previous unit's epilogue must have read O_X before it is overwritten.
        if (!wait_bounded(smem_u32(&bars->o_free[X]), (uc - 1) & 1, abort_flag, p.err,
                          X_MMA_OFREE)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      const uint32_t vs = vc % VS2, vph = (vc / VS2) & 1;
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        if (!((f >> hb) & 1u)) continue;
        if (!wait_bounded(smem_u32(&bars->v_full[vs][hb]), vph, abort_flag, p.err, X_MMA_V)) {
          ok = false;
          break;
        }
        // MN-major V: K-step kk reads key rows 16 kk .. 16 kk + 15; P of block
        // hb sits at S columns 64 hb .. 64 hb + 31.
        const uint32_t b0 = v_lo + vs * (PAIR_BYTES >> 4) + hb * (HALF_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk)
          umma_ts_w(tO, tS + hb * 64 + kk * 8, b0 + ((kk * 16 * 128) >> 4), kDescHi, idesc_o,
                    (first && kk == 0) ? 0u : 1u);
        first = false;
      }
      if (!ok) break;
      pend = true;
      pend_st = vs;
      pend_ph = vph;
      pend_mask = ~f & 3u;
      ++vc;
      if (j == np - 1) tc_commit(smem_u32(&bars->o_full[X]));
    }
    ++uc;
  }
  if (ok && !release_pending()) ok = false;
  if (!ok) {
    // Let every MMA already issued finish before TMEM and shared memory go away.
    tc_commit(smem_u32(&bars->drain[X]));
    wait_drain(smem_u32(&bars->drain[X]), 0);
  }
}

// --------------------------------------------------------------- softmax --
// 64 fp32 logits of this thread's row from TMEM columns [taddr, taddr + 64).
__device__ __forceinline__ void load_block(uint32_t taddr, float (&x)[64]) {
  uint32_t r0[32], r1[32];
  tmem_ld32(taddr, r0);
  tmem_ld32(taddr + 32, r1);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    x[c] = __uint_as_float(r0[c]);
    x[32 + c] = __uint_as_float(r1[c]);
  }
}

// p = 2^(x[OFF+c] * scale_log2 - m) for the 64 logits of one block: the
// argument and the row sum in packed f32x2 arithmetic, the exponentials on
// MUFU; P goes to TMEM as 32 columns of bf16 pairs.
__device__ __forceinline__ float exp_block_to_tmem(const float (&x)[64], uint64_t sl2,
                                                   uint64_t nmb, uint32_t taddr) {
  constexpr int OFF = 0;
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  uint32_t pk[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    float a0, a1;
    f2_unpack(f2_fma(f2_pack(x[OFF + 2 * c], x[OFF + 2 * c + 1]), sl2, nmb), a0, a1);
    const float p0 = ex2(a0), p1 = ex2(a1);
    acc[c & 3] = f2_add(acc[c & 3], f2_pack(p0, p1));
    pk[c] = pack_bf16x2(p0, p1);
  }
  tmem_st32(taddr, pk);
  float s0, s1;
  f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), s0, s1);
  return s0 + s1;
}

__device__ void softmax2(const PrefillParams& p, Bars2* bars, uint32_t tmem, int warp, int lane) {
  volatile int* abort_flag = &bars->abort;
  volatile uint32_t* flags = bars->flags;
  const int x = (warp - 4) >> 2;               // head slot
  const int q4 = warp & 3;                     // TMEM lane quadrant of this warp
  const int row = q4 * 32 + lane;              // query row within the tile
  const bool leader = (warp & 3) == 0 && lane == 0;
  const uint32_t bar_id = 1 + x;               // named barrier of this warpgroup
  const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
  const uint32_t tS = tmem + lane_base + kColS + 128 * x;
  const uint32_t tO = tmem + lane_base + kColO + 128 * x;
  const bool post_dec = p.gate && !p.stats_only;
  uint32_t g = 0, uc = 0;

  for (uint32_t n = 0;; ++n) {
    Unit2 u;
    if (!take_unit2(p, bars, n, &u, X_SM_UNIT, true)) return;
    if (u.n < 0) break;
    const int h = 2 * u.hp + x;
    const int i = u.t * kTileQ + row;
    const bool row_ok = i < p.N;
    const int64_t orow = (int64_t)(u.b * p.H + h) * p.N + i;
    const int64_t tile_base = ((int64_t)(u.b * p.H + h) * p.T + u.t) * p.n_kb;
    const float tau = post_dec ? __ldg(p.thresholds + h) : 0.f;
    float m = -INFINITY, l = 0.f;
    uint32_t kept = 0;   // pairs of this unit with at least one kept block
    const int np = (u.n + 1) >> 1;

    for (int j = 0; j < np; ++j, ++g) {
      const int nb = min(2, u.n - 2 * j);
      const int ea = __ldg(p.entries + u.beg + 2 * j);
      const int eb = nb == 2 ? __ldg(p.entries + u.beg + 2 * j + 1) : 0;
      const int kba = ea >> 1, kbb = eb >> 1;
      const bool pa = ea & 1, pb = eb & 1;
      uint64_t visa = ~0ull, visb = ~0ull;
      if (pa || pb) {
        // The paired-head kernel never sees random tables; the row's part of
        // the predicate is cheap enough to build per partial pair.
        RowRandom none;
        none.n = 0;
        none.row = nullptr;
        const RowVis rv = row_vis(p, none, i);
        if (pa) visa = vis_bits(p, rv, h, i, kba);
        if (pb) visb = vis_bits(p, rv, h, i, kbb);
      }
      bool slot_ok = true;
      if (leader && post_dec)
        slot_ok = wait_bounded(smem_u32(&bars->dec_empty[x][g % kDecRing2]),
                               ((g / kDecRing2) & 1) ^ 1, abort_flag, p.err, X_SM_DEC);
      if (!wait_bounded(smem_u32(&bars->s_full[x]), g & 1, abort_flag, p.err, X_SM_S)) return;
      tc_fence_after();
      // Pass 1: the row maxima of the two blocks, one block (64 logits) in
      // registers at a time; block b stays in registers for pass 2.
      float xb[64];
      float mxa, mxb = -INFINITY;
      {
        float xa[64];
        load_block(tS, xa);
        if (pa) apply_mask(visa, xa);
        mxa = row_max64(xa);
      }
      if (nb == 2) {
        load_block(tS + 64, xb);
        if (pb) apply_mask(visb, xb);
        mxb = row_max64(xb);
      }
      uint32_t keep = (1u << nb) - 1u;
      if (p.want_stats) {
        const float wa = warp_max(mxa), wb = warp_max(mxb);
        const uint32_t fb = g & 1;
        if (lane == 0) {
          bars->red[x][fb][0][q4] = wa;
          bars->red[x][fb][1][q4] = wb;
        }
        named_bar_sync(bar_id, 128);
        const float ta = fmaxf(fmaxf(bars->red[x][fb][0][0], bars->red[x][fb][0][1]),
                               fmaxf(bars->red[x][fb][0][2], bars->red[x][fb][0][3]));
        const float tb = fmaxf(fmaxf(bars->red[x][fb][1][0], bars->red[x][fb][1][1]),
                               fmaxf(bars->red[x][fb][1][2], bars->red[x][fb][1][3]));
        const float sta = ta * p.scale, stb = tb * p.scale;
        if (p.gate) {
          keep = 0;
          if (!p.stats_only) {
            if (pa || !(sta < tau)) keep |= 1u;
            if (nb == 2 && (pb || !(stb < tau))) keep |= 2u;
          }
        }
        if (leader) {
          if (p.stat_out) {
            p.stat_out[tile_base + kba] = sta;
            if (nb == 2) p.stat_out[tile_base + kbb] = stb;
          }
          if (p.mask_out) {
            p.mask_out[tile_base + kba] = (keep & 1u) || p.stats_only ? 1 : 2;
            if (nb == 2) p.mask_out[tile_base + kbb] = (keep & 2u) || p.stats_only ? 1 : 2;
          }
          if (post_dec && slot_ok) {
            const uint32_t slot = g % kDecRing2;
            reinterpret_cast<volatile uint32_t*>(bars->dec_val[x])[slot] = keep;
            mbar_arrive(smem_u32(&bars->dec_full[x][slot]));
          }
        }
      } else if (leader && p.mask_out) {
        p.mask_out[tile_base + kba] = 1;
        if (nb == 2) p.mask_out[tile_base + kbb] = 1;
      }
      if (leader) flags[x] = keep;
      if (keep == 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_ready[x]));
        continue;
      }

      // Online softmax in the log2 domain with a lazily updated max.
      float mx = -INFINITY;
      if (keep & 1u) mx = mxa;
      if (keep & 2u) mx = fmaxf(mx, mxb);
      const float m_new = fmaxf(m, mx * p.scale_log2);
      const bool need = m_new > m + kRescaleLog2b || (m == -INFINITY && m_new != -INFINITY);
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m - m_new);   // m = -inf -> 0
        l *= alpha;
        m = m_new;
      }
      const float mb = (m == -INFINITY) ? 0.f : m;
      const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
      const uint64_t nmb = f2_pack(-mb, -mb);
      // Pass 2: P of block b over S columns 64..95 (block b's logits are in
      // registers), then block a read again and its P over columns 0..31.
      if (keep & 2u) l += exp_block_to_tmem(xb, sl2, nmb, tS + 64);
      if (keep & 1u) {
        float xa[64];
        load_block(tS, xa);
        if (pa) apply_mask(visa, xa);
        l += exp_block_to_tmem(xa, sl2, nmb, tS);
      }
      if (kept > 0 && __any_sync(0xffffffffu, need)) {
        // Every earlier PV of this head has completed (S_x of this pair was
        // issued after them): rescale O_x in place.  Done after P is written
        // (the logits are no longer live) and before the hand-off, which is
        // what orders it before this pair's PV.
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_ready[x]));
      ++kept;
    }

    if (p.stats_only) continue;
    uint16_t* orow_ptr = p.O + orow * kD;
    if (u.n > 0) {
      if (!wait_bounded(smem_u32(&bars->o_full[x]), uc & 1, abort_flag, p.err, X_SM_O)) return;
      ++uc;
      tc_fence_after();
      if (kept > 0) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->o_free[x]));
    }
    if (kept == 0 && row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(orow_ptr);
      for (int v = 0; v < kD / 8; ++v) dst[v] = make_uint4(0, 0, 0, 0);
    }
    if (row_ok && p.lse)
      p.lse[orow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
}

__global__ void __launch_bounds__(kThreads2, 1)
    prefill_pair_kernel(const __grid_constant__ PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars2* bars = reinterpret_cast<Bars2*>(smem + OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 2);   // released by both issuers
    for (int s = 0; s < KS2; ++s) {
      mbar_init(smem_u32(&bars->k_full[s]), 1);
      mbar_init(smem_u32(&bars->k_empty[s]), 2);   // released by both issuers
    }
    for (int s = 0; s < VS2; ++s) {
      mbar_init(smem_u32(&bars->v_full[s][0]), 1);
      mbar_init(smem_u32(&bars->v_full[s][1]), 1);
      mbar_init(smem_u32(&bars->v_empty[s]), 2);   // released by both issuers
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_u32(&bars->s_full[x]), 1);
      mbar_init(smem_u32(&bars->p_ready[x]), 4);
      mbar_init(smem_u32(&bars->o_full[x]), 1);
      mbar_init(smem_u32(&bars->o_free[x]), 4);
      for (uint32_t r = 0; r < kDecRing2; ++r) {
        mbar_init(smem_u32(&bars->dec_full[x][r]), 1);
        mbar_init(smem_u32(&bars->dec_empty[x][r]), 1);
      }
    }
    for (uint32_t r = 0; r < kUnitRing2; ++r) {
      mbar_init(smem_u32(&bars->u_full[r]), 1);
      mbar_init(smem_u32(&bars->u_empty[r]), kUnitConsumers2);
    }
    mbar_init(smem_u32(&bars->drain[0]), 1);
    mbar_init(smem_u32(&bars->drain[1]), 1);
    bars->abort = 0;
    bars->flags[0] = bars->flags[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols2);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegControl));
    if (lane == 0) {
      if (warp == 0) producer2(p, smem, bars);
      else if (warp == 1) mma_issuer<0>(p, smem, bars, tmem);
      else if (warp == 2) vloader2(p, smem, bars);
      else mma_issuer<1>(p, smem, bars, tmem);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols2);
    // The last CTA to finish resets the work-queue counters for the next launch.
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(p.sched + 1, 1) == int(gridDim.x) - 1) {
        atomicExch(p.sched, 0);
        atomicExch(p.sched + 1, 0);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
    softmax2(p, bars, tmem, warp, lane);
    tc_fence_before();
    __syncthreads();
  }
}

int g_num_sms2[64] = {0};
bool g_attr_set2[64] = {false};

}  // namespace

int launch_prefill_pair(const PrefillParams& p, int d, cudaStream_t stream) {
  if (d != kD) return set_error(SA_ERR_UNSUPPORTED, "paired-head kernel: head dim %d", d);
  if (p.head_pat || p.H % 2 || (p.H / p.Hkv) % 2)
    return set_error(SA_ERR_INVALID_ARG, "paired-head kernel: heads cannot be paired");
  if (p.dil != 1) return set_error(SA_ERR_UNSUPPORTED, "paired-head kernel: dilated window");
  if (p.skip_denominator)
    return set_error(SA_ERR_UNSUPPORTED, "paired-head kernel: skipped keys kept in the denominator");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return set_error(SA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  if (g_num_sms2[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_num_sms2[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_error(e, "cudaDeviceGetAttribute");
  }
  if (p.n_units == 0) return SA_OK;
  if (!g_attr_set2[dev]) {
    // The register split assumes kRegLaunch registers per thread at launch.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, prefill_pair_kernel);
    if (e != cudaSuccess) return cuda_error(e, "cudaFuncGetAttributes");
    if (fa.numRegs != kRegLaunch)
      return set_error(SA_ERR_UNSUPPORTED,
                       "paired-head kernel built with %d registers per thread, its register "
                       "split needs %d",
                       fa.numRegs, kRegLaunch);
    e = cudaFuncSetAttribute(prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM2);
    if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute");
    g_attr_set2[dev] = true;
  }
  const int grid = p.n_units < g_num_sms2[dev] ? p.n_units : g_num_sms2[dev];
  prefill_pair_kernel<<<grid, kThreads2, SMEM2, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "paired-head prefill launch");
  return SA_OK;
}

}  // namespace sa
