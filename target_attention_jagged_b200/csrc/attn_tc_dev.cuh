// Tensor-core split-L single-query attention over the jagged encoded history:
// the kernel's device code (parameters, shared-memory layout, body), shared by
// its own kernel (attn_tc.cu) and the pipelined step kernel (step_tc.cu).
//
// For request r the T_r * h query rows are u_j of every target t and head j,
// scaled by log2(e) / sqrt(d_h) ("Make It Long, Keep It Fast" digest §2.1,
// Eq. (13); the blog's reordered single-query attention, §2.4).  They all
// attend to the same L_r keys X~_r, so one pass over X~_r serves every target:
//   S = U_tile X~_tile^T         (tcgen05, M = 128 query rows, N = 128 keys, K = d)
//   P = exp2(S - m), online max / sum per row (CUDA cores, one row per thread)
//   O += P X~_tile               (tcgen05, M = 128, N = d, K = 128 keys)
// The same shared-memory copy of each X~ tile is the K-major B operand of the
// first MMA and the MN-major B operand of the second.  With d <= 128, P stays
// in TMEM (packed bf16) and the second MMA takes it from there, which keeps
// shared-memory bandwidth for the MMAs' operands and the TMA writes.  Work is
// cut stream-K style: every CTA gets an equal run of (query tile, key tile)
// units in (request, query tile, key) order, so ragged lengths do not
// unbalance the SMs; each maximal run inside one (request, query tile) pair is
// an item that writes an unnormalised partial (O, m, l) for the split combine.
//
// The running max is rescaled lazily: O and l are corrected only when a row's
// max grows by more than 8 (log2 units); otherwise P uses the stale max and
// stays below 2^8, well inside bf16 and fp32 range.
//
// The naive form (Eq. (12), SEPV) runs the same kernel on projected keys and
// values: the query rows are q W_Q of G = 64 / d_h heads packed into one tile
// (each row non-zero only in its own head's d_h features), S contracts the
// tile's 64 head-group features of K = X~ W_K, and O += P V takes the same 64
// features of V = X~ W_V from a second shared-memory tile loaded beside K.
//
// Warp roles (352 threads): warp 0 TMA, warp 1 issues S (and owns TMEM),
// warps 2-9 softmax / correction / partial store (one query row per thread,
// two warps -- key halves -- per row), warp 10 issues P X~.  Two issuers let
// S of later tiles run ahead of the P X~ products, which wait for the
// softmax.
#pragma once

#include <cuda.h>

#include "stca_internal.h"
#include "softmax_exp.cuh"
#include "tc_common.cuh"

namespace stca {
namespace {

using namespace tc;

struct AttnParams {
  const AttnItem* items;
  const int32_t* cta_item_begin;   // gridDim.x + 1
  float* pacc;                     // G x d (PROJ: G x d_h, the projected rows)
  float* pm;                       // G
  float* pl;                       // G
  int* status;
  int stop_tiles;                  // > 0: the loader stops after this many key tiles (test hook)
  int h, dh;                       // PROJ: heads and head width (query row r is head r % h)
  // PROJ with qslot: partials are kept per (query row, item of its pair), at
  // most kQslots items per pair: row q's item w at pacc[(q kQslots + w) d_h],
  // its (m, l) at qml[(q kQslots + w) 2], and the pair's item count at qn[q]
  int qslot;
  const int32_t* pair_item_begin;  // pairs + 1
  float* qml;
  int* qn;
};

// P_TMEM: P lives in TMEM (packed bf16, 64 columns per buffer) and the P X~
// product reads it from there; with d = 256 TMEM is full (S and O) and P goes
// through shared memory.  Keeping P out of shared memory matters: the MMAs'
// operand reads, the TMA writes of X~ and the P writes would otherwise all
// share its bandwidth.
// QT: the query tile is copied from shared memory into TMEM once per item and
// S = U X~^T takes it from there (a TMEM A operand), so the key tiles' S
// products read only X~ from shared memory.
// PROJ (with QT, d = 128): the item's output rows are projected by W_V in the
// kernel (Eqs. (6), (13): o_j = alpha_j X~ W_V^j, and the split combine is
// linear, so the unnormalised partials may be projected before it): O is
// rounded to bf16 into the P columns of TMEM, one more product O W_V (all
// heads' W_V^j side by side, B = [W_V]^T from shared memory, loaded once per
// CTA) overwrites the O accumulator, and each row keeps only its head's d_h
// columns.  Partials shrink from d to d_h floats per row, and the per-target
// step starts from o_j directly.
template <int D, int QB, int KS, int PB, bool SEPV, bool QT = false, bool PROJ = false>
struct AttnCfg {
  static constexpr bool P_TMEM = D <= 128;
  static constexpr int KB = D / 64;
  static constexpr uint32_t kBlock = 128u * 128u;       // [128 rows x 64] bf16
  static constexpr uint32_t kTile = KB * kBlock;         // [128 rows x D]
  static constexpr uint32_t kStage = SEPV ? 2 * kTile : kTile;   // key tile (+ value tile)
  static constexpr uint32_t kPBytes = 2 * kBlock;        // [128 rows x 128 keys]
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + QB * kTile;
  static constexpr uint32_t oP = oK + KS * kStage;
  static constexpr uint32_t oWv = oP + (P_TMEM ? 0 : PB * kPBytes);  // PROJ: [W_V]^T, d x d
  static constexpr uint32_t oX = oWv + (PROJ ? kTile : 0);   // pair exchange: 2 x 2 x 128 floats
  static constexpr uint32_t oBar = oX + 2 * 2 * 128 * 4;
  static constexpr int kBars = 2 * QB + 2 * KS + 4 + 2 * PB + 3 + 1 + 8 + 1 + 3;
  static constexpr uint32_t oMisc = oBar + kBars * 8;
  // No alignment slack: the dynamic shared memory of a block starts at a
  // 1024-byte boundary (after the 1 KB the system reserves), and the kernel
  // checks that before it uses any of it.
  static constexpr uint32_t kSmem = oMisc + 16;
  static constexpr uint32_t kS = 0;        // 2 x 128 TMEM columns of scores
  static constexpr uint32_t kO = 256;      // D columns of the output accumulator
  static constexpr uint32_t kPt = kO + D;  // P_TMEM: PB x 64 columns of P
  static constexpr uint32_t kQt = kPt + (P_TMEM ? PB * 64 : 0);   // QT: D / 2 columns of U
  static_assert(kQt + (QT ? D / 2 : 0) <= 512, "TMEM overflow");
  static_assert(!QT || (P_TMEM && !SEPV), "the TMEM query tile is for the reordered form, d <= 128");
  static_assert(!PROJ || (QT && D == 128 && PB == 1), "the in-kernel projection reuses the P columns");
  static_assert(kSmem <= 227 * 1024, "shared memory overflow");
};

constexpr int kSoftWarps = 8;               // two per TMEM lane quarter
constexpr int kPvWarp = 2 + kSoftWarps;     // issues the P X~ products
constexpr int kAttnThreads = 32 * (kPvWarp + 1);
constexpr float kRescaleThreshold = 8.0f;   // log2 units
#ifndef STCA_TC_FMA_PAIRS
#define STCA_TC_FMA_PAIRS 1
#endif
// Of every 4 key pairs, this many take exp2 on the FMA pipe (the degree-3
// polynomial) and the rest the MUFU; at c3 one in four measured best (forward
// 0.232 ms, against 0.243 with none and 0.234 with two).
constexpr int kFmaPairs = STCA_TC_FMA_PAIRS;

__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      int* status) {
  if (mbar_wait(bar, parity, abort_flag)) return true;
  *abort_flag = 1;
  atomicOr(status, kStatusAttnTimeout);
  return false;
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > ns) break;
}

using sx::ex2;
using sx::ex2_fma;

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}


// The kernel's body for CTA `cta` of its grid (the CTA's work is the plan's
// items cta_item_begin[cta] .. [cta + 1]), on dynamic shared memory smem_raw
// (1024-byte aligned) and kAttnThreads threads.  tmV: the value tiles (SEPV)
// or the [W_V]^T tile (PROJ); otherwise unused.  The tensor maps must be
// kernel parameters (__grid_constant__) of the calling kernel.
template <int D, int QB, int KS, int PB, bool SEPV, bool QT, bool PROJ>
__device__ __forceinline__ void attn_tc_body(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                             const CUtensorMap& tmV, const AttnParams& p,
                                             uint8_t* smem_raw, int cta) {
  using C = AttnCfg<D, QB, KS, PB, SEPV, QT, PROJ>;
  if (smem_u32(smem_raw) & 1023u) {      // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.status, kStatusAttnTimeout);
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* qfull = reinterpret_cast<uint64_t*>(sm + C::oBar);
  uint64_t* qempty = qfull + QB;
  uint64_t* kfull = qempty + QB;
  uint64_t* kempty = kfull + KS;
  uint64_t* sfull = kempty + KS;      // 2
  uint64_t* sempty = sfull + 2;       // 2
  uint64_t* pfull = sempty + 2;       // PB
  uint64_t* pempty = pfull + PB;      // PB
  uint64_t* odone = pempty + PB;      // one phase per P X~ MMA group
  uint64_t* ofinal = odone + 1;       // one phase per item
  uint64_t* oempty = ofinal + 1;      // one phase per item (partial stored)
  uint64_t* mdrain = oempty + 1;
  uint64_t* xmax = mdrain + 1;        // [quarter][parity]: the pair's exchange
  uint64_t* qtdone = xmax + 8;        // QT: one phase per item (its S products are done)
  uint64_t* wvfull = qtdone + 1;      // PROJ: the [W_V]^T tile has landed
  uint64_t* obready = wvfull + 1;     // PROJ: one phase per item (O as bf16 is in TMEM)
  uint64_t* vdone = obready + 1;      // PROJ: one phase per item (O W_V is done)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int it0 = p.cta_item_begin[cta], it1 = p.cta_item_begin[cta + 1];
  if (threadIdx.x == 0) {
    for (int i = 0; i < QB; ++i) { mbar_init(&qfull[i], 1); mbar_init(&qempty[i], 1); }
    for (int i = 0; i < KS; ++i) { mbar_init(&kfull[i], 1); mbar_init(&kempty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&sfull[i], 1); mbar_init(&sempty[i], kSoftWarps); }
    for (int i = 0; i < PB; ++i) { mbar_init(&pfull[i], kSoftWarps); mbar_init(&pempty[i], 1); }
    mbar_init(odone, 1);
    mbar_init(ofinal, 1);
    mbar_init(oempty, kSoftWarps);
    mbar_init(mdrain, 2);
    for (int i = 0; i < 8; ++i) mbar_init(&xmax[i], 2);
    mbar_init(qtdone, 1);
    mbar_init(wvfull, 1);
    mbar_init(obready, kSoftWarps);
    mbar_init(vdone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    if constexpr (SEPV || PROJ) prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();                          // the predecessor's results are visible from here on
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t stream_policy = policy_evict_first();   // X~ is read once per layer
      uint32_t qi = 0, ki = 0;
      bool ok = true;
      if constexpr (PROJ) {
        if (it0 < it1) {
          mbar_arrive_expect_tx(wvfull, C::kTile);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(sm + C::oWv + kb * C::kBlock, &tmV, kb * 64, 0, wvfull);
        }
      }
      for (int it = it0; ok && it < it1; ++it) {
        const AttnItem item = p.items[it];
        const int qb = qi % QB;
        if (!(ok = bwait(&qempty[qb], ((qi / QB) & 1) ^ 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(&qfull[qb], C::kTile);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(sm + C::oQ + qb * C::kTile + kb * C::kBlock, &tmQ, kb * 64,
                      static_cast<int>(item.qrow0), &qfull[qb]);
        ++qi;
        const int nt = (item.nkeys + 127) >> 7;
        for (int j = 0; j < nt; ++j) {
          if (p.stop_tiles > 0 && ki >= static_cast<uint32_t>(p.stop_tiles)) {
            // test hook: give up here as a wait that ran out would
            *abort_flag = 1;
            atomicOr(p.status, kStatusAttnTimeout);
            ok = false;
            break;
          }
          const int s = ki % KS;
          if (!(ok = bwait(&kempty[s], ((ki / KS) & 1) ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(&kfull[s], C::kStage);
          const int kx = SEPV ? item.kcol : 0;      // head-group features (naive form)
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d_hint(sm + C::oK + s * C::kStage + kb * C::kBlock, &tmK, kx + kb * 64,
                             static_cast<int>(item.key0 + j * 128), &kfull[s], stream_policy);
          if constexpr (SEPV)
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_2d_hint(sm + C::oK + s * C::kStage + C::kTile + kb * C::kBlock, &tmV,
                               kx + kb * 64, static_cast<int>(item.key0 + j * 128), &kfull[s],
                               stream_policy);
          ++ki;
        }
      }
      // Let every copy still in flight land before the CTA can exit: after a
      // failed wait elsewhere the consumers may have stopped waiting for them.
      // (On the normal path these phases have completed and the waits return
      // at once.)
      for (uint32_t c = ki > KS ? ki - KS : 0; c < ki; ++c) drain_wait(&kfull[c % KS], (c / KS) & 1, 100000000ull);
      for (uint32_t c = qi > QB ? qi - QB : 0; c < qi; ++c) drain_wait(&qfull[c % QB], (c / QB) & 1, 100000000ull);
      if (PROJ && it0 < it1) drain_wait(wvfull, 0, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    // S of the next tile is issued as soon as its TMEM buffer is free (the
    // softmax has loaded the tile two back), ahead of the P X~ products.
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128);                 // Q K-major, X~ K-major
      uint32_t qi = 0, ki = 0, sc = 0;
      bool ok = true;
      for (int it = it0; ok && it < it1; ++it) {
        const AttnItem item = p.items[it];
        const int nt = (item.nkeys + 127) >> 7;
        const int qb = qi % QB;
        if constexpr (QT) {
          // the previous item's S products read the TMEM copy of its query tile
          if (qi > 0 && !(ok = bwait(qtdone, (qi - 1) & 1, abort_flag, p.status))) break;
        }
        if (!(ok = bwait(&qfull[qb], (qi / QB) & 1, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t qaddr = sbase + C::oQ + qb * C::kTile;
        if constexpr (QT) {
          // 16 features of the 128 rows per copy, into the columns the S
          // products read as their A operand (2 bf16 per column)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tmem_cp_128x256b(tmem + C::kQt + kk * 8,
                             sdesc_sw128(qaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024));
          mma_commit(&qempty[qb]);           // the shared-memory tile is free once copied
        }
        for (int j = 0; ok && j < nt; ++j, ++sc, ++ki) {
          const int sb = sc & 1;
          if (!(ok = bwait(&sempty[sb], ((sc >> 1) & 1) ^ 1, abort_flag, p.status))) break;
          const int s = ki % KS;
          if (!(ok = bwait(&kfull[s], (ki / KS) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t kaddr = sbase + C::oK + s * C::kStage;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t kd = sdesc_sw128(kaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024);
            if constexpr (QT)
              mma_bf16_ts(tmem + C::kS + sb * 128, tmem + C::kQt + kk * 8, kd, idS, kk != 0);
            else
              mma_bf16_ss(tmem + C::kS + sb * 128,
                          sdesc_sw128(qaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024), kd,
                          idS, kk != 0);
          }
          mma_commit(&sfull[sb]);
          if (j + 1 == nt) mma_commit(QT ? qtdone : &qempty[qb]);
        }
        ++qi;
      }
      mma_commit(mdrain);
      drain_wait(mdrain, 0, 500000000ull);
    }
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ P X~ issuer
    // The K tile of S(j) is the V tile of this product; its arrival is known
    // from the S issuer's wait (S(j) -> softmax(j) -> pfull), and its stage is
    // released here.
    if (lane == 0) {
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);      // P K-major, X~ MN-major
      uint32_t ki = 0, pc = 0, ic = 0;
      bool ok = true;
      for (int it = it0; ok && it < it1; ++it, ++ic) {
        const AttnItem item = p.items[it];
        const int nt = (item.nkeys + 127) >> 7;
        for (int j = 0; ok && j < nt; ++j, ++pc, ++ki) {
          const int pb = pc % PB;
          if (!(ok = bwait(&pfull[pb], (pc / PB) & 1, abort_flag, p.status))) break;
          if (j == 0 && !(ok = bwait(oempty, (ic & 1) ^ 1, abort_flag, p.status))) break;
          tc_fence_after();
          const int s = ki % KS;
          const uint32_t vaddr = sbase + C::oK + s * C::kStage + (SEPV ? C::kTile : 0u);
          if constexpr (C::P_TMEM) {
            // P: keys 2c, 2c+1 in column c of the buffer; 16 keys = 8 columns per MMA
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_bf16_ts(tmem + C::kO, tmem + C::kPt + pb * 64 + kk * 8,
                          sdesc_sw128(vaddr + kk * 2048, C::kBlock, 1024), idO, (j | kk) != 0);
          } else {
            const uint32_t paddr = sbase + C::oP + pb * C::kPBytes;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)   // 16 keys per MMA
              mma_bf16_ss(tmem + C::kO,
                          sdesc_sw128(paddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024),
                          sdesc_sw128(vaddr + kk * 2048, C::kBlock, 1024), idO,
                          (j | kk) != 0);
          }
          mma_commit(&kempty[s]);
          mma_commit(&pempty[pb]);
          mma_commit(odone);
        }
        if (!ok) break;
        mma_commit(ofinal);
        if constexpr (PROJ) {
          // O W_V: A = O as bf16 (written by the softmax warps into the P
          // columns), B = [W_V]^T K-major; the result overwrites O
          constexpr uint32_t idV = idesc_bf16(128, D);
          if (ic == 0 && !(ok = bwait(wvfull, 0, abort_flag, p.status))) break;
          if (!(ok = bwait(obready, ic & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t waddr = sbase + C::oWv;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ts(tmem + C::kO, tmem + C::kPt + kk * 8,
                        sdesc_sw128(waddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024), idV, kk != 0);
          mma_commit(vdone);
        }
      }
      mma_commit(mdrain);
      drain_wait(mdrain, 0, 500000000ull);
    }
  } else {
    // ------------------------------------------------------------ softmax + partials
    // Two warps per TMEM lane quarter: half hf of the pair takes keys
    // [64 hf, 64 hf + 64) of every tile for the quarter's 32 query rows, and
    // columns [hf D/2, (hf + 1) D/2) of O when it is rescaled or stored.  The
    // pair swaps row maxima (and, at the end of an item, row sums) through
    // shared memory; both then take identical rescaling decisions.
    const int q = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = q * 32 + lane;              // query row of the tile (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    float* xbuf = reinterpret_cast<float*>(sm + C::oX);   // [2 parity][2 halves][128 rows]
    uint64_t* xbar = xmax + q * 2;            // this pair's exchange barriers
    uint32_t xp = 0;                          // exchanges so far
    // swap v with the partner warp: returns the partner's value for row r
    auto swap_with_pair = [&](float v, bool& okk) -> float {
      float* xs = xbuf + (xp & 1) * 256;
      xs[hf * 128 + r] = v;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xbar[xp & 1]);
      okk = bwait(&xbar[xp & 1], (xp >> 1) & 1, abort_flag, p.status);
      const float o = xs[(hf ^ 1) * 128 + r];
      ++xp;
      return o;
    };
    uint32_t sc = 0, pc = 0, ic = 0;
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it, ++ic) {
      const AttnItem item = p.items[it];
      const int nt = (item.nkeys + 127) >> 7;
      float m_used = -1e30f, l = 0.f;         // l: this half's share of the row sum
      for (int j = 0; j < nt; ++j) {
        const int sb = sc & 1;
        if (!(ok = bwait(&sfull[sb], (sc >> 1) & 1, abort_flag, p.status))) break;
        __syncwarp();
        tc_fence_after();
        uint32_t sv[2][32];
#pragma unroll
        for (int cb = 0; cb < 2; ++cb)
          tmem_ld32(tmem + lane_off + C::kS + sb * 128 + hf * 64 + cb * 32, sv[cb]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
        ++sc;
        const int nvalid = min(128, item.nkeys - j * 128) - hf * 64;
        if (nvalid < 64) {   // the request's last tile: keys past its end take no weight
#pragma unroll
          for (int cb = 0; cb < 2; ++cb)
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (cb * 32 + k >= nvalid) sv[cb][k] = __float_as_uint(-INFINITY);
        }
        float m4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {            // 4 chains of 16 keys, two keys per 3-input max
          const uint32_t* v = &sv[c >> 1][(c & 1) * 16];
          m4[c] = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
          for (int k = 2; k < 16; k += 2) m4[c] = sx::max3(m4[c], __uint_as_float(v[k]), __uint_as_float(v[k + 1]));
        }
        const float mloc = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        const float mx = fmaxf(mloc, swap_with_pair(mloc, ok));
        if (!ok) break;
        const bool resc = mx > m_used + kRescaleThreshold;
        const float m_new = resc ? mx : m_used;
        const float corr = resc ? ex2(m_used - m_new) : 1.f;
        l *= corr;
        m_used = m_new;
        // pairs of keys: the subtraction and the sums in packed f32x2 form;
        // kFmaPairs of every 4 pairs take exp2 on the FMA pipe (d <= 128)
        uint32_t pk[32];
        const uint64_t negm = sx::f2(-m_new, -m_new);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int cb = 0; cb < 2; ++cb)
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const uint64_t x = sx::f2_add(sx::f2(__uint_as_float(sv[cb][k]), __uint_as_float(sv[cb][k + 1])), negm);
            float x0, x1, p0, p1;
            sx::f2_split(x, x0, x1);
            if (C::P_TMEM && ((k >> 1) & 3) < kFmaPairs) {
              sx::ex2_fma2(x0, x1, p0, p1);
            } else {
              p0 = ex2(x0);                      // exp2(-inf) = 0
              p1 = ex2(x1);
            }
            ls2[(k >> 1) & 3] = sx::f2_add(ls2[(k >> 1) & 3], sx::f2(p0, p1));
            pk[(cb * 32 + k) >> 1] = pack_bf16x2(p0, p1);
          }
        {
          float a0, a1;
          sx::f2_split(sx::f2_add(sx::f2_add(ls2[0], ls2[1]), sx::f2_add(ls2[2], ls2[3])), a0, a1);
          l += a0 + a1;
        }
        const int pb = pc % PB;
        if (!(ok = bwait(&pempty[pb], ((pc / PB) & 1) ^ 1, abort_flag, p.status))) break;
        __syncwarp();
        if constexpr (C::P_TMEM) {
          // P row, keys 64 hf .. 64 hf + 63: columns 32 hf .. 32 hf + 31 of the buffer
          tmem_st32(tmem + lane_off + C::kPt + pb * 64 + hf * 32, pk);
          tmem_st_wait();
        } else {
          // P row, keys 64 hf .. 64 hf + 63: block hf of the tile, K-major, 128-B swizzle
          const uint32_t prow = sbase + C::oP + pb * C::kPBytes + hf * C::kBlock + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(prow + ((c ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                         pk[4 * c + 3]);
        }
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
          // O holds the rows' sums up to tile j-1: wait for that MMA, then rescale
          if (!(ok = bwait(odone, (pc - 1) & 1, abort_flag, p.status))) break;
          __syncwarp();
          tc_fence_after();
#pragma unroll 1
          for (int cb = hf * (D / 64); cb < (hf + 1) * (D / 64); ++cb) {
            uint32_t ov[32];
            tmem_ld32(tmem + lane_off + C::kO + cb * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * corr);
            tmem_st32(tmem + lane_off + C::kO + cb * 32, ov);
          }
          tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pfull[pb]);
        ++pc;
      }
      if (!ok) break;
      // item done: the row sum is both halves' shares
      l += swap_with_pair(l, ok);
      if (!ok) break;
      // store the unnormalised partial of the valid rows, this half's columns
      if (!(ok = bwait(ofinal, ic & 1, abort_flag, p.status))) break;
      __syncwarp();
      tc_fence_after();
      const bool valid = r < item.rows;
      const int64_t g = item.row_base + r;
      if constexpr (PROJ) {
        // O (this half's D / 2 features) as bf16 into the P columns: column c
        // holds features 2c, 2c + 1, the A operand of O W_V
        {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t ov[32];
            tmem_ld32(tmem + lane_off + C::kO + hf * 64 + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k)
              pk[c * 16 + k] = pack_bf16x2(__uint_as_float(ov[2 * k]), __uint_as_float(ov[2 * k + 1]));
          }
          tmem_st32(tmem + lane_off + C::kPt + hf * 32, pk);
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(obready);
        if (!(ok = bwait(vdone, ic & 1, abort_flag, p.status))) break;
        __syncwarp();
        tc_fence_after();
        // the row's head j = r % h keeps columns [j d_h, (j + 1) d_h) of O W_V;
        // this half holds columns [64 hf, 64 hf + 64)
        const int j0 = (r % p.h) * p.dh - 64 * hf;     // the head's first column, in this half's terms
        int64_t slot = g;
        if (p.qslot) {
          const int w0 = p.pair_item_begin[item.pair];
          const int64_t qrow = item.qrow0 + r;
          slot = qrow * kQslots + (it - w0);
          if (valid && hf == 0) {
            p.qn[qrow] = p.pair_item_begin[item.pair + 1] - w0;
            p.qml[slot * 2] = m_used;
            p.qml[slot * 2 + 1] = l;
          }
        }
        float* dst = p.pacc + slot * p.dh;             // column j0 + c of this half -> dst[c]
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + C::kO + hf * 64 + c * 32, ov);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const int col = c * 32 + k;
              if (col >= j0 && col < j0 + p.dh) dst[col - j0] = __uint_as_float(ov[k]);
            }
          }
        }
      } else {
      float* dst = p.pacc + g * D;
#pragma unroll 1
      for (int cb = hf * (D / 64); cb < (hf + 1) * (D / 64); ++cb) {
        uint32_t ov[32];
        tmem_ld32(tmem + lane_off + C::kO + cb * 32, ov);
        tmem_ld_wait();
        if (valid) {
          float4* d4 = reinterpret_cast<float4*>(dst + cb * 32);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            d4[k] = make_float4(__uint_as_float(ov[4 * k]), __uint_as_float(ov[4 * k + 1]),
                                __uint_as_float(ov[4 * k + 2]), __uint_as_float(ov[4 * k + 3]));
        }
      }
      }   // PROJ
      if (valid && hf == 0 && !(PROJ && p.qslot)) {
        p.pm[g] = m_used;
        p.pl[g] = l;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(oempty);
    }
  }
  tc_fence_before();
  __syncthreads();
  pdl_trigger();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace
}  // namespace stca
