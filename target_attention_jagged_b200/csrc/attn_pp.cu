// Tensor-core split-L single-query attention for d in {64, 128}, with the
// split combine inside the kernel.
//
// What it computes ("Make It Long, Keep It Fast" digest §2.1, Eq. (13); the
// STCA blog's reordered single-query attention, §2.4): for request r, its
// T_r * h query rows u (target t, head j; pre-scaled by log2(e) / sqrt(d_h))
// attend to the request's L_r encoded history rows X~_r, and the merged row
// c = softmax(u X~_r^T) X~_r is written for every query row.  One pass over X~_r
// per layer serves all of the request's targets and heads:
//   S = U_tile X~_tile^T       tcgen05, M = 128 query rows, N = 128 keys, K = d
//   P = 2^(S - m), online      CUDA cores, one query row per thread
//   O += P X~_tile             tcgen05, M = 128, N = d, K = 128 keys, P from TMEM
//
// Two softmax groups.  Key tiles alternate between two groups of four warps
// (group g & 1 takes the CTA's g-th key tile).  Each group keeps its own
// running maximum m, sum l and accumulator O (its own TMEM columns), so a
// thread owns a whole row of its tile (all 128 keys) and no row statistics are
// exchanged while the tiles stream: while one group computes the
// exponentials of tile g, the tensor core runs S of tile g + 1 for the other
// group and the P X~ product of tile g - 1.  P (bf16) overwrites the first 64
// of the tile's 128 S columns; one thread issues every MMA, so S of tile g + 2
// (same columns) is ordered after the P X~ product of tile g.  The two groups'
// states are merged once per work item.  The maximum is rescaled lazily: O and
// l change only when a row's maximum grows by more than 8 (log2 units).
//
// Work and the split combine.  Work is cut stream-K style, as for the other
// tensor-core attention: each CTA takes an equal run of (query tile, key
// tile) units in (request, query tile, key) order; every maximal run inside
// one (request, query tile) pair is an item.  A pair that one item covers
// writes its normalised rows c directly.  The items of a split pair write
// unnormalised partials (O, m, l); each warp then counts its arrival on the
// pair's counter for its slot (lane quarter, column half) -- an atomic add,
// never a wait -- and the warp that arrives last merges the slot's rows of all
// the pair's items into c.  The counters must be zero when the kernel starts.
//
// Warp roles (384 threads): warp 0 loads Q and X~ tiles (TMA), warp 1 owns
// TMEM and issues all MMAs, warps 2-3 idle, warps 4-7 are softmax group 0,
// warps 8-11 group 1 (warp w reads TMEM lane quarter w % 4).  Every wait is a bounded mbarrier
// wait; a wait that gives up sets the device status and stops the CTA's other
// roles, and the CTA lets its copies and MMAs in flight finish before it exits.
#include <cuda.h>

#include <string>

#include "softmax_exp.cuh"
#include "stca_internal.h"
#include "tc_common.cuh"

namespace stca {
namespace {

using namespace tc;

struct PPParams {
  const AttnItem* items;
  const int32_t* cta_item_begin;    // gridDim.x + 1
  const int32_t* pair_item_begin;   // pairs + 1
  float* pacc;                      // G x D: unnormalised partial rows (split pairs)
  float* pml;                       // G x 4: m of each column half, then l of each half
  float* cout;                      // T h x D: merged rows c, row = query row
  int* counters;                    // pairs x 8 arrivals, zero at launch
  float* stats;                     // NULL, or T h x 2: the row's softmax max (log2 units) and sum
  int* status;
  int stop_tiles;                   // > 0: the loader stops after this many key tiles (test hook)
};

template <int D>
struct PPCfg {
  static constexpr int KB = D / 64;
  static constexpr uint32_t kBlock = 128u * 128u;          // [128 rows x 64] bf16
  static constexpr uint32_t kTile = KB * kBlock;            // [128 rows x D]
  static constexpr int QB = 2;
  static constexpr int KS = D == 128 ? 5 : 10;
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + QB * kTile;
  static constexpr uint32_t oX = oK + KS * kTile;           // (m, l) of both groups: 2 x 128 float2
  static constexpr uint32_t oBar = oX + 2 * 128 * 8;
  // qfull, qempty [QB]; kfull, kempty [KS]; sfull, pfull, odone [2]; ofinal, oempty, xbar, mdrain
  static constexpr int kBars = 2 * QB + 2 * KS + 6 + 4;
  static constexpr uint32_t oMisc = oBar + kBars * 8;
  static constexpr uint32_t kSmem = oMisc + 16;
  static constexpr uint32_t kS = 0;      // S (then P) of group b: TMEM columns 128 b ..
  static constexpr uint32_t kO = 256;    // O of group b: columns 256 + D b ..
  static_assert(kO + 2 * D <= 512, "TMEM overflow");
  static_assert(kSmem <= 227 * 1024, "shared memory overflow");
};

// Three warpgroups: warps 0-3 (loader, MMA issuer, two idle) hand registers
// to the two softmax warpgroups, so a softmax thread can hold its whole row of
// a key tile.  Launched at 168 per thread (65536 / 384, rounded down to the
// allocation unit); 128 x 48 + 256 x 224 = 63488 <= 384 x 168 = 64512.
constexpr int kPPThreads = 384;
constexpr int kPPRegsLow = 48, kPPRegsHigh = 224;
static_assert(128 * kPPRegsLow + 256 * kPPRegsHigh <= kPPThreads * 168, "register split");
constexpr float kRescale = 8.0f;                 // log2 units

__device__ __forceinline__ bool pwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      int* status) {
  if (mbar_wait(bar, parity, abort_flag)) return true;
  *abort_flag = 1;
  atomicOr(status, kStatusAttnTimeout);
  return false;
}

// The same, waited by every lane of a warp: one answer for the whole warp, so
// that the warp-collective TMEM accesses after it run on all lanes or none.
__device__ __forceinline__ bool pwait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           int* status) {
  const bool ok = pwait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ void pdrain(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > ns) break;
}

__device__ __forceinline__ void st_tmem32(uint32_t taddr, const uint32_t (&r)[32]) {
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

// The last warp to arrive on a split pair's slot merges the slot's rows (lane
// quarter q: rows 32 q .. 32 q + 31; column half b) of all the pair's items:
// c = sum_w 2^(m_w - m) acc_w / sum_w 2^(m_w - m) l_w, m = max_w m_w.  Lane r
// takes row 32 q + r: first the items' (m, l) -- a running maximum and sum --
// then, item by item, all D / 8 float4 of its half row at once, so each item
// costs one round trip to L2 (other CTAs wrote the partials; the merge runs
// at the tail of the kernel, where latency is what counts).
template <int D>
__device__ __forceinline__ void merge_slot(const PPParams& p, const AttnItem& item, int b, int q,
                                           int lane) {
  constexpr int kC4 = D / 8;                  // float4 of a half row
  const int row = q * 32 + lane;
  if (row >= item.rows) return;               // the items of a pair share its rows
  const int w0 = p.pair_item_begin[item.pair], w1 = p.pair_item_begin[item.pair + 1];
  float mx = -INFINITY, L = 0.f;
#pragma unroll 4
  for (int w = w0; w < w1; ++w) {
    const int64_t g = p.items[w].row_base + row;
    const float mw = __ldcg(p.pml + g * 4 + b), lw = __ldcg(p.pml + g * 4 + 2 + b);
    if (mw > mx) {
      L = L * sx::ex2(mx - mw) + lw;           // 0 from mx = -inf
      mx = mw;
    } else {
      L = fmaf(lw, sx::ex2(mw - mx), L);
    }
  }
  const float inv = 1.f / L;
  if (p.stats && b == 0) {
    p.stats[(item.qrow0 + row) * 2] = mx;
    p.stats[(item.qrow0 + row) * 2 + 1] = L;
  }
  float4 acc[kC4];
#pragma unroll
  for (int c = 0; c < kC4; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
  for (int w = w0; w < w1; ++w) {
    const int64_t g = p.items[w].row_base + row;
    const float f = sx::ex2(__ldcg(p.pml + g * 4 + b) - mx) * inv;
    const float4* src = reinterpret_cast<const float4*>(p.pacc + g * D + b * (D / 2));
    float4 v[kC4];
#pragma unroll
    for (int c = 0; c < kC4; ++c) v[c] = __ldcg(src + c);
#pragma unroll
    for (int c = 0; c < kC4; ++c) {
      acc[c].x = fmaf(f, v[c].x, acc[c].x);
      acc[c].y = fmaf(f, v[c].y, acc[c].y);
      acc[c].z = fmaf(f, v[c].z, acc[c].z);
      acc[c].w = fmaf(f, v[c].w, acc[c].w);
    }
  }
  float4* dst = reinterpret_cast<float4*>(p.cout + (item.qrow0 + row) * D + b * (D / 2));
#pragma unroll
  for (int c = 0; c < kC4; ++c) dst[c] = acc[c];
}

// FMA_PAIRS of every 4 consecutive pairs of a row's exponentials go to the
// FMA pipe (sx::ex2_fma2), the rest to the MUFU.
template <int D, int FMA_PAIRS>
__global__ void __launch_bounds__(kPPThreads, 1)
attn_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const PPParams p) {
  using C = PPCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {      // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.status, kStatusAttnTimeout);
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* qfull = reinterpret_cast<uint64_t*>(sm + C::oBar);
  uint64_t* qempty = qfull + C::QB;
  uint64_t* kfull = qempty + C::QB;
  uint64_t* kempty = kfull + C::KS;
  uint64_t* sfull = kempty + C::KS;    // [group]: S of the group's tile is in TMEM
  uint64_t* pfull = sfull + 2;         // [group]: P of the group's tile is in TMEM
  uint64_t* odone = pfull + 2;         // [group]: the group's P X~ products so far are done
  uint64_t* ofinal = odone + 2;        // the item's P X~ products are done
  uint64_t* oempty = ofinal + 1;       // both groups have read O of the item
  uint64_t* xbar = oempty + 1;         // both groups have posted (m, l) of the item
  uint64_t* mdrain = xbar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int it0 = p.cta_item_begin[blockIdx.x], it1 = p.cta_item_begin[blockIdx.x + 1];
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::QB; ++i) { mbar_init(&qfull[i], 1); mbar_init(&qempty[i], 1); }
    for (int i = 0; i < C::KS; ++i) { mbar_init(&kfull[i], 1); mbar_init(&kempty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pfull[i], 4);
      mbar_init(&odone[i], 1);
    }
    mbar_init(ofinal, 1);
    mbar_init(oempty, 8);
    mbar_init(xbar, 8);
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
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

  if (warp < 4) {
  regs_dec<kPPRegsLow>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA loader
    if (lane == 0) {
      const uint64_t stream_policy = policy_evict_first();   // X~ is read once per layer
      uint32_t qi = 0, ki = 0;
      bool ok = true;
      for (int it = it0; ok && it < it1; ++it) {
        const AttnItem item = p.items[it];
        const int qb = qi % C::QB;
        if (!(ok = pwait(&qempty[qb], ((qi / C::QB) & 1) ^ 1, abort_flag, p.status))) break;
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
          const int s = ki % C::KS;
          if (!(ok = pwait(&kempty[s], ((ki / C::KS) & 1) ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(&kfull[s], C::kTile);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d_hint(sm + C::oK + s * C::kTile + kb * C::kBlock, &tmK, kb * 64,
                             static_cast<int>(item.key0 + j * 128), &kfull[s], stream_policy);
          ++ki;
        }
      }
      // Let every copy still in flight land before the CTA can exit (after a
      // failed wait the consumers may have stopped waiting for them; on the
      // normal path these phases are complete and the waits return at once).
      for (uint32_t c = ki > C::KS ? ki - C::KS : 0; c < ki; ++c)
        pdrain(&kfull[c % C::KS], (c / C::KS) & 1, 100000000ull);
      for (uint32_t c = qi > C::QB ? qi - C::QB : 0; c < qi; ++c)
        pdrain(&qfull[c % C::QB], (c / C::QB) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Order: S(0), S(1), PV(0), S(2), PV(1), S(3), ... -- S(g + 1) runs while
    // a group computes P(g), and S(g + 2), which overwrites P(g), is issued
    // after PV(g) (MMAs of one thread execute in issue order).
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128);                 // Q K-major, X~ K-major
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);      // P K-major, X~ MN-major
      uint32_t g = 0, qi = 0, ic = 0;
      bool ok = true;
      bool pend = false, pfirst = false, plast = false;
      uint32_t pg = 0, pic = 0;
      auto issue_pv = [&]() -> bool {
        const int b = pg & 1;
        if (!pwait(&pfull[b], (pg >> 1) & 1, abort_flag, p.status)) return false;
        // an item's first product into each group's O overwrites it: the
        // previous item's O must have been read
        if (pfirst && !pwait(oempty, (pic & 1) ^ 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const int s = pg % C::KS;
        const uint32_t vaddr = sbase + C::oK + s * C::kTile;
        // P: keys 2c, 2c + 1 in column c of the group's S columns; 16 keys per MMA
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + C::kO + b * D, tmem + C::kS + b * 128 + kk * 8,
                      sdesc_sw128(vaddr + kk * 2048, C::kBlock, 1024), idO,
                      (!pfirst || kk != 0) ? 1u : 0u);
        mma_commit(&kempty[s]);
        mma_commit(&odone[b]);
        if (plast) mma_commit(ofinal);
        return true;
      };
      for (int it = it0; ok && it < it1; ++it, ++ic) {
        const AttnItem item = p.items[it];
        const int nt = (item.nkeys + 127) >> 7;
        const int qb = qi % C::QB;
        if (!(ok = pwait(&qfull[qb], (qi / C::QB) & 1, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t qaddr = sbase + C::oQ + qb * C::kTile;
        for (int j = 0; j < nt; ++j, ++g) {
          const int b = g & 1, s = g % C::KS;
          if (!(ok = pwait(&kfull[s], (g / C::KS) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t kaddr = sbase + C::oK + s * C::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + C::kS + b * 128,
                        sdesc_sw128(qaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024),
                        sdesc_sw128(kaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024),
                        idS, kk != 0);
          mma_commit(&sfull[b]);
          if (j + 1 == nt) mma_commit(&qempty[qb]);
          if (pend && !(ok = issue_pv())) break;
          pend = true;
          pg = g;
          pfirst = j <= 1;
          plast = j + 1 == nt;
          pic = ic;
        }
        ++qi;
      }
      if (ok && pend) ok = issue_pv();
      mma_commit(mdrain);
      pdrain(mdrain, 0, 500000000ull);
    }
  }
  } else {
    regs_inc<kPPRegsHigh>();
    // ------------------------------------------------------------ softmax groups
    const int b = (warp - 4) >> 2;           // group: tiles g with g % 2 == b
    const int q = warp & 3;                  // TMEM lane quarter
    const int r = q * 32 + lane;             // query row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    float2* xs = reinterpret_cast<float2*>(sm + C::oX);
    uint32_t cb = 0, g = 0, ic = 0;          // group's tiles, CTA's tiles, items
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it, ++ic) {
      const AttnItem item = p.items[it];
      const int nt = (item.nkeys + 127) >> 7;
      float m_run = -INFINITY, l = 0.f;
      bool have = false;
      for (int j = 0; j < nt; ++j, ++g) {
        if ((g & 1u) != static_cast<uint32_t>(b)) continue;
        if (!(ok = pwait_warp(&sfull[b], cb & 1, abort_flag, p.status))) break;
        __syncwarp();
        tc_fence_after();
        // the thread's whole row of the tile's S (128 columns) in one TMEM
        // round trip: the row maximum, then the exponentials, written back as
        // packed bf16 P over the first 64 columns
        const int nvalid = min(128, item.nkeys - j * 128);
        const uint32_t srow = tmem + lane_off + C::kS + b * 128;
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(srow + 32 * c, sv[c]);
        tmem_ld_wait();
        if (nvalid < 128) {     // the item's last tile: keys past its end take no weight
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (c * 32 + k >= nvalid) sv[c][k] = __float_as_uint(-INFINITY);
        }
        float mx;
        {
          float m4[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            m4[c] = fmaxf(__uint_as_float(sv[c][0]), __uint_as_float(sv[c][1]));
#pragma unroll
            for (int k = 2; k < 32; k += 2)
              m4[c] = sx::max3(m4[c], __uint_as_float(sv[c][k]), __uint_as_float(sv[c][k + 1]));
          }
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        const bool resc = mx > m_run + kRescale;          // always on the item's first tile
        const float m_new = resc ? mx : m_run;
        const float corr = resc ? sx::ex2(m_run - m_new) : 1.f;   // 0 from m_run = -inf
        l *= corr;
        const uint64_t negm = sx::f2(-m_new, -m_new);
        uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[32];
#pragma unroll
          for (int k = 0; k < 64; k += 2) {
            const int c = 2 * hh + (k >> 5), e = k & 31;
            const uint64_t x = sx::f2_add(sx::f2(__uint_as_float(sv[c][e]), __uint_as_float(sv[c][e + 1])), negm);
            float x0, x1, p0, p1;
            sx::f2_split(x, x0, x1);
            if (((k >> 1) & 3) < FMA_PAIRS) {
              sx::ex2_fma2(x0, x1, p0, p1);
            } else {
              p0 = sx::ex2(x0);                        // exp2(-inf) = 0
              p1 = sx::ex2(x1);
            }
            ls[(k >> 1) & 3] = sx::f2_add(ls[(k >> 1) & 3], sx::f2(p0, p1));
            pk[k >> 1] = pack_bf16x2(p0, p1);
          }
          // P of keys 64 hh .. 64 hh + 63: columns 32 hh .. 32 hh + 31 (the
          // whole row is already in registers)
          st_tmem32(srow + hh * 32, pk);
        }
        tmem_st_wait();
        {
          const uint64_t s2 = sx::f2_add(sx::f2_add(ls[0], ls[1]), sx::f2_add(ls[2], ls[3]));
          float s0, s1;
          sx::f2_split(s2, s0, s1);
          l += s0 + s1;
        }
        if (have && __any_sync(0xffffffffu, resc)) {
          // O holds the group's sums up to its previous tile: wait for that
          // product, then rescale (rows without a new maximum: corr = 1)
          if (!(ok = pwait_warp(&odone[b], (cb - 1) & 1, abort_flag, p.status))) break;
          __syncwarp();
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tmem + lane_off + C::kO + b * D + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * corr);
            st_tmem32(tmem + lane_off + C::kO + b * D + c * 32, ov);
          }
          tmem_st_wait();
        }
        have = true;
        m_run = m_new;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pfull[b]);
        ++cb;
      }
      if (!ok) break;
      // ---- item done: merge the two groups' (m, l, O) for each row
      xs[b * 128 + r] = make_float2(m_run, l);
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar);
      if (!(ok = pwait_warp(xbar, ic & 1, abort_flag, p.status))) break;
      const float2 o = xs[(b ^ 1) * 128 + r];
      const float mx = fmaxf(m_run, o.x);
      const float f_self = l > 0.f ? sx::ex2(m_run - mx) : 0.f;   // a group without tiles: 0
      const float f_oth = o.y > 0.f ? sx::ex2(o.x - mx) : 0.f;
      const float Ltot = f_self * l + f_oth * o.y;
      const float fA = b == 0 ? f_self : f_oth, fB = b == 0 ? f_oth : f_self;
      if (!(ok = pwait_warp(ofinal, ic & 1, abort_flag, p.status))) break;
      __syncwarp();
      tc_fence_after();
      const int np = p.pair_item_begin[item.pair + 1] - p.pair_item_begin[item.pair];
      const bool valid = r < item.rows;
      // one item covers the pair: c = O / l directly; else the unnormalised partial
      float* dst = np == 1 ? p.cout + (item.qrow0 + r) * D : p.pacc + (item.row_base + r) * D;
      const float scale = np == 1 ? 1.f / Ltot : 1.f;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {       // this group's half of the columns
        const int col = b * (D / 2) + 32 * c;
        uint32_t oa[32], ob[32];
        tmem_ld32(tmem + lane_off + C::kO + col, oa);
        tmem_ld32(tmem + lane_off + C::kO + D + col, ob);
        tmem_ld_wait();
        if (valid) {
          float4* d4 = reinterpret_cast<float4*>(dst + col);
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              // a group that had no tile of this item left stale columns: skip them
              const float a = fA > 0.f ? fA * __uint_as_float(oa[4 * k4 + u]) : 0.f;
              const float bb = fB > 0.f ? fB * __uint_as_float(ob[4 * k4 + u]) : 0.f;
              v[u] = (a + bb) * scale;
            }
            d4[k4] = make_float4(v[0], v[1], v[2], v[3]);
          }
        }
      }
      if (np > 1 && valid) {
        p.pml[(item.row_base + r) * 4 + b] = mx;
        p.pml[(item.row_base + r) * 4 + 2 + b] = Ltot;
      }
      if (np == 1 && valid && p.stats && b == 0) {
        p.stats[(item.qrow0 + r) * 2] = mx;
        p.stats[(item.qrow0 + r) * 2 + 1] = Ltot;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(oempty);
      if (np > 1) {
        // publish this warp's slot, count it; the last arrival merges the slot
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(&p.counters[item.pair * 8 + b * 4 + q], 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == np - 1) {
          __threadfence();
          merge_slot<D>(p, item, b, q, lane);
        }
      }
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

template <int D, int FMA_PAIRS>
int launch_pp(const CUtensorMap& tmQ, const CUtensorMap& tmK, const PPParams& p, int grid,
              cudaStream_t s) {
  using C = PPCfg<D>;
  auto k = attn_pp_kernel<D, FMA_PAIRS>;
  cudaFuncAttributes fa{};
  cudaError_t e = cudaFuncGetAttributes(&fa, k);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("attn_pp attributes: ") + cudaGetErrorString(e));
  // the warpgroups' register split must fit what the block is launched with,
  // or the raising warpgroups would wait for registers that never come
  if (fa.numRegs * kPPThreads < 128 * kPPRegsLow + 256 * kPPRegsHigh)
    return set_error(STCA_ECUDA, "attn_pp: built with too few registers per thread for its register split");
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("attn_pp smem: ") + cudaGetErrorString(e));
  e = launch_pdl(k, dim3(grid), dim3(kPPThreads), C::kSmem, s, tmQ, tmK, p);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("attn_pp launch: ") + cudaGetErrorString(e));
  return STCA_OK;
}

}  // namespace

bool attn_pp_supported(int d) { return d == 64 || d == 128; }

int launch_attn_pp(int d, const CUtensorMap& tmQ, const CUtensorMap& tmK, const AttnItem* items_d,
                   const int32_t* cta_begin_d, const int32_t* pair_item_begin_d, int grid,
                   float* part, int64_t G, float* cout, int* counters, int* status, int stop_tiles,
                   cudaStream_t s, float* stats) {
  PPParams p{};
  p.stats = stats;
  p.items = items_d;
  p.cta_item_begin = cta_begin_d;
  p.pair_item_begin = pair_item_begin_d;
  p.pacc = part;
  p.pml = part + G * d;
  p.cout = cout;
  p.counters = counters;
  p.status = status;
  p.stop_tiles = stop_tiles;
  switch (d) {
    case 64: return launch_pp<64, 2>(tmQ, tmK, p, grid, s);
    case 128: return launch_pp<128, 1>(tmQ, tmK, p, grid, s);
    default: return set_error(STCA_EINVAL, "this attention kernel needs d in {64, 128}");
  }
}

}  // namespace stca
