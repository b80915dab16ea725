// Tensor-core history encoder: X~(i) = LN_i(((X W_u) * SiLU(X W_g)) W_d) for all
// M layers ("Make It Long, Keep It Fast" digest §2.1, Eqs. (1)-(2); the blog's
// "high-throughput SwiGLU" and "optimised LayerNorm", §3.4).
//
// One persistent CTA per SM walks 128-row tiles of the jagged history buffer
// (the rows of all requests, concatenated: the encoder is row-wise, so request
// boundaries do not matter here).  Per tile it keeps the X tile in shared
// memory for all M layers, and per layer streams the weights in hidden chunks
// of 64 columns:
//   GEMM1  acc1[128 x 128] = X_tile * [W_u | W_g/2]_chunk      (tcgen05, SMEM operands)
//   gate   H[128 x 64]     = u * g' * (1 + tanh(g'))          (g' = g/2; CUDA cores)
//   GEMM2  acc2[128 x d]  += H * W_d,chunk                    (tcgen05, H read from TMEM)
// then LayerNorm on acc2 and a bf16 store of the tile of X~(i).  The hidden
// activations never leave the SM, and never touch shared memory: the gate
// warps write H as packed bf16 back into the TMEM columns of u they have just
// read, and GEMM2 takes its A operand from there.  u * SiLU(g) =
// u * g' * (1 + tanh(g')) with g' = g/2, so W_g is stored pre-halved (exact in
// bf16) and each gate value costs one MUFU tanh.
//
// What paces the kernel is the issue of the MMAs: the tensor pipe queues
// little work ahead, a 128 x 128 x 16 MMA lasts 64 cycles, and each wait on an
// mbarrier or commit costs about as much to the thread that issues it.  So two
// threads in different warps issue the MMAs -- one GEMM1, one GEMM2 -- and the
// waits of each overlap the MMAs of the other.  GEMM1 does not overwrite an
// acc1 buffer before the GEMM2 issuer reports (g2done) that the GEMM2 reading
// its H has completed; acc1 has NB = 3 buffers for d <= 128 (2 for d = 256), so
// that chain spans three chunks.  X, W1 and W2 stream through separate rings,
// each with a single consumer that takes its stages in order (an mbarrier
// parity wait tells apart adjacent phases only).
//
// Warp roles (608 threads): warp 0 loads X, W1 and W2; warp 1 issues GEMM1
// (one thread) and owns the TMEM allocation; warps 2-9 run the gate, warps
// 10-17 the LayerNorm and warp 18 issues GEMM2.  A warp may only touch its own
// 32-lane quarter of TMEM (one row per thread), so two gate warps share each
// quarter and split its columns in halves, and two LayerNorm warps split each
// row.  With d <= 128 the LayerNorm warps copy a tile's acc2 into registers at
// once, so one acc2 buffer serves.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <string>
#include <vector>

#include "stca_internal.h"
#include "tc_common.cuh"

namespace stca {
namespace {

using namespace tc;

struct EncParams {
  int64_t N;                 // history rows of this launch
  int64_t layer_rows;        // rows of one layer's X~ (the whole batch)
  int ntiles;                // ceil(N / 128)
  int M;                     // layers
  int nchunk;                // rd / 64
  uint8_t* xt;               // X~ of this launch's first row; layer i at xt + i * layer_rows * d * 2
  const float* ln_g[16];
  const float* ln_b[16];
  int* status;
};

// Shared-memory pipeline of one configuration: the X tile, a ring of W1
// stages (KPS blocks of W1, [128 rows x 64] bf16 = 16 KB each; a chunk takes
// W1S = KB / KPS of them) and a ring of W2 stages (one [d rows x 64] block per
// chunk).  A W1 stage is released as soon as its GEMM1 completes, a W2 stage
// when its GEMM2 does, a few chunks later; separate rings keep the slow
// release of W2 from holding back the prefetch of W1.
template <int D, int XB, int AB2, int S1, int S2, int NB>
struct EncCfg {
  static constexpr int KB = D / 64;                       // 64-wide K blocks of X
  static constexpr uint32_t kBlock = 128u * 128u;         // [128 rows x 64] bf16
  static constexpr uint32_t kXBytes = KB * kBlock;
  static constexpr int KPS = KB < 2 ? KB : 2;             // W1 blocks per stage
  static constexpr int W1S = KB / KPS;                    // W1 stages per chunk
  static constexpr uint32_t kW1Stage = KPS * kBlock;
  static constexpr uint32_t kW2Stage = D * 128u;          // [D rows x 64]
  static constexpr uint32_t oX = 0;
  static constexpr uint32_t oW1 = oX + XB * kXBytes;
  static constexpr uint32_t oW2 = oW1 + S1 * kW1Stage;
  static constexpr uint32_t oBar = oW2 + S2 * kW2Stage;
  static constexpr int kBars = 2 * S1 + 2 * S2 + 2 * XB + 3 * NB + 2 * AB2 + 1 + 8;
  static constexpr uint32_t oXch = oBar + kBars * 8;      // LayerNorm half-row statistics
  static constexpr uint32_t oMisc = oXch + 2 * 2 * 128 * 8;
  static constexpr uint32_t kSmem = oMisc + 16 + 1024;    // + alignment slack
  static constexpr uint32_t kAcc1 = 0;                    // NB x 128 columns (H aliases u)
  static constexpr uint32_t kAcc2 = NB * 128;             // AB2 x D columns
  static_assert(kAcc2 + AB2 * D <= 512, "TMEM overflow");
  static_assert(kSmem <= 227 * 1024, "shared memory overflow");
  static_assert(S1 >= W1S && S2 >= 2, "too few stages to make progress");
};

constexpr int kEpiWarps = 8;                          // gate: two per TMEM lane quarter
constexpr int kLnWarps = 8;                           // LayerNorm: two per lane quarter
constexpr int kLnWarp0 = 2 + kEpiWarps;
constexpr int kIssuer2Warp = kLnWarp0 + kLnWarps;     // issues GEMM2
constexpr int kEncThreads = 32 * (kIssuer2Warp + 1);

__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      int* status) {
  if (mbar_wait(bar, parity, abort_flag)) return true;
  *abort_flag = 1;
  atomicOr(status, kStatusEncodeTimeout);
  return false;
}

// Wait without the abort shortcut, for at most `ns` (used while draining).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > ns) break;
}

template <int D, int XB, int AB2, int S1, int S2, int NB>
__global__ void __launch_bounds__(kEncThreads, 1)
encode_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW1,
                 const __grid_constant__ CUtensorMap tmW2, const EncParams p) {
  using C = EncCfg<D, XB, AB2, S1, S2, NB>;
  constexpr int W1S = C::W1S;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* full1 = reinterpret_cast<uint64_t*>(sm + C::oBar);
  uint64_t* empty1 = full1 + S1;
  uint64_t* full2 = empty1 + S1;
  uint64_t* empty2 = full2 + S2;
  uint64_t* xfull = empty2 + S2;
  uint64_t* xempty = xfull + XB;
  uint64_t* a1full = xempty + XB;     // GEMM1 of a chunk done
  uint64_t* hfull = a1full + NB;      // its gate written to TMEM (and u, g read)
  uint64_t* g2done = hfull + NB;      // GEMM2 of a chunk done: its H may be overwritten
  uint64_t* a2full = g2done + NB;
  uint64_t* a2empty = a2full + AB2;
  uint64_t* mdrain = a2empty + AB2;   // completion of every MMA, before TMEM is freed
  uint64_t* lnx = mdrain + 1;         // [quarter][unit parity]: both halves' statistics written
  float2* xch = reinterpret_cast<float2*>(sm + C::oXch);   // [unit parity][half][row]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S1; ++i) { mbar_init(&full1[i], 1); mbar_init(&empty1[i], 1); }
    for (int i = 0; i < S2; ++i) { mbar_init(&full2[i], 1); mbar_init(&empty2[i], 1); }
    for (int i = 0; i < XB; ++i) { mbar_init(&xfull[i], 1); mbar_init(&xempty[i], 1); }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&a1full[i], 1);
      mbar_init(&hfull[i], kEpiWarps);
      mbar_init(&g2done[i], 1);
    }
    for (int i = 0; i < AB2; ++i) { mbar_init(&a2full[i], 1); mbar_init(&a2empty[i], kLnWarps); }
    mbar_init(mdrain, 2);
    for (int i = 0; i < 8; ++i) mbar_init(&lnx[i], 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW1);
    prefetch_tmap(&tmW2);
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
  // Dependents may launch now: every CTA of this persistent grid is resident
  // (a dependent launches only once all of them have passed this point), so a
  // dependent CTA takes an SM only when an encoder CTA has left it.  Each
  // dependent waits for this grid's completion before it reads what this grid
  // writes, except the query init after stca_encode_forward, which reads none
  // of it and uses the SMs of the CTAs that finish a round of tiles early.
  pdl_trigger();
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loader
    // Three streams -- X tiles, W1 stages, W2 stages -- each in its own ring.
    // One thread serves them by polling (never blocking on) the ring of each,
    // so the slow release of W2 never holds back X or W1.
    if (lane == 0) {
      const uint64_t x_policy = policy_evict_first();    // X is read once
      const uint64_t w_policy = policy_evict_last();     // weights: re-read by every SM
      const int my_tiles = blockIdx.x < p.ntiles ? (p.ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
      const uint32_t per_tile = static_cast<uint32_t>(p.M * p.nchunk);
      const uint32_t n_chunks = static_cast<uint32_t>(my_tiles) * per_tile;
      uint32_t xi = 0, g1 = 0, g2 = 0;                   // next X tile, W1 stage, W2 stage
      bool ok = true;
      uint64_t t_idle = 0;
      while (xi < static_cast<uint32_t>(my_tiles) || g1 < n_chunks * W1S || g2 < n_chunks) {
        bool progressed = false;
        if (xi < static_cast<uint32_t>(my_tiles) && mbar_test(&xempty[xi % XB], ((xi / XB) & 1) ^ 1)) {
          const int xb = xi % XB;
          const int tile = blockIdx.x + static_cast<int>(xi) * gridDim.x;
          mbar_arrive_expect_tx(&xfull[xb], C::kXBytes);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d_hint(sm + C::oX + xb * C::kXBytes + kb * C::kBlock, &tmX, kb * 64,
                             tile * 128, &xfull[xb], x_policy);
          ++xi;
          progressed = true;
        }
        if (g1 < n_chunks * W1S && mbar_test(&empty1[g1 % S1], ((g1 / S1) & 1) ^ 1)) {
          const int s = g1 % S1;
          const uint32_t k = g1 / W1S, j = g1 % W1S;
          const int w1row = static_cast<int>(k % per_tile) * 128;   // (layer, chunk) row block
          uint8_t* st = sm + C::oW1 + s * C::kW1Stage;
          mbar_arrive_expect_tx(&full1[s], C::kW1Stage);
          for (int kk = 0; kk < C::KPS; ++kk)
            tma_load_2d_hint(st + kk * C::kBlock, &tmW1, (static_cast<int>(j) * C::KPS + kk) * 64,
                             w1row, &full1[s], w_policy);
          ++g1;
          progressed = true;
        }
        if (g2 < n_chunks && mbar_test(&empty2[g2 % S2], ((g2 / S2) & 1) ^ 1)) {
          const int s = g2 % S2;
          const uint32_t lc = g2 % per_tile;                 // layer * nchunk + chunk
          const int layer = static_cast<int>(lc / p.nchunk), c = static_cast<int>(lc % p.nchunk);
          mbar_arrive_expect_tx(&full2[s], C::kW2Stage);
          tma_load_2d_hint(sm + C::oW2 + s * C::kW2Stage, &tmW2, c * 64, layer * D, &full2[s],
                           w_policy);
          ++g2;
          progressed = true;
        }
        if (progressed) {
          t_idle = 0;
        } else {
          const uint64_t now = globaltimer();
          if (t_idle == 0) t_idle = now;
          if (*abort_flag) { ok = false; break; }
          if (now - t_idle > kWaitTimeoutNs) {
            *abort_flag = 1;
            atomicOr(p.status, kStatusEncodeTimeout);
            ok = false;
            break;
          }
        }
      }
      if (!ok) {   // let the copies already issued land before the CTA exits
        for (uint32_t c = g1 > S1 ? g1 - S1 : 0; c < g1; ++c) drain_wait(&full1[c % S1], (c / S1) & 1, 100000000ull);
        for (uint32_t c = g2 > S2 ? g2 - S2 : 0; c < g2; ++c) drain_wait(&full2[c % S2], (c / S2) & 1, 100000000ull);
        for (uint32_t c = xi > XB ? xi - XB : 0; c < xi; ++c) drain_wait(&xfull[c % XB], (c / XB) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ GEMM1 issuer
    if (lane == 0) {
      constexpr uint32_t idesc1 = idesc_bf16(128, 128);
      uint32_t g = 0, xc = 0, cc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.ntiles; tile += gridDim.x, ++xc) {
        const int xb = xc % XB;
        if (!(ok = bwait(&xfull[xb], (xc / XB) & 1, abort_flag, p.status))) break;
        const uint32_t xaddr = sbase + C::oX + xb * C::kXBytes;
        for (int layer = 0; ok && layer < p.M; ++layer) {
          for (int c = 0; ok && c < p.nchunk; ++c, ++cc, g += W1S) {
            // acc1[cc % NB] last held chunk cc-NB, whose H GEMM2 reads from there
            const int b = cc % NB;
            if (cc >= NB && !(ok = bwait(&g2done[b], ((cc / NB) & 1) ^ 1, abort_flag, p.status)))
              break;
            const uint32_t acc1 = tmem + C::kAcc1 + b * 128;
            for (int j = 0; j < W1S; ++j) {
              const uint32_t gs = g + j;
              const int s = gs % S1;
              if (!(ok = bwait(&full1[s], (gs / S1) & 1, abort_flag, p.status))) break;
              tc_fence_after();
              const uint32_t waddr = sbase + C::oW1 + s * C::kW1Stage;
#pragma unroll
              for (int kk = 0; kk < C::KPS; ++kk) {
                const int kb = j * C::KPS + kk;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                  mma_bf16_ss(acc1, sdesc_sw128(xaddr + kb * C::kBlock + k4 * 32, 16, 1024),
                              sdesc_sw128(waddr + kk * C::kBlock + k4 * 32, 16, 1024), idesc1,
                              (kb | k4) != 0);
              }
              mma_commit(&empty1[s]);   // this W1 stage is done with
            }
            if (!ok) break;
            mma_commit(&a1full[b]);
          }
        }
        if (ok) mma_commit(&xempty[xb]);    // the tile's GEMM1s are done with X
      }
      mma_commit(mdrain);
      drain_wait(mdrain, 0, 500000000ull);
    }
  } else if (warp == kIssuer2Warp) {
    // ------------------------------------------------------------ GEMM2 issuer
    if (lane == 0) {
      constexpr uint32_t idesc2 = idesc_bf16(128, D);
      uint32_t hc = 0, uc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.ntiles; tile += gridDim.x) {
        for (int layer = 0; ok && layer < p.M; ++layer, ++uc) {
          const int b2 = uc % AB2;
          const uint32_t acc2 = tmem + C::kAcc2 + b2 * D;
          for (int c = 0; ok && c < p.nchunk; ++c, ++hc) {
            // acc2 += H[hc % NB] * W_d chunk, once the gate has written H
            const int hb = hc % NB;
            if (!(ok = bwait(&hfull[hb], (hc / NB) & 1, abort_flag, p.status))) break;
            if (c == 0 && !(ok = bwait(&a2empty[b2], ((uc / AB2) & 1) ^ 1, abort_flag, p.status)))
              break;
            const int s = hc % S2;
            if (!(ok = bwait(&full2[s], (hc / S2) & 1, abort_flag, p.status))) break;
            tc_fence_after();
            const uint32_t w2addr = sbase + C::oW2 + s * C::kW2Stage;
            // H of the chunk: hidden columns 0..31 in TMEM columns 0..15 of
            // acc1[hb], columns 32..63 in 32..47 (each gate warp's own u columns)
            const uint32_t haddr = tmem + C::kAcc1 + hb * 128;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              mma_bf16_ts(acc2, haddr + (k4 >> 1) * 32 + (k4 & 1) * 8,
                          sdesc_sw128(w2addr + k4 * 32, 16, 1024), idesc2, (c | k4) != 0);
            mma_commit(&empty2[s]);
            mma_commit(&g2done[hb]);
            if (c == p.nchunk - 1) mma_commit(&a2full[b2]);
          }
        }
      }
      mma_commit(mdrain);
      drain_wait(mdrain, 0, 500000000ull);
    }
  } else {
    // ------------------------------------------------------------ gate / LayerNorm
    // A warp may only touch TMEM lanes 32 * (warp % 4) .. +31 (one row per
    // thread).  Gate warps 2-9: two per lane quarter, each on half (`ch`) of the
    // chunk's hidden columns.  LayerNorm warps 10-17: two per lane quarter, on
    // acc2 of the previous (tile, layer) while the gate warps work on the next.
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    bool ok = true;
    if (warp < 2 + kEpiWarps) {
      const int ch = (warp - 2) >> 2;
      uint32_t cc = 0;
      for (int tile = blockIdx.x; ok && tile < p.ntiles; tile += gridDim.x) {
        for (int layer = 0; ok && layer < p.M; ++layer) {
          for (int c = 0; c < p.nchunk; ++c, ++cc) {
            const int b = cc % NB;
            if (!(ok = bwait(&a1full[b], (cc / NB) & 1, abort_flag, p.status))) break;
            __syncwarp();
            tc_fence_after();
            uint32_t packed[16];
            {
              uint32_t u[32], g[32];
              const uint32_t a = tmem + lane_off + C::kAcc1 + b * 128 + ch * 32;
              tmem_ld32(a, u);
              tmem_ld32(a + 64, g);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float g0 = __uint_as_float(g[2 * j]), g1 = __uint_as_float(g[2 * j + 1]);
                const float p0 = __uint_as_float(u[2 * j]) * g0;
                const float p1 = __uint_as_float(u[2 * j + 1]) * g1;
                packed[j] = pack_bf16x2(fmaf(p0, tanh_approx(g0), p0), fmaf(p1, tanh_approx(g1), p1));
              }
            }
            // H (bf16 pairs) over this warp's own u columns, read above
            tmem_st16(tmem + lane_off + C::kAcc1 + b * 128 + ch * 32, packed);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&hfull[b]);
          }
        }
      }
    } else {
      // LayerNorm warps 10-17: two per lane quarter; half hh of a pair takes
      // columns [hh D/2, (hh + 1) D/2) of the quarter's rows.  Each half reduces
      // its values to (mean, M2); the pair swaps them through shared memory and
      // merges them (the pairwise update of Chan, Golub and LeVeque) into the
      // row's mean and variance.  With d <= 128 a half row fits in registers,
      // so acc2 is handed back to the MMAs right after one TMEM read.
      constexpr int DH = D / 2;
      constexpr bool kInRegs = DH <= 64;
      const int hh = (warp - kLnWarp0) >> 2;
      const uint64_t out_policy = policy_evict_first();      // X~ is written once here
      uint32_t uc = 0;
      for (int tile = blockIdx.x; ok && tile < p.ntiles; tile += gridDim.x) {
        const int64_t row = static_cast<int64_t>(tile) * 128 + row_in_tile;
        for (int layer = 0; ok && layer < p.M; ++layer, ++uc) {
          const int b2 = uc % AB2;
          if (!(ok = bwait(&a2full[b2], (uc / AB2) & 1, abort_flag, p.status))) break;
          __syncwarp();
          tc_fence_after();
          const uint32_t arow = tmem + lane_off + C::kAcc2 + b2 * D + hh * DH;
          uint32_t rv[kInRegs ? DH / 32 : 1][32];
          float mean_h, m2_h;
          if constexpr (kInRegs) {
#pragma unroll
            for (int cb = 0; cb < DH / 32; ++cb) tmem_ld32(arow + cb * 32, rv[cb]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a2empty[b2]);    // acc2 may be overwritten now
            float s = 0.f;
#pragma unroll
            for (int cb = 0; cb < DH / 32; ++cb)
#pragma unroll
              for (int j = 0; j < 32; ++j) s += __uint_as_float(rv[cb][j]);
            mean_h = s * (1.0f / DH);
            float m2 = 0.f;
#pragma unroll
            for (int cb = 0; cb < DH / 32; ++cb)
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float x = __uint_as_float(rv[cb][j]) - mean_h;
                m2 = fmaf(x, x, m2);
              }
            m2_h = m2;
          } else {
            // sums shifted by the half row's first value against cancellation
            float shift = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll 1
            for (int cb = 0; cb < DH / 32; ++cb) {
              tmem_ld32(arow + cb * 32, rv[0]);
              tmem_ld_wait();
              if (cb == 0) shift = __uint_as_float(rv[0][0]);
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float x = __uint_as_float(rv[0][j]) - shift;
                s1 += x;
                s2 = fmaf(x, x, s2);
              }
            }
            const float m1 = s1 * (1.0f / DH);
            mean_h = shift + m1;
            m2_h = fmaxf(s2 - s1 * m1, 0.f);
          }
          // swap half statistics with the partner warp (same rows, other half)
          float2* xs = xch + (uc & 1) * 256;
          xs[hh * 128 + row_in_tile] = make_float2(mean_h, m2_h);
          __syncwarp();
          uint64_t* xbar = &lnx[q * 2 + (uc & 1)];
          if (lane == 0) mbar_arrive(xbar);
          if (!(ok = bwait(xbar, (uc >> 1) & 1, abort_flag, p.status))) break;
          const float2 other = xs[(hh ^ 1) * 128 + row_in_tile];
          const float dm = other.x - mean_h;
          const float mean = 0.5f * (mean_h + other.x);
          const float var = fmaxf((m2_h + other.y + dm * dm * (0.5f * DH)) * (1.0f / D), 0.f);
          const float rstd = rsqrtf(var + 1e-5f);
          const float4* gam = reinterpret_cast<const float4*>(p.ln_g[layer] + hh * DH);
          const float4* bet = reinterpret_cast<const float4*>(p.ln_b[layer] + hh * DH);
          uint8_t* orow = p.xt + (static_cast<int64_t>(layer) * p.layer_rows + row) * (D * 2) + hh * DH * 2;
#pragma unroll
          for (int cb = 0; cb < DH / 32; ++cb) {
            const uint32_t* vv;
            if constexpr (kInRegs) {
              vv = rv[cb];
            } else {
              tmem_ld32(arow + cb * 32, rv[0]);
              tmem_ld_wait();
              vv = rv[0];
            }
            uint32_t o[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 gg = __ldg(gam + cb * 8 + j);
              const float4 bb = __ldg(bet + cb * 8 + j);
              const float y0 = (__uint_as_float(vv[4 * j]) - mean) * rstd * gg.x + bb.x;
              const float y1 = (__uint_as_float(vv[4 * j + 1]) - mean) * rstd * gg.y + bb.y;
              const float y2 = (__uint_as_float(vv[4 * j + 2]) - mean) * rstd * gg.z + bb.z;
              const float y3 = (__uint_as_float(vv[4 * j + 3]) - mean) * rstd * gg.w + bb.w;
              o[2 * j] = pack_bf16x2(y0, y1);
              o[2 * j + 1] = pack_bf16x2(y2, y3);
            }
            if (row < p.N) {
              uint4* dst = reinterpret_cast<uint4*>(orow + cb * 64);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                st_global_v4_hint(dst + k, make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]),
                                  out_policy);
            }
          }
          if constexpr (!kInRegs) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a2empty[b2]);
          }
        }
      }
    }
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    else
      cudaGetLastError();
  }
  return fn;
}

template <int D, int XB, int AB2, int S1, int S2, int NB>
int launch_cfg(stca_handle* H, const CUtensorMap& tmX, const EncParams& p, cudaStream_t s) {
  using C = EncCfg<D, XB, AB2, S1, S2, NB>;
  auto k = encode_tc_kernel<D, XB, AB2, S1, S2, NB>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("encode_tc smem: ") + cudaGetErrorString(e));
  const int grid = std::min(p.ntiles, H->num_sms);
  e = launch_pdl(k, dim3(grid), dim3(kEncThreads), C::kSmem, s, tmX, H->tmW1, H->tmW2, p);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("encode_tc launch: ") + cudaGetErrorString(e));
  return STCA_OK;
}

}  // namespace

int make_tmap_f32_3d(CUtensorMap* m, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                     const uint32_t box[3]) {
  auto fn = encode_fn();
  if (!fn) return set_error(STCA_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides[0], strides[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), d, st, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(STCA_ECUDA, "cuTensorMapEncodeTiled (fp32, 3-d) failed (" + std::to_string(int(r)) + ")");
  return STCA_OK;
}

int make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                      uint32_t box_inner, uint32_t box_outer) {
  return make_tmap_bf16_2d_strided(m, base, inner, outer, inner * 2, box_inner, box_outer);
}

int make_tmap_bf16_2d_strided(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return set_error(STCA_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(STCA_ECUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(int(r)) + ")");
  return STCA_OK;
}

bool encode_tc_supported(int d, int rd) {
  return (d == 64 || d == 128 || d == 256) && rd % 64 == 0 && rd >= 64;
}

// Lay out the tensor-core operands of all layers and build their tensor maps.
//   W1T: rows (layer, chunk c, j): j < 64 -> column c*64+j of W_u; j >= 64 ->
//        column c*64+j-64 of W_g times 1/2; each row holds d values (K-major).
//   W2T: rows (layer, n) = column n of W_d, rd values each (K-major).
int encode_tc_setup(stca_handle* H, const std::vector<const float*>& Wu,
                    const std::vector<const float*>& Wg, const std::vector<const float*>& Wd) {
  const int d = H->d, rd = H->rd, M = H->M, nchunk = rd / 64;
  const size_t w1_rows = static_cast<size_t>(M) * nchunk * 128;
  const size_t w2_rows = static_cast<size_t>(M) * d;
  std::vector<uint16_t> host(w1_rows * d + w2_rows * rd);
  auto bf = [](float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return static_cast<uint16_t>(u >> 16);   // values are bf16-exact already
  };
  for (int i = 0; i < M; ++i)
    for (int c = 0; c < nchunk; ++c)
      for (int j = 0; j < 128; ++j) {
        uint16_t* dst = host.data() + ((static_cast<size_t>(i) * nchunk + c) * 128 + j) * d;
        const int col = c * 64 + (j & 63);
        for (int k = 0; k < d; ++k)
          dst[k] = j < 64 ? bf(Wu[i][static_cast<size_t>(k) * rd + col])
                          : bf(0.5f * Wg[i][static_cast<size_t>(k) * rd + col]);
      }
  uint16_t* w2 = host.data() + w1_rows * d;
  for (int i = 0; i < M; ++i)
    for (int n = 0; n < d; ++n)
      for (int k = 0; k < rd; ++k)
        w2[(static_cast<size_t>(i) * d + n) * rd + k] = bf(Wd[i][static_cast<size_t>(k) * d + n]);
  if (cudaMalloc(&H->wtc, host.size() * 2) != cudaSuccess) {
    cudaGetLastError();
    return set_error(STCA_ENOMEM, "tensor-core weight allocation failed");
  }
  STCA_CUDA_TRY(cudaMemcpy(H->wtc, host.data(), host.size() * 2, cudaMemcpyHostToDevice));
  if (int rc = make_tmap_bf16_2d(&H->tmW1, H->wtc, d, w1_rows, 64, 128)) return rc;
  if (int rc = make_tmap_bf16_2d(&H->tmW2, H->wtc + w1_rows * d, rd, w2_rows, 64, d)) return rc;
  H->tc_encode_ready = true;
  return STCA_OK;
}

int launch_encode_tc(stca_handle* H, const void* X, int64_t N, cudaStream_t s, int64_t row0) {
  CUtensorMap tmX;
  if (int rc = make_tmap_bf16_2d(&tmX, X, H->d, N, 64, 128)) return rc;
  EncParams p{};
  p.N = N;
  p.layer_rows = H->N;
  p.ntiles = static_cast<int>((N + 127) / 128);
  p.M = H->M;
  p.nchunk = H->rd / 64;
  p.xt = static_cast<uint8_t*>(H->xt) + row0 * H->d * 2;
  for (int i = 0; i < H->M; ++i) {
    p.ln_g[i] = H->L32[i].ln_g;
    p.ln_b[i] = H->L32[i].ln_b;
  }
  p.status = H->status_d;
  switch (H->d) {
    case 64: return launch_cfg<64, 2, 2, 6, 8, 3>(H, tmX, p, s);
    case 128: return launch_cfg<128, 2, 1, 3, 3, 3>(H, tmX, p, s);
    case 256: return launch_cfg<256, 1, 1, 2, 2, 2>(H, tmX, p, s);
    default: return set_error(STCA_EINVAL, "tensor-core encoder needs d in {64, 128, 256}");
  }
}

}  // namespace stca
