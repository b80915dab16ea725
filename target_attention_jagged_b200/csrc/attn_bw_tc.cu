// Backward of the merged single-query attention on the tensor cores, d in
// {64, 128}, bf16 handles.
//
// The forward ("Make It Long, Keep It Fast" digest §2.1, Eq. (13)) computes for
// each query row u of request r (target t, head j; the 1/sqrt(d_h) scale is in
// u) the merged row c = P X~_r with P = softmax(S), S = u X~_r^T over the
// request's L_r keys.  Given dC (the loss gradient of c), with request-level
// batching summing a history row's gradient over all its targets ([blog] §2.5):
//   dP = dC X~^T,   delta = rowsum(P * dP) = dC . c,   dS = P * (dP - delta),
//   dU = dS X~,     dX~ = P^T dC + dS^T U.
//
// Before this kernel the host runs: the query rows and dC converted to bf16
// (the rows pre-scaled by log2(e)); the tensor-core forward attention on
// them, which gives c and each row's softmax maximum m (log2 units) and sum l;
// and delta = dC . c per row.  Then P = 2^(S' - m) / l exactly as the forward
// formed it (S' = the log2-scaled scores of the same bf16 rows), with no
// pass over the keys to find m and l.
//
// Work is the forward's stream-K plan: each CTA takes a run of (query tile,
// key tile) units; per key tile of 128 keys:
//   S' = U' X~^T, dP = dC X~^T      tcgen05, M = 128 rows, N = 128 keys, K = d
//   P, dS, dS ln 2                  CUDA cores, one query row per thread; P and
//                                   dS ln 2 to shared memory, dS to TMEM
//   dX~ = P^T dC + (dS ln 2)^T U'   tcgen05, M = 128 keys, N = d, K = 128 rows;
//                                   P and dS ln 2 as MN-major A operands (the
//                                   rows a thread wrote are the K dimension)
//   dU += dS X~                     tcgen05, M = 128 rows, N = d, K = 128 keys,
//                                   dS read from TMEM, X~ as MN-major B
// Rows past the query tile's end and keys past the item's end get P = dS = 0,
// so they add nothing to dX~.  dX~ of the tile is written by four epilogue
// warps (one key per thread); dU of the item by the softmax warps at its end.
// Where a request has more than one query tile, several items add to the same
// dX~ rows (atomic adds into rows the host zeroed); where a query tile's keys
// are split over several items, their dU parts are added atomically the same
// way; otherwise rows are stored.
//
// Warp roles (320 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer,
// warps 2-5 softmax (row per thread), warps 6-9 dX~ epilogue (key per
// thread).  Every wait is bounded; on a failed wait the kernel sets the status
// word, lets copies and products in flight finish, frees TMEM and returns.
#include <cuda.h>

#include <string>

#include "softmax_exp.cuh"
#include "stca_internal.h"
#include "tc_common.cuh"

namespace stca {
namespace {

using namespace tc;

struct BwTcParams {
  const AttnItem* items;
  const int32_t* cta_item_begin;    // gridDim.x + 1
  const int32_t* pair_item_begin;   // pairs + 1
  const int32_t* req_pair_begin;    // R + 1
  const float* stats;               // T h x 2: m (log2 units), l
  const float* delta;               // T h
  float* dU;                        // T h x D
  float* dX;                        // N x D
  int* status;
  int stop_tiles;                   // > 0: the loader stops after this many key tiles (test hook)
};

template <int D>
struct BwCfg {
  static constexpr int KB = D / 64;
  static constexpr uint32_t kBlock = 128u * 128u;          // [128 rows x 64] bf16
  static constexpr uint32_t kTile = KB * kBlock;            // [128 rows x D]
  static constexpr uint32_t kPTile = 2 * kBlock;            // [128 rows x 128 keys]
  static constexpr int KS = D == 128 ? 3 : 6;
  static constexpr uint32_t oQ = 0;                         // U' tile
  static constexpr uint32_t oC = oQ + kTile;                // dC tile
  static constexpr uint32_t oK = oC + kTile;                // X~ stages
  static constexpr uint32_t oP = oK + KS * kTile;           // P
  static constexpr uint32_t oD = oP + kPTile;               // dS ln 2
  static constexpr uint32_t oBar = oD + kPTile;
  // qfull, qempty; kfull, kempty [KS]; sfull, pready, dxfull, dxempty, ufinal, uempty, mdrain
  static constexpr int kBars = 2 + 2 * KS + 7;
  static constexpr uint32_t oMisc = oBar + kBars * 8;
  static constexpr uint32_t kSmem = oMisc + 16;
  static constexpr uint32_t kS = 0;          // S' (then dS, packed bf16, first 64 columns)
  static constexpr uint32_t kDP = 128;       // dP
  static constexpr uint32_t kDX = 256;       // dX~ of the key tile
  static constexpr uint32_t kDU = 256 + D;   // dU of the item
  static_assert(kDU + D <= 512, "TMEM overflow");
  static_assert(kSmem <= 227 * 1024, "shared memory overflow");
};

constexpr int kBwTcThreads = 320;

__device__ __forceinline__ bool bw_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        int* status) {
  if (mbar_wait(bar, parity, abort_flag)) return true;
  *abort_flag = 1;
  atomicOr(status, kStatusAttnTimeout);
  return false;
}

// Waited by every lane of a warp; one answer for the warp.
__device__ __forceinline__ bool bw_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             int* status) {
  const bool ok = bw_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ void bw_drain(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > ns) break;
}

__device__ __forceinline__ void tmem_st16x(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(kBwTcThreads, 1)
attn_bw_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
                  const __grid_constant__ CUtensorMap tmK, const BwTcParams p) {
  using C = BwCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusAttnTimeout);
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* qfull = reinterpret_cast<uint64_t*>(sm + C::oBar);
  uint64_t* qempty = qfull + 1;
  uint64_t* kfull = qempty + 1;
  uint64_t* kempty = kfull + C::KS;
  uint64_t* sfull = kempty + C::KS;    // S' and dP of the tile are in TMEM
  uint64_t* pready = sfull + 1;        // P, dS ln 2 (shared) and dS (TMEM) are written
  uint64_t* dxfull = pready + 1;       // dX~ of the tile is in TMEM
  uint64_t* dxempty = dxfull + 1;      // the epilogue has read it
  uint64_t* ufinal = dxempty + 1;      // dU of the item is complete
  uint64_t* uempty = ufinal + 1;       // the softmax warps have read it
  uint64_t* mdrain = uempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int it0 = p.cta_item_begin[blockIdx.x], it1 = p.cta_item_begin[blockIdx.x + 1];
  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int i = 0; i < C::KS; ++i) { mbar_init(&kfull[i], 1); mbar_init(&kempty[i], 1); }
    mbar_init(sfull, 1);
    mbar_init(pready, 4);
    mbar_init(dxfull, 1);
    mbar_init(dxempty, 4);
    mbar_init(ufinal, 1);
    mbar_init(uempty, 4);
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmC);
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
  pdl_wait();
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loader
    if (lane == 0) {
      uint32_t qi = 0, ki = 0;
      bool ok = true;
      for (int it = it0; ok && it < it1; ++it) {
        const AttnItem item = p.items[it];
        if (!(ok = bw_wait(qempty, (qi & 1) ^ 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(qfull, 2 * C::kTile);
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_2d(sm + C::oQ + kb * C::kBlock, &tmQ, kb * 64, static_cast<int>(item.qrow0), qfull);
          tma_load_2d(sm + C::oC + kb * C::kBlock, &tmC, kb * 64, static_cast<int>(item.qrow0), qfull);
        }
        ++qi;
        const int nt = (item.nkeys + 127) >> 7;
        for (int j = 0; j < nt; ++j) {
          if (p.stop_tiles > 0 && ki >= static_cast<uint32_t>(p.stop_tiles)) {
            *abort_flag = 1;
            atomicOr(p.status, kStatusAttnTimeout);
            ok = false;
            break;
          }
          const int s = ki % C::KS;
          if (!(ok = bw_wait(&kempty[s], ((ki / C::KS) & 1) ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(&kfull[s], C::kTile);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(sm + C::oK + s * C::kTile + kb * C::kBlock, &tmK, kb * 64,
                        static_cast<int>(item.key0 + j * 128), &kfull[s]);
          ++ki;
        }
      }
      for (uint32_t c = ki > C::KS ? ki - C::KS : 0; c < ki; ++c)
        bw_drain(&kfull[c % C::KS], (c / C::KS) & 1, 100000000ull);
      if (qi > 0) bw_drain(qfull, (qi - 1) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128);                // rows x keys, both K-major
      constexpr uint32_t idX = idesc_bf16(128, D, true, true);      // keys x d: A, B MN-major
      constexpr uint32_t idU = idesc_bf16(128, D, false, true);     // rows x d: A (TMEM), B MN-major
      uint32_t g = 0, ic = 0;
      bool ok = true;
      for (int it = it0; ok && it < it1; ++it, ++ic) {
        const AttnItem item = p.items[it];
        const int nt = (item.nkeys + 127) >> 7;
        if (!(ok = bw_wait(qfull, ic & 1, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t qaddr = sbase + C::oQ, caddr = sbase + C::oC;
        for (int j = 0; j < nt; ++j, ++g) {
          const int s = g % C::KS;
          if (!(ok = bw_wait(&kfull[s], (g / C::KS) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t kaddr = sbase + C::oK + s * C::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t kd = sdesc_sw128(kaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024);
            mma_bf16_ss(tmem + C::kS, sdesc_sw128(qaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024),
                        kd, idS, kk != 0);
            mma_bf16_ss(tmem + C::kDP, sdesc_sw128(caddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024),
                        kd, idS, kk != 0);
          }
          mma_commit(sfull);
          if (!(ok = bw_wait(pready, g & 1, abort_flag, p.status))) break;
          if (!(ok = bw_wait(dxempty, (g & 1) ^ 1, abort_flag, p.status))) break;
          if (j == 0 && !(ok = bw_wait(uempty, (ic & 1) ^ 1, abort_flag, p.status))) break;
          tc_fence_after();
          // dX~ = P^T dC + (dS ln 2)^T U': 16 query rows per MMA
          const uint32_t paddr = sbase + C::oP, daddr = sbase + C::oD;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + C::kDX, sdesc_sw128(paddr + kk * 2048, C::kBlock, 1024),
                        sdesc_sw128(caddr + kk * 2048, C::kBlock, 1024), idX, kk != 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + C::kDX, sdesc_sw128(daddr + kk * 2048, C::kBlock, 1024),
                        sdesc_sw128(qaddr + kk * 2048, C::kBlock, 1024), idX, 1u);
          mma_commit(dxfull);
          // dU += dS X~: dS from TMEM, 16 keys (8 packed columns) per MMA
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + C::kDU, tmem + C::kS + kk * 8,
                        sdesc_sw128(kaddr + kk * 2048, C::kBlock, 1024), idU, (j | kk) != 0);
          mma_commit(&kempty[s]);
          if (j + 1 == nt) {
            mma_commit(ufinal);
            mma_commit(qempty);
          }
        }
      }
      mma_commit(mdrain);
      bw_drain(mdrain, 0, 500000000ull);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax: P, dS
    const int q = warp & 3;
    const int r = q * 32 + lane;                // query row of the tile (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t g = 0, ic = 0;
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it, ++ic) {
      const AttnItem item = p.items[it];
      const int nt = (item.nkeys + 127) >> 7;
      const bool rvalid = r < item.rows;
      const int64_t qrow = item.qrow0 + r;
      const float m = rvalid ? p.stats[qrow * 2] : 0.f;
      const float inv_l = rvalid ? 1.f / p.stats[qrow * 2 + 1] : 0.f;
      const float delta = rvalid ? p.delta[qrow] : 0.f;
      for (int j = 0; j < nt; ++j, ++g) {
        if (!(ok = bw_wait_warp(sfull, g & 1, abort_flag, p.status))) break;
        tc_fence_after();
        const int nvalid = rvalid ? min(128, item.nkeys - j * 128) : 0;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {            // 32 keys at a time
          uint32_t sv[32], dv[32];
          tmem_ld32(tmem + lane_off + C::kS + 32 * c, sv);
          tmem_ld32(tmem + lane_off + C::kDP + 32 * c, dv);
          tmem_ld_wait();
          uint32_t pp[16], dd[16], d2[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const int key = 32 * c + k;
            float pv[2], dsv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const bool kv = key + e < nvalid;
              const float pr = kv ? sx::ex2(__uint_as_float(sv[k + e]) - m) * inv_l : 0.f;
              pv[e] = pr;
              dsv[e] = pr * (__uint_as_float(dv[k + e]) - delta);
            }
            pp[k >> 1] = pack_bf16x2(pv[0], pv[1]);
            dd[k >> 1] = pack_bf16x2(dsv[0], dsv[1]);
            d2[k >> 1] = pack_bf16x2(dsv[0] * 0.6931471805599453f, dsv[1] * 0.6931471805599453f);
          }
          // P and dS ln 2: row r of block (32 c) / 64, 16-byte chunks (32 c % 64) / 8 .. + 3
          const uint32_t blk = static_cast<uint32_t>((32 * c) >> 6) * C::kBlock + r * 128;
#pragma unroll
          for (int h4 = 0; h4 < 4; ++h4) {
            const int chunk = ((32 * c) & 63) / 8 + h4;
            const uint32_t off = blk + ((chunk ^ (r & 7)) << 4);
            st_shared_v4(sbase + C::oP + off, pp[4 * h4], pp[4 * h4 + 1], pp[4 * h4 + 2], pp[4 * h4 + 3]);
            st_shared_v4(sbase + C::oD + off, d2[4 * h4], d2[4 * h4 + 1], d2[4 * h4 + 2], d2[4 * h4 + 3]);
          }
          // dS of keys 32 c .. 32 c + 31: packed columns 16 c .. 16 c + 15 (S columns
          // this row has already read)
          tmem_st16x(tmem + lane_off + C::kS + 16 * c, dd);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pready);
      }
      if (!ok) break;
      // item done: its dU rows
      if (!(ok = bw_wait_warp(ufinal, ic & 1, abort_flag, p.status))) break;
      tc_fence_after();
      const int pr = item.pair;
      const bool split = p.pair_item_begin[pr + 1] - p.pair_item_begin[pr] > 1;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + C::kDU + 32 * c, v);
        tmem_ld_wait();
        if (rvalid) {
          float* dst = p.dU + qrow * D + 32 * c;
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            if (split)
              red_add_v4(dst + k, __uint_as_float(v[k]), __uint_as_float(v[k + 1]),
                         __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
            else
              *reinterpret_cast<float4*>(dst + k) =
                  make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]),
                              __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(uempty);
    }
  } else {
    // ------------------------------------------------------------ dX~ epilogue
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t g = 0;
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it) {
      const AttnItem item = p.items[it];
      const int nt = (item.nkeys + 127) >> 7;
      // several query tiles of the request add to the same history rows
      const bool shared_rows = p.req_pair_begin[item.req + 1] - p.req_pair_begin[item.req] > 1;
      for (int j = 0; j < nt; ++j, ++g) {
        if (!(ok = bw_wait_warp(dxfull, g & 1, abort_flag, p.status))) break;
        tc_fence_after();
        const int key = j * 128 + q * 32 + lane;
        const bool kvalid = key < item.nkeys;
        float* dst = p.dX + (item.key0 + key) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + C::kDX + 32 * c, v);
          tmem_ld_wait();
          if (kvalid) {
#pragma unroll
            for (int k = 0; k < 32; k += 4) {
              if (shared_rows)
                red_add_v4(dst + 32 * c + k, __uint_as_float(v[k]), __uint_as_float(v[k + 1]),
                           __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
              else
                *reinterpret_cast<float4*>(dst + 32 * c + k) =
                    make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]),
                                __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dxempty);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// U' = bf16(U log2 e) and dC' = bf16(dC), 8 values per thread.
__global__ void bw_prep_kernel(const float* __restrict__ U, const float* __restrict__ dC,
                               uint16_t* __restrict__ Ub, uint16_t* __restrict__ dCb, int64_t n8) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4* u = reinterpret_cast<const float4*>(U) + 2 * i;
  const float4* c = reinterpret_cast<const float4*>(dC) + 2 * i;
  const float k = 1.4426950408889634f;
  const float4 u0 = u[0], u1 = u[1], c0 = c[0], c1 = c[1];
  reinterpret_cast<uint4*>(Ub)[i] = make_uint4(pack_bf16x2(u0.x * k, u0.y * k), pack_bf16x2(u0.z * k, u0.w * k),
                                               pack_bf16x2(u1.x * k, u1.y * k), pack_bf16x2(u1.z * k, u1.w * k));
  reinterpret_cast<uint4*>(dCb)[i] = make_uint4(pack_bf16x2(c0.x, c0.y), pack_bf16x2(c0.z, c0.w),
                                                pack_bf16x2(c1.x, c1.y), pack_bf16x2(c1.z, c1.w));
}

// delta = dC . c per row: one warp per row.
__global__ void bw_delta_kernel(const float* __restrict__ dC, const float* __restrict__ c,
                                float* __restrict__ delta, int64_t rows, int d) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  float s = 0.f;
  for (int k = lane * 4; k < d; k += 128) {
    const float4 a = *reinterpret_cast<const float4*>(dC + row * d + k);
    const float4 b = *reinterpret_cast<const float4*>(c + row * d + k);
    s = fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, s))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) delta[row] = s;
}

}  // namespace

bool attn_bw_tc_supported(int d) { return d == 64 || d == 128; }

void launch_bw_prep(const float* U, const float* dC, uint16_t* Ub, uint16_t* dCb, int64_t n, cudaStream_t s) {
  const int64_t n8 = n / 8;
  if (n8 > 0) bw_prep_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, s>>>(U, dC, Ub, dCb, n8);
}

void launch_bw_delta(const float* dC, const float* c, float* delta, int64_t rows, int d, cudaStream_t s) {
  if (rows > 0) bw_delta_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(dC, c, delta, rows, d);
}

int launch_attn_bw_tc(int d, const CUtensorMap& tmQ, const CUtensorMap& tmC, const CUtensorMap& tmK,
                      const AttnItem* items, const int32_t* cta_begin, const int32_t* pair_item_begin,
                      const int32_t* req_pair_begin, int grid, const float* stats, const float* delta,
                      float* dU, float* dX, int* status, int stop_tiles, cudaStream_t s) {
  BwTcParams p{};
  p.items = items;
  p.cta_item_begin = cta_begin;
  p.pair_item_begin = pair_item_begin;
  p.req_pair_begin = req_pair_begin;
  p.stats = stats;
  p.delta = delta;
  p.dU = dU;
  p.dX = dX;
  p.status = status;
  p.stop_tiles = stop_tiles;
  auto go = [&](auto kernel, uint32_t smem) -> int {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("attn_bw_tc smem: ") + cudaGetErrorString(e));
    kernel<<<grid, kBwTcThreads, smem, s>>>(tmQ, tmC, tmK, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("attn_bw_tc launch: ") + cudaGetErrorString(e));
    return STCA_OK;
  };
  switch (d) {
    case 64: return go(attn_bw_tc_kernel<64>, BwCfg<64>::kSmem);
    case 128: return go(attn_bw_tc_kernel<128>, BwCfg<128>::kSmem);
    default: return set_error(STCA_EINVAL, "the tensor-core attention backward needs d in {64, 128}");
  }
}

}  // namespace stca
