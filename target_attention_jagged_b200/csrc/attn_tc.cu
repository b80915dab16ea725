// Tensor-core split-L single-query attention over the jagged encoded history.
//
// For request r the T_r * h query rows are u_j of every target t and head j,
// scaled by log2(e) / sqrt(d_h) ("Make It Long, Keep It Fast" digest §2.1,
// Eq. (13); the blog's reordered single-query attention, §2.4).  They all
// attend to the same L_r keys X~_r, so one pass over X~_r serves every target:
//   S = U_tile X~_tile^T         (tcgen05, M = 128 query rows, N = 128 keys, K = d)
//   P = exp2(S - m), online max / sum per row (CUDA cores, one row per thread)
//   O += P X~_tile               (tcgen05, M = 128, N = d, K = 128 keys)
// The same shared-memory copy of each X~ tile is the K-major B operand of the
// first MMA and the MN-major B operand of the second.  Work is cut stream-K
// style: every CTA gets an equal run of (query tile, key tile) units in
// (request, query tile, key) order, so ragged lengths do not unbalance the SMs;
// each maximal run inside one (request, query tile) pair is an item that
// writes an unnormalised partial (O, m, l) for the split combine.
//
// The running max is rescaled lazily: O and l are corrected only when a row's
// max grows by more than 8 (log2 units); otherwise P uses the stale max and
// stays below 2^8, well inside bf16 and fp32 range.
//
// Warp roles (192 threads): warp 0 TMA, warp 1 MMA issue + TMEM owner, warps
// 2-5 softmax / correction / partial store, one query row per thread.
#include <cuda.h>

#include <algorithm>
#include <string>
#include <vector>

#include "stca_internal.h"
#include "tc_common.cuh"

namespace stca {
namespace {

using namespace tc;

struct AttnParams {
  const AttnItem* items;
  const int32_t* cta_item_begin;   // gridDim.x + 1
  float* pacc;                     // G x d
  float* pm;                       // G
  float* pl;                       // G
  int* status;
};

template <int D, int QB, int KS, int PB>
struct AttnCfg {
  static constexpr int KB = D / 64;
  static constexpr uint32_t kBlock = 128u * 128u;       // [128 rows x 64] bf16
  static constexpr uint32_t kTile = KB * kBlock;         // [128 rows x D]
  static constexpr uint32_t kPBytes = 2 * kBlock;        // [128 rows x 128 keys]
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + QB * kTile;
  static constexpr uint32_t oP = oK + KS * kTile;
  static constexpr uint32_t oBar = oP + PB * kPBytes;
  static constexpr int kBars = 2 * QB + 2 * KS + 4 + 2 * PB + 3 + 1;
  static constexpr uint32_t oMisc = oBar + kBars * 8;
  static constexpr uint32_t kSmem = oMisc + 16 + 1024;
  static constexpr uint32_t kS = 0;        // 2 x 128 TMEM columns of scores
  static constexpr uint32_t kO = 256;      // D columns of the output accumulator
  static_assert(kO + D <= 512, "TMEM overflow");
  static_assert(kSmem <= 227 * 1024, "shared memory overflow");
};

constexpr int kAttnThreads = 192;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

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

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

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


template <int D, int QB, int KS, int PB>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const AttnParams p) {
  using C = AttnCfg<D, QB, KS, PB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int it0 = p.cta_item_begin[blockIdx.x], it1 = p.cta_item_begin[blockIdx.x + 1];
  if (threadIdx.x == 0) {
    for (int i = 0; i < QB; ++i) { mbar_init(&qfull[i], 1); mbar_init(&qempty[i], 1); }
    for (int i = 0; i < KS; ++i) { mbar_init(&kfull[i], 1); mbar_init(&kempty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&sfull[i], 1); mbar_init(&sempty[i], 4); }
    for (int i = 0; i < PB; ++i) { mbar_init(&pfull[i], 4); mbar_init(&pempty[i], 1); }
    mbar_init(odone, 1);
    mbar_init(ofinal, 1);
    mbar_init(oempty, 4);
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
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t stream_policy = policy_evict_first();   // X~ is read once per layer
      uint32_t qi = 0, ki = 0;
      bool ok = true;
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
          const int s = ki % KS;
          if (!(ok = bwait(&kempty[s], ((ki / KS) & 1) ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(&kfull[s], C::kTile);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d_hint(sm + C::oK + s * C::kTile + kb * C::kBlock, &tmK, kb * 64,
                             static_cast<int>(item.key0 + j * 128), &kfull[s], stream_policy);
          ++ki;
        }
      }
      if (!ok) {
        for (uint32_t c = ki > KS ? ki - KS : 0; c < ki; ++c) drain_wait(&kfull[c % KS], (c / KS) & 1, 100000000ull);
        for (uint32_t c = qi > QB ? qi - QB : 0; c < qi; ++c) drain_wait(&qfull[c % QB], (c / QB) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128);                 // Q K-major, X~ K-major
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);      // P K-major, X~ MN-major
      uint32_t qi = 0, ki = 0, sc = 0, pc = 0, ic = 0;
      bool ok = true;
      for (int it = it0; ok && it < it1; ++it, ++ic) {
        const AttnItem item = p.items[it];
        const int nt = (item.nkeys + 127) >> 7;
        const int qb = qi % QB;
        if (!(ok = bwait(&qfull[qb], (qi / QB) & 1, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t qaddr = sbase + C::oQ + qb * C::kTile;
        uint32_t stage_prev = 0;
        // S(0)
        auto issue_s = [&](uint32_t& stage_out) -> bool {
          const int sb = sc & 1;
          if (!bwait(&sempty[sb], ((sc >> 1) & 1) ^ 1, abort_flag, p.status)) return false;
          tc_fence_after();
          const int s = ki % KS;
          if (!bwait(&kfull[s], (ki / KS) & 1, abort_flag, p.status)) return false;
          tc_fence_after();
          const uint32_t kaddr = sbase + C::oK + s * C::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + C::kS + sb * 128,
                        sdesc_sw128(qaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024),
                        sdesc_sw128(kaddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024),
                        idS, kk != 0);
          mma_commit(&sfull[sb]);
          stage_out = s;
          ++sc;
          ++ki;
          return true;
        };
        if (!(ok = issue_s(stage_prev))) break;
        for (int j = 0; ok && j < nt; ++j) {
          const uint32_t stage_j = stage_prev;
          if (j + 1 < nt) {
            if (!(ok = issue_s(stage_prev))) break;
          }
          if (j + 1 == nt) mma_commit(&qempty[qb]);
          const int pb = pc % PB;
          if (!(ok = bwait(&pfull[pb], (pc / PB) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          if (j == 0) {
            if (!(ok = bwait(oempty, (ic & 1) ^ 1, abort_flag, p.status))) break;
            tc_fence_after();
          }
          const uint32_t paddr = sbase + C::oP + pb * C::kPBytes;
          const uint32_t vaddr = sbase + C::oK + stage_j * C::kTile;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // 16 keys per MMA
            mma_bf16_ss(tmem + C::kO,
                        sdesc_sw128(paddr + (kk >> 2) * C::kBlock + (kk & 3) * 32, 16, 1024),
                        sdesc_sw128(vaddr + kk * 2048, C::kBlock, 1024), idO,
                        (j | kk) != 0);
          mma_commit(&kempty[stage_j]);
          mma_commit(&pempty[pb]);
          mma_commit(odone);
          ++pc;
        }
        if (!ok) break;
        mma_commit(ofinal);
        ++qi;
      }
      mma_commit(mdrain);
      drain_wait(mdrain, 0, 500000000ull);
    }
  } else {
    // ------------------------------------------------------------ softmax + partials
    const int q = warp & 3;
    const int r = q * 32 + lane;              // query row of the tile (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t sc = 0, pc = 0, ic = 0;
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it, ++ic) {
      const AttnItem item = p.items[it];
      const int nt = (item.nkeys + 127) >> 7;
      float m_used = -1e30f, l = 0.f;
      for (int j = 0; j < nt; ++j) {
        const int sb = sc & 1;
        if (!(ok = bwait(&sfull[sb], (sc >> 1) & 1, abort_flag, p.status))) break;
        __syncwarp();
        tc_fence_after();
        uint32_t sv[4][32];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) tmem_ld32(tmem + lane_off + C::kS + sb * 128 + cb * 32, sv[cb]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
        ++sc;
        const int nvalid = min(128, item.nkeys - j * 128);
        if (nvalid < 128) {   // the request's last tile: keys past its end take no weight
#pragma unroll
          for (int cb = 0; cb < 4; ++cb)
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (cb * 32 + k >= nvalid) sv[cb][k] = __float_as_uint(-INFINITY);
        }
        float mx = -INFINITY;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
#pragma unroll
          for (int k = 0; k < 32; ++k) mx = fmaxf(mx, __uint_as_float(sv[cb][k]));
        const bool resc = mx > m_used + kRescaleThreshold;
        const float m_new = resc ? mx : m_used;
        const float corr = resc ? ex2(m_used - m_new) : 1.f;
        l *= corr;
        m_used = m_new;
        uint32_t pk[64];
        float lsum = 0.f;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float p0 = ex2(__uint_as_float(sv[cb][k]) - m_new);      // exp2(-inf) = 0
            const float p1 = ex2(__uint_as_float(sv[cb][k + 1]) - m_new);
            lsum += p0 + p1;
            pk[(cb * 32 + k) >> 1] = pack_bf16x2(p0, p1);
          }
        l += lsum;
        const int pb = pc % PB;
        if (!(ok = bwait(&pempty[pb], ((pc / PB) & 1) ^ 1, abort_flag, p.status))) break;
        __syncwarp();
        // P row: keys 0..63 in block 0, 64..127 in block 1, K-major, 128-B swizzle
        const uint32_t prow = sbase + C::oP + pb * C::kPBytes + r * 128;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t blk = (c >> 3) * C::kBlock;
          st_shared_v4(prow + blk + (((c & 7) ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1],
                       pk[4 * c + 2], pk[4 * c + 3]);
        }
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
          // O holds the rows' sums up to tile j-1: wait for that MMA, then rescale
          if (!(ok = bwait(odone, (pc - 1) & 1, abort_flag, p.status))) break;
          __syncwarp();
          tc_fence_after();
#pragma unroll 1
          for (int cb = 0; cb < D / 32; ++cb) {
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
      // item done: store the unnormalised partial of the valid rows
      if (!(ok = bwait(ofinal, ic & 1, abort_flag, p.status))) break;
      __syncwarp();
      tc_fence_after();
      const bool valid = r < item.rows;
      const int64_t g = item.row_base + r;
      float* dst = p.pacc + g * D;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
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
      if (valid) {
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int QB, int KS, int PB>
int launch_cfg(stca_handle* H, const CUtensorMap& tmQ, const CUtensorMap& tmK, const AttnParams& p,
               int grid, cudaStream_t s) {
  using C = AttnCfg<D, QB, KS, PB>;
  auto k = attn_tc_kernel<D, QB, KS, PB>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("attn_tc smem: ") + cudaGetErrorString(e));
  k<<<grid, kAttnThreads, C::kSmem, s>>>(tmQ, tmK, p);
  return STCA_OK;
}

}  // namespace

bool attn_tc_supported(int d) { return d == 64 || d == 128 || d == 256; }

int launch_attn_tc(stca_handle* H, int layer, const AttnItem* items_d, const int32_t* cta_begin_d,
                   int grid, cudaStream_t s) {
  AttnParams p{};
  p.items = items_d;
  p.cta_item_begin = cta_begin_d;
  const int64_t G = H->last_G;
  p.pacc = H->part;
  p.pm = H->part + G * H->d;
  p.pl = p.pm + G;
  p.status = H->status_d;
  const CUtensorMap& tmK = H->tmXt[layer];
  switch (H->d) {
    case 64: return launch_cfg<64, 2, 6, 2>(H, H->tmU, tmK, p, grid, s);
    case 128: return launch_cfg<128, 2, 3, 2>(H, H->tmU, tmK, p, grid, s);
    case 256: return launch_cfg<256, 1, 2, 1>(H, H->tmU, tmK, p, grid, s);
    default: return set_error(STCA_EINVAL, "tensor-core attention needs d in {64, 128, 256}");
  }
}

// The same kernel with every buffer given explicitly (no handle state).
int launch_attn_tc_ws(int d, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                      const AttnItem* items_d, const int32_t* cta_begin_d, int grid, float* part,
                      int64_t G, int* status, cudaStream_t s) {
  AttnParams p{};
  p.items = items_d;
  p.cta_item_begin = cta_begin_d;
  p.pacc = part;
  p.pm = part + G * d;
  p.pl = p.pm + G;
  p.status = status;
  switch (d) {
    case 64: return launch_cfg<64, 2, 6, 2>(nullptr, tmQ, tmK, p, grid, s);
    case 128: return launch_cfg<128, 2, 3, 2>(nullptr, tmQ, tmK, p, grid, s);
    case 256: return launch_cfg<256, 1, 2, 1>(nullptr, tmQ, tmK, p, grid, s);
    default: return set_error(STCA_EINVAL, "tensor-core attention needs d in {64, 128, 256}");
  }
}

}  // namespace stca
