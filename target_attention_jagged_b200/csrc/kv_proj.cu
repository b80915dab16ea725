// K/V projection of the naive attention form on the tensor cores.
//
// The naive form of the attention ("Make It Long, Keep It Fast" digest §2.1,
// Eq. (12)) projects the keys and values of every history row once per layer,
// K = X~ W_K and V = X~ W_V, and shares them across all of a request's targets
// (the LONGER page's K/V-cache serving idea).  This kernel computes both as
// one product, [K | V] = X~ [W_K | W_V]: N x d bf16 rows times a d x 2d
// matrix, fp32 accumulation, bf16 out (row n of the output is [K_n | V_n]).
//
// It is bound by HBM (2 d bf16 in, 4 d bf16 out per row; 2 d / 3 FLOP/byte
// against a ridge of about 260), so the design keeps the operands moving:
//   * the weight, transposed ([2d outputs x d inputs], K-major, 128-byte
//     swizzle), is cut into slices of 256 outputs; a CTA loads its slice into
//     shared memory once and keeps it (64 KB for d = 128, 128 KB for d = 256);
//   * the CTAs of a slice stride over the 128-row tiles of X~, which TMA
//     streams through a ring of [128 rows x 64] blocks;
//   * one tcgen05.mma per 16 inputs, M = 128 rows, N = 256 outputs, into one
//     of two TMEM accumulators (256 columns each), so the epilogue of one
//     tile overlaps the products of the next;
//   * four epilogue warps read a row each from TMEM and store it as bf16.
// With two slices (d = 256) the two CTAs that read the same rows run side by
// side (CTA c takes slice c % 2), so the second read of a tile comes from L2.
//
// Warp roles (192 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer,
// warps 2-5 epilogue (warp w reads TMEM lane quarter w % 4).  Every wait is a
// bounded mbarrier wait; on a failed wait the kernel sets the status word,
// lets its copies and products in flight finish, frees TMEM and returns.
#include <cuda.h>

#include <string>

#include "stca_internal.h"
#include "tc_common.cuh"

namespace stca {
namespace {

using namespace tc;

constexpr int kKvThreads = 192;
constexpr int kAS = 5;                        // A ring stages ([128 x 64] bf16 each)
constexpr uint32_t kABlock = 128u * 128u;     // 16 KB
constexpr uint32_t kBBlock = 256u * 128u;     // [256 outputs x 64 inputs]: 32 KB

template <int D>
struct KvCfg {
  static constexpr int KB = D / 64;                       // 64-input blocks
  static constexpr int NS = 2 * D / 256;                  // 256-output slices
  static constexpr uint32_t oB = 0;
  static constexpr uint32_t oA = oB + KB * kBBlock;
  static constexpr uint32_t oStg = oA + kAS * kABlock;     // epilogue staging: 4 warps x 32 rows x 72 bf16
  static constexpr uint32_t oBar = oStg + 4 * 32 * 72 * 2;
  // bfull; afull, aempty [kAS]; accfull, accempty [2]; mdrain
  static constexpr int kBars = 1 + 2 * kAS + 4 + 1;
  static constexpr uint32_t oMisc = oBar + kBars * 8;
  static constexpr uint32_t kSmem = oMisc + 16;
  static_assert(kSmem <= 227 * 1024, "shared memory overflow");
};

struct KvParams {
  uint16_t* out;          // N x 2d bf16
  int64_t N;
  int d;
  int* status;
};

__device__ __forceinline__ bool kwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      int* status) {
  if (mbar_wait(bar, parity, abort_flag)) return true;
  *abort_flag = 1;
  atomicOr(status, kStatusKvTimeout);
  return false;
}

__device__ __forceinline__ void kdrain(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > ns) break;
}

template <int D>
__global__ void __launch_bounds__(kKvThreads, 1)
kv_proj_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
               const KvParams p) {
  using C = KvCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {      // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.status, kStatusKvTimeout);
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* bfull = reinterpret_cast<uint64_t*>(sm + C::oBar);
  uint64_t* afull = bfull + 1;
  uint64_t* aempty = afull + kAS;
  uint64_t* accfull = aempty + kAS;
  uint64_t* accempty = accfull + 2;
  uint64_t* mdrain = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slice = blockIdx.x % C::NS;
  const int64_t ntiles = (p.N + 127) / 128;
  const int64_t tile0 = blockIdx.x / C::NS, tstep = gridDim.x / C::NS;
  if (threadIdx.x == 0) {
    mbar_init(bfull, 1);
    for (int i = 0; i < kAS; ++i) { mbar_init(&afull[i], 1); mbar_init(&aempty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 4); }
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
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
      // the weight slice, once: rows 256 slice .. + 255 of W^T, all D inputs
      mbar_arrive_expect_tx(bfull, C::KB * kBBlock);
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_2d(sm + C::oB + kb * kBBlock, &tmW, kb * 64, slice * 256, bfull);
      const uint64_t pol = policy_evict_first();
      uint32_t ai = 0;
      bool ok = true;
      for (int64_t t = tile0; ok && t < ntiles; t += tstep) {
        for (int kb = 0; kb < C::KB; ++kb, ++ai) {
          const int s = ai % kAS;
          if (!(ok = kwait(&aempty[s], ((ai / kAS) & 1) ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(&afull[s], kABlock);
          // with two slices the partner CTA reads the same block: keep it in
          // L2 for that read (normal policy); with one slice it is read once
          if (C::NS == 1)
            tma_load_2d_hint(sm + C::oA + s * kABlock, &tmX, kb * 64, static_cast<int>(t * 128),
                             &afull[s], pol);
          else
            tma_load_2d(sm + C::oA + s * kABlock, &tmX, kb * 64, static_cast<int>(t * 128), &afull[s]);
        }
      }
      // let the copies in flight land before the CTA can exit
      kdrain(bfull, 0, 100000000ull);
      for (uint32_t c = ai > kAS ? ai - kAS : 0; c < ai; ++c)
        kdrain(&afull[c % kAS], (c / kAS) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 256);
      uint32_t ai = 0, u = 0;
      bool ok = kwait(bfull, 0, abort_flag, p.status);
      tc_fence_after();
      for (int64_t t = tile0; ok && t < ntiles; t += tstep, ++u) {
        const int buf = u & 1;
        if (!(ok = kwait(&accempty[buf], ((u >> 1) & 1) ^ 1, abort_flag, p.status))) break;
        tc_fence_after();
        for (int kb = 0; kb < C::KB; ++kb, ++ai) {
          const int s = ai % kAS;
          if (!(ok = kwait(&afull[s], (ai / kAS) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t a = sbase + C::oA + s * kABlock;
          const uint32_t b = sbase + C::oB + kb * kBBlock;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            mma_bf16_ss(tmem + buf * 256, sdesc_sw128(a + k4 * 32, 16, 1024),
                        sdesc_sw128(b + k4 * 32, 16, 1024), idesc, (kb | k4) != 0);
          mma_commit(&aempty[s]);
        }
        if (!ok) break;
        mma_commit(&accfull[buf]);
      }
      mma_commit(mdrain);
      kdrain(mdrain, 0, 500000000ull);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int ld_out = 2 * D;
    uint32_t u = 0;
    for (int64_t t = tile0; t < ntiles; t += tstep, ++u) {
      const int buf = u & 1;
      // one answer for the warp: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, kwait(&accfull[buf], (u >> 1) & 1, abort_flag, p.status))) break;
      __syncwarp();
      tc_fence_after();
      // 64 outputs at a time: each thread stages its row's 64 bf16, then the
      // warp writes its 32 rows coalesced (8 lanes x 16 bytes per row, 4 rows
      // per instruction)
      uint16_t* stg = reinterpret_cast<uint16_t*>(sm + C::oStg) + q * 32 * 72;
      const int64_t row0 = t * 128 + q * 32;
#pragma unroll 1
      for (int c64 = 0; c64 < 4; ++c64) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + buf * 256 + c64 * 64 + h * 32, v);
          tmem_ld_wait();
          uint4* d4 = reinterpret_cast<uint4*>(stg + lane * 72 + 32 * h);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            d4[k] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * k]), __uint_as_float(v[8 * k + 1])),
                               pack_bf16x2(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3])),
                               pack_bf16x2(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5])),
                               pack_bf16x2(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7])));
        }
        __syncwarp();
#pragma unroll
        for (int rr = 0; rr < 32; rr += 4) {
          const int rl = rr + (lane >> 3);
          const int64_t row = row0 + rl;
          if (row < p.N)
            *reinterpret_cast<uint4*>(p.out + row * ld_out + slice * 256 + c64 * 64 + 8 * (lane & 7)) =
                *reinterpret_cast<const uint4*>(stg + rl * 72 + 8 * (lane & 7));
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[buf]);
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

template <int D>
int launch_kv(const CUtensorMap& tmX, const CUtensorMap& tmW, const KvParams& p, int num_sms,
              cudaStream_t s) {
  using C = KvCfg<D>;
  auto k = kv_proj_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("kv_proj smem: ") + cudaGetErrorString(e));
  // every slice gets the same number of CTAs
  const int grid = (num_sms / C::NS) * C::NS;
  e = launch_pdl(k, dim3(grid), dim3(kKvThreads), C::kSmem, s, tmX, tmW, p);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("kv_proj launch: ") + cudaGetErrorString(e));
  return STCA_OK;
}

}  // namespace

bool kv_proj_supported(int d) { return d == 128 || d == 256; }

int launch_kv_proj(int d, const CUtensorMap& tmX, const CUtensorMap& tmW, uint16_t* out, int64_t N,
                   int num_sms, int* status, cudaStream_t s) {
  KvParams p{};
  p.out = out;
  p.N = N;
  p.d = d;
  p.status = status;
  switch (d) {
    case 128: return launch_kv<128>(tmX, tmW, p, num_sms, s);
    case 256: return launch_kv<256>(tmX, tmW, p, num_sms, s);
    default: return set_error(STCA_EINVAL, "the K/V projection kernel needs d in {128, 256}");
  }
}

}  // namespace stca
