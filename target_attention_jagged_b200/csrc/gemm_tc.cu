// Tensor-core GEMM with TF32 operands and fp32 accumulation, for the backward
// products of bf16 handles (the products of the history encoding's backward,
// the attention projections' and the fusion blocks'; "Make It Long, Keep It
// Fast" digest §2.1, Eqs. (1)-(3), (6), (7), (9), (13)).
//
// Row-major C (m x n) = alpha op(A) op(B) + beta C, where op(A) is m x k and
// op(B) is k x n; A or B may be stored transposed.  Each operand reaches
// shared memory by TMA in the layout the tensor core reads directly:
//   * op(A) = A (row-major m x k, k contiguous): K-major A, one [128 x 32] box;
//   * op(A) = A^T (A stored k x m, m contiguous): MN-major A, four [32 k x 32 m]
//     boxes side by side (a 128-byte row holds 32 of the 128 m values);
//   * op(B) = B^T (B stored n x k, k contiguous): K-major B, one [BN x 32] box;
//   * op(B) = B (B stored k x n, n contiguous): MN-major B, BN / 32 boxes.
// One tcgen05.mma.kind::tf32 is M = 128 x N = BN x K = 8; a stage holds K = 32.
// Partial tiles are zero-filled by TMA.  A batch of products is the third
// tensor-map dimension.  When the output has few tiles and K is long (the
// weight gradients, whose K is every history row), K is split over CTAs and
// each adds its part to C atomically (C pre-scaled by the host).
//
// Warp roles (192 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer,
// warps 2-5 epilogue (warp w reads TMEM lane quarter w % 4, one output row per
// thread).  Waits are bounded; a failed wait sets the status word, in-flight
// copies and products are let finish and TMEM is freed.
#include <cuda.h>

#include <algorithm>
#include <string>

#include "stca_internal.h"
#include "tc_common.cuh"

namespace stca {
namespace {

using namespace tc;

constexpr int kGemmThreads = 192;
constexpr int kGemmStages = 6;
constexpr uint32_t kAStage = 128u * 128u;      // [128 x 32] fp32

struct GemmArgs {
  int64_t m, n, k;
  int tiles_m, tiles_n, ksplit;
  int64_t k_per_split;          // multiple of 32
  float* C;
  int64_t ldc, sC;
  float alpha, beta;
  int atomic;                   // 1: add alpha acc to C atomically (C pre-scaled)
  int a_bmid, b_bmid;           // the batch is the tensor map's middle dimension (see below)
  int* status;
};

__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                          // D format: f32
         | (2u << 7)                        // A format: tf32
         | (2u << 10)                       // B format: tf32
         | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (mbar_wait(bar, parity, abort_flag)) return true;
  *abort_flag = 1;
  atomicOr(status, kStatusStepTimeout);
  return false;
}

__device__ __forceinline__ void gdrain(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > ns) break;
}

template <int BN, bool AMN, bool BMN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tf32_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmArgs g) {
  constexpr uint32_t kBStage = BN * 128u;
  constexpr uint32_t kStage = kAStage + kBStage;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(g.status, kStatusStepTimeout);
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kGemmStages * kStage);
  uint64_t* empty = full + kGemmStages;
  uint64_t* accfull = empty + kGemmStages;
  uint64_t* mdrain = accfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdrain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int u = blockIdx.x;
  const int ks = u % g.ksplit; u /= g.ksplit;
  const int tn = u % g.tiles_n; u /= g.tiles_n;
  const int tm = u % g.tiles_m;
  const int b = u / g.tiles_m;
  const int64_t m0 = static_cast<int64_t>(tm) * 128, n0 = static_cast<int64_t>(tn) * BN;
  const int64_t k0 = ks * g.k_per_split, k1 = min(g.k, k0 + g.k_per_split);
  const int nst = static_cast<int>((k1 - k0 + 31) / 32);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(accfull, 1);
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  constexpr uint32_t kCols = BN < 32 ? 32 : BN;
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int st = 0;
      for (; ok && st < nst; ++st) {
        const int s = st % kGemmStages;
        if (!(ok = gwait(&empty[s], ((st / kGemmStages) & 1) ^ 1, abort_flag, g.status))) break;
        mbar_arrive_expect_tx(&full[s], kStage);
        uint8_t* a = sm + s * kStage;
        uint8_t* bb = a + kAStage;
        const int kk = static_cast<int>(k0 + 32 * st);
        // (inner, outer) coordinates, with the batch index in the middle or last
        auto ld = [&](void* dst, const CUtensorMap* map, int x, int y, int bmid) {
          if (bmid) tma_load_3d(dst, map, x, b, y, &full[s]);
          else tma_load_3d(dst, map, x, y, b, &full[s]);
        };
        if constexpr (AMN) {
          for (int i = 0; i < 4; ++i) ld(a + i * 4096, &tmA, static_cast<int>(m0) + 32 * i, kk, g.a_bmid);
        } else {
          ld(a, &tmA, kk, static_cast<int>(m0), g.a_bmid);
        }
        if constexpr (BMN) {
          for (int i = 0; i < BN / 32; ++i) ld(bb + i * 4096, &tmB, static_cast<int>(n0) + 32 * i, kk, g.b_bmid);
        } else {
          ld(bb, &tmB, kk, static_cast<int>(n0), g.b_bmid);
        }
      }
      for (int c = st > kGemmStages ? st - kGemmStages : 0; c < st; ++c)
        gdrain(&full[c % kGemmStages], (c / kGemmStages) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32(128, BN, AMN, BMN);
      bool ok = true;
      for (int st = 0; st < nst; ++st) {
        const int s = st % kGemmStages;
        if (!(ok = gwait(&full[s], (st / kGemmStages) & 1, abort_flag, g.status))) break;
        tc_fence_after();
        const uint32_t a = sbase + s * kStage, bb = a + kAStage;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {          // K = 8 per MMA
          const uint64_t ad = AMN ? sdesc_sw128(a + kk * 1024, 4096, 1024) : sdesc_sw128(a + kk * 32, 16, 1024);
          const uint64_t bd = BMN ? sdesc_sw128(bb + kk * 1024, 4096, 1024) : sdesc_sw128(bb + kk * 32, 16, 1024);
          mma_tf32(tmem, ad, bd, idesc, (st | kk) != 0);
        }
        mma_commit(&empty[s]);
      }
      if (ok) mma_commit(accfull);
      mma_commit(mdrain);
      gdrain(mdrain, 0, 500000000ull);
    }
  } else {
    // epilogue: rows staged in the pipeline's (now free) shared memory, lane =
    // row, then written row by row with the whole warp (coalesced)
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const bool ok = __all_sync(0xffffffffu, nst == 0 || gwait(accfull, 0, abort_flag, g.status)) != 0;
    if (ok && nst > 0) {
      tc_fence_after();
      constexpr int kLd = BN + 4;
      float* stg = reinterpret_cast<float*>(sm) + q * 32 * kLd;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + 32 * c, v);
        tmem_ld_wait();
        float4* d4 = reinterpret_cast<float4*>(stg + lane * kLd + 32 * c);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          d4[j] = make_float4(g.alpha * __uint_as_float(v[4 * j]), g.alpha * __uint_as_float(v[4 * j + 1]),
                              g.alpha * __uint_as_float(v[4 * j + 2]), g.alpha * __uint_as_float(v[4 * j + 3]));
      }
      __syncwarp();
      for (int rr = 0; rr < 32; ++rr) {
        const int64_t row = m0 + q * 32 + rr;
        if (row >= g.m) break;
        float* crow = g.C + static_cast<int64_t>(b) * g.sC + row * g.ldc;
        for (int cc = lane; cc < BN; cc += 32) {
          const int64_t col = n0 + cc;
          if (col < g.n) {
            const float x = stg[rr * kLd + cc];
            if (g.atomic) atomicAdd(crow + col, x);
            else crow[col] = g.beta != 0.f ? fmaf(g.beta, crow[col], x) : x;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// ---------------------------------------------------------------- bf16 operands
// The same GEMM with bf16 operands (tcgen05.mma.kind::f16), which the tensor
// core reads K-major or MN-major alike: a stage holds K = 64 (one 128-byte row
// of 64 bf16), one MMA is K = 16.  MN-major operands arrive as [64 k x 64 mn]
// boxes (8 KB) side by side.  Three epilogues:
//   kEpiStore   C (fp32) = alpha acc + beta C, or atomic adds under split K;
//   kEpiSwigluF the 128 columns of a tile are the up and gate projections of
//               64 hidden units (the weight's rows interleaved per 64): writes
//               A, G and H = A SiLU(G) as bf16 at hidden columns 64 tn ..;
//   kEpiSwigluB acc is dH for hidden columns 128 tn ..: reads A and G there
//               (bf16) and writes dA = dH SiLU(G) over A and
//               dG = dH A SiLU'(G) over G.
enum : int { kEpiStore = 0, kEpiSwigluF = 1, kEpiSwigluB = 2 };

struct Gemm16Args {
  int64_t m, n, k;
  int tiles_m, tiles_n, ksplit;
  int64_t k_per_split;          // multiple of 64
  float* C;
  int64_t ldc;
  float alpha, beta;
  int atomic;
  uint16_t *A16, *G16, *H16;    // SwiGLU epilogues: N x rd bf16 (A, G: ld = ld16; H: ld = ldh)
  int64_t ld16, ldh;
  int* status;
};

constexpr uint32_t kA16Stage = 128u * 128u;     // [128 x 64] bf16
constexpr int kGemm16Stages = 4;
constexpr int kGemm16Threads = 320;             // loader, MMA issuer, eight epilogue warps
// eight warps' staged rows; the largest is the SwiGLU backward's (A and G,
// 32 rows x 72 bf16 each); the plain store's is 32 x 68 floats
constexpr uint32_t kGemm16Staging = 8u * 2 * 32 * 72 * 2;

__device__ __forceinline__ float sigmoid_f(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }

template <int BN, bool AMN, bool BMN, int EPI>
__global__ void __launch_bounds__(kGemm16Threads, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const Gemm16Args g) {
  // Persistent: CTA c takes units c, c + gridDim.x, ... (unit = (row tile,
  // column tile, K split)); two TMEM accumulators let the epilogue of one unit
  // run while the next unit's stages load and multiply.
  constexpr int kStages = kGemm16Stages;
  constexpr uint32_t kBStage = BN * 128u;
  constexpr uint32_t kStage = kA16Stage + kBStage;
  constexpr uint32_t kStgOff = kStages * kStage;           // epilogue staging
  constexpr uint32_t kBarOff = kStgOff + kGemm16Staging;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(g.status, kStatusStepTimeout);
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* accfull = empty + kStages;       // [2]
  uint64_t* accempty = accfull + 2;          // [2]
  uint64_t* mdrain = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdrain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t units = static_cast<int64_t>(g.tiles_m) * g.tiles_n * g.ksplit;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 8); }
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);
  // unit -> (row tile, column tile, K range)
  auto decode = [&](int64_t u, int64_t& m0, int64_t& n0, int& tn, int64_t& k0, int& nst) {
    const int ks = static_cast<int>(u % g.ksplit);
    const int64_t r = u / g.ksplit;
    tn = static_cast<int>(r % g.tiles_n);
    const int64_t tm = r / g.tiles_n;
    m0 = tm * 128;
    n0 = static_cast<int64_t>(tn) * BN;
    k0 = ks * g.k_per_split;
    const int64_t k1 = min(g.k, k0 + g.k_per_split);
    nst = static_cast<int>((k1 - k0 + 63) / 64);
  };

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      uint32_t st = 0;
      for (int64_t u = blockIdx.x; ok && u < units; u += gridDim.x) {
        int64_t m0, n0, k0;
        int tn, nst;
        decode(u, m0, n0, tn, k0, nst);
        for (int j = 0; j < nst; ++j, ++st) {
          const int s = st % kStages;
          if (!(ok = gwait(&empty[s], ((st / kStages) & 1) ^ 1, abort_flag, g.status))) break;
          mbar_arrive_expect_tx(&full[s], kStage);
          uint8_t* a = sm + s * kStage;
          uint8_t* bb = a + kA16Stage;
          const int kk = static_cast<int>(k0 + 64 * j);
          if constexpr (AMN) {
            for (int i = 0; i < 2; ++i) tma_load_2d(a + i * 8192, &tmA, static_cast<int>(m0) + 64 * i, kk, &full[s]);
          } else {
            tma_load_2d(a, &tmA, kk, static_cast<int>(m0), &full[s]);
          }
          if constexpr (BMN) {
            for (int i = 0; i < BN / 64; ++i)
              tma_load_2d(bb + i * 8192, &tmB, static_cast<int>(n0) + 64 * i, kk, &full[s]);
          } else {
            tma_load_2d(bb, &tmB, kk, static_cast<int>(n0), &full[s]);
          }
        }
      }
      for (uint32_t c = st > kStages ? st - kStages : 0; c < st; ++c)
        gdrain(&full[c % kStages], (c / kStages) & 1, 100000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, AMN, BMN);
      bool ok = true;
      uint32_t st = 0, uc = 0;
      for (int64_t u = blockIdx.x; ok && u < units; u += gridDim.x, ++uc) {
        int64_t m0, n0, k0;
        int tn, nst;
        decode(u, m0, n0, tn, k0, nst);
        const int buf = uc & 1;
        if (!(ok = gwait(&accempty[buf], ((uc >> 1) & 1) ^ 1, abort_flag, g.status))) break;
        tc_fence_after();
        for (int j = 0; j < nst; ++j, ++st) {
          const int s = st % kStages;
          if (!(ok = gwait(&full[s], (st / kStages) & 1, abort_flag, g.status))) break;
          tc_fence_after();
          const uint32_t a = sbase + s * kStage, bb = a + kA16Stage;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {          // K = 16 per MMA
            const uint64_t ad = AMN ? sdesc_sw128(a + kk * 2048, 8192, 1024) : sdesc_sw128(a + kk * 32, 16, 1024);
            const uint64_t bd = BMN ? sdesc_sw128(bb + kk * 2048, 8192, 1024) : sdesc_sw128(bb + kk * 32, 16, 1024);
            mma_bf16_ss(tmem + buf * BN, ad, bd, idesc, (j | kk) != 0);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&accfull[buf]);
      }
      mma_commit(mdrain);
      gdrain(mdrain, 0, 500000000ull);
    }
  } else {
    // Epilogue, eight warps: warp w takes TMEM lane quarter q = w % 4 (rows
    // m0 + 32 q .. + 31 of a unit) and column half hf; it stages its rows in
    // its own shared-memory area (lane = row), frees the accumulator once all
    // eight have read it, and writes the rows with the whole warp (coalesced).
    const int q = warp & 3, hf = (warp - 2) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint8_t* stg_base = sm + kStgOff + (warp - 2) * (kGemm16Staging / 8);
    uint32_t uc = 0;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++uc) {
      int64_t m0, n0, k0;
      int tn, nst;
      decode(u, m0, n0, tn, k0, nst);
      const int buf = uc & 1;
      const int64_t rbase = m0 + q * 32;
      if constexpr (EPI == kEpiSwigluB) {
        // dH of hidden columns n0 + 64 hf .. + 63: the A and G rows come in
        // coalesced (4 rows per instruction) before the accumulator is ready
        constexpr int kLd = 72;                           // 64 bf16 + 8 pad per staged row
        uint16_t* sA = reinterpret_cast<uint16_t*>(stg_base);
        uint16_t* sG = sA + 32 * kLd;
        const int64_t col = n0 + 64 * hf + 8 * (lane & 7);
        for (int rr = 0; rr < 32; rr += 4) {
          const int r = rr + (lane >> 3);
          const int64_t row = rbase + r;
          const int off = r * kLd + 8 * (lane & 7);
          uint4 av = make_uint4(0u, 0u, 0u, 0u), gv = av;
          if (row < g.m) {
            av = *reinterpret_cast<const uint4*>(g.A16 + row * g.ld16 + col);
            gv = *reinterpret_cast<const uint4*>(g.G16 + row * g.ld16 + col);
          }
          *reinterpret_cast<uint4*>(sA + off) = av;
          *reinterpret_cast<uint4*>(sG + off) = gv;
        }
        __syncwarp();
      }
      if (!__all_sync(0xffffffffu, gwait(&accfull[buf], (uc >> 1) & 1, abort_flag, g.status))) break;
      tc_fence_after();
      const uint32_t tacc = tmem + buf * BN;
      if constexpr (EPI == kEpiStore) {
        constexpr int kHalf = BN / 2;                     // columns per warp
        constexpr int kLd = kHalf + 4;                    // floats per staged row
        float* stg = reinterpret_cast<float*>(stg_base);
#pragma unroll 1
        for (int c = 0; c < kHalf / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + lane_off + kHalf * hf + 32 * c, v);
          tmem_ld_wait();
          float4* d4 = reinterpret_cast<float4*>(stg + lane * kLd + 32 * c);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            d4[j] = make_float4(g.alpha * __uint_as_float(v[4 * j]), g.alpha * __uint_as_float(v[4 * j + 1]),
                                g.alpha * __uint_as_float(v[4 * j + 2]), g.alpha * __uint_as_float(v[4 * j + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[buf]);
        // kHalf / 4 float4 per row: 32 / (kHalf / 4) rows per warp instruction
        constexpr int kC4 = kHalf / 4, kRows = 32 / kC4;
        const bool vec = (g.ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(g.C) & 15) == 0;
        const int c4 = lane % kC4;
        const int64_t col = n0 + kHalf * hf + 4 * c4;
        for (int rr = 0; rr < 32; rr += kRows) {
          const int r = rr + lane / kC4;
          const int64_t row = rbase + r;
          if (row >= g.m) continue;
          float* crow = g.C + row * g.ldc;
          const float4 x = reinterpret_cast<const float4*>(stg + r * kLd)[c4];
          if (vec && col + 3 < g.n) {
            if (g.atomic) {
              asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(crow + col), "f"(x.x),
                           "f"(x.y), "f"(x.z), "f"(x.w)
                           : "memory");
            } else {
              float4 y = x;
              if (g.beta != 0.f) {
                const float4 o = *reinterpret_cast<const float4*>(crow + col);
                y = make_float4(fmaf(g.beta, o.x, x.x), fmaf(g.beta, o.y, x.y), fmaf(g.beta, o.z, x.z),
                                fmaf(g.beta, o.w, x.w));
              }
              *reinterpret_cast<float4*>(crow + col) = y;
            }
          } else {
            const float xs[4] = {x.x, x.y, x.z, x.w};
            for (int e = 0; e < 4; ++e)
              if (col + e < g.n) {
                if (g.atomic) atomicAdd(crow + col + e, xs[e]);
                else crow[col + e] = g.beta != 0.f ? fmaf(g.beta, crow[col + e], xs[e]) : xs[e];
              }
          }
        }
      } else if constexpr (EPI == kEpiSwigluF) {
        // columns 0..63: up projection of hidden units 64 tn .. +63; 64..127:
        // gate.  Half hf takes hidden units 32 hf .. 32 hf + 31 of the tile.
        constexpr int kLd = 40;                           // 32 bf16 + 8 pad per staged row
        uint16_t* sA = reinterpret_cast<uint16_t*>(stg_base);
        uint16_t* sG = sA + 32 * kLd;
        uint16_t* sH = sG + 32 * kLd;
        {
          uint32_t va[32], vg[32];
          tmem_ld32(tacc + lane_off + 32 * hf, va);
          tmem_ld32(tacc + lane_off + 64 + 32 * hf, vg);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&accempty[buf]);
#pragma unroll
          for (int j8 = 0; j8 < 4; ++j8) {
            uint32_t wa[4], wg[4], wh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a0 = __uint_as_float(va[8 * j8 + 2 * e]), a1 = __uint_as_float(va[8 * j8 + 2 * e + 1]);
              const float g0 = __uint_as_float(vg[8 * j8 + 2 * e]), g1 = __uint_as_float(vg[8 * j8 + 2 * e + 1]);
              wa[e] = pack_bf16x2(a0, a1);
              wg[e] = pack_bf16x2(g0, g1);
              wh[e] = pack_bf16x2(a0 * g0 * sigmoid_f(g0), a1 * g1 * sigmoid_f(g1));
            }
            const int off = lane * kLd + 8 * j8;
            *reinterpret_cast<uint4*>(sA + off) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
            *reinterpret_cast<uint4*>(sG + off) = make_uint4(wg[0], wg[1], wg[2], wg[3]);
            *reinterpret_cast<uint4*>(sH + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          }
        }
        __syncwarp();
        // 8 rows per warp instruction: lanes 4 i .. 4 i + 3 write row rr + i (64 bytes)
        const int64_t col = static_cast<int64_t>(tn) * 64 + 32 * hf + 8 * (lane & 3);
        for (int rr = 0; rr < 32; rr += 8) {
          const int r = rr + (lane >> 2);
          const int64_t row = rbase + r;
          if (row < g.m) {
            const int off = r * kLd + 8 * (lane & 3);
            *reinterpret_cast<uint4*>(g.A16 + row * g.ld16 + col) = *reinterpret_cast<const uint4*>(sA + off);
            *reinterpret_cast<uint4*>(g.G16 + row * g.ld16 + col) = *reinterpret_cast<const uint4*>(sG + off);
            *reinterpret_cast<uint4*>(g.H16 + row * g.ldh + col) = *reinterpret_cast<const uint4*>(sH + off);
          }
        }
      } else {
        constexpr int kLd = 72;
        uint16_t* sA = reinterpret_cast<uint16_t*>(stg_base);
        uint16_t* sG = sA + 32 * kLd;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + lane_off + 64 * hf + 32 * c, v);
          tmem_ld_wait();
#pragma unroll
          for (int j8 = 0; j8 < 4; ++j8) {
            const int off = lane * kLd + 32 * c + 8 * j8;
            const uint4 av = *reinterpret_cast<const uint4*>(sA + off);
            const uint4 gv = *reinterpret_cast<const uint4*>(sG + off);
            const uint32_t aw[4] = {av.x, av.y, av.z, av.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t da[4], dg[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float outa[2], outg[2];
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const float aa = __uint_as_float(hh ? (aw[e] & 0xFFFF0000u) : (aw[e] << 16));
                const float gg = __uint_as_float(hh ? (gw[e] & 0xFFFF0000u) : (gw[e] << 16));
                const float dh = __uint_as_float(v[8 * j8 + 2 * e + hh]);
                const float sg = sigmoid_f(gg);
                outa[hh] = dh * gg * sg;
                outg[hh] = dh * aa * sg * (1.f + gg * (1.f - sg));
              }
              da[e] = pack_bf16x2(outa[0], outa[1]);
              dg[e] = pack_bf16x2(outg[0], outg[1]);
            }
            *reinterpret_cast<uint4*>(sA + off) = make_uint4(da[0], da[1], da[2], da[3]);
            *reinterpret_cast<uint4*>(sG + off) = make_uint4(dg[0], dg[1], dg[2], dg[3]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[buf]);
        const int64_t col = n0 + 64 * hf + 8 * (lane & 7);
        for (int rr = 0; rr < 32; rr += 4) {
          const int r = rr + (lane >> 3);
          const int64_t row = rbase + r;
          if (row < g.m) {
            const int off = r * kLd + 8 * (lane & 7);
            *reinterpret_cast<uint4*>(g.A16 + row * g.ld16 + col) = *reinterpret_cast<const uint4*>(sA + off);
            *reinterpret_cast<uint4*>(g.G16 + row * g.ld16 + col) = *reinterpret_cast<const uint4*>(sG + off);
          }
        }
      }
      __syncwarp();                                     // staging rows are reused by the next unit
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// 128-bit alignment of an address and of a stride in elements.
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool st16(int64_t elems) { return ((elems * 4) & 15) == 0; }

// Tensor map of one operand stored row-major as `rows` x `inner` with row
// stride ld, the box `bx` inner x `by` rows.  A batch whose members sit side by
// side along the rows (stride below a whole matrix: one head's columns) is
// the map's middle dimension, so the strides grow outward; a batch of whole
// matrices is the outer dimension.  *bmid tells the kernel which.
int operand_map(CUtensorMap* m, const float* base, int64_t inner, int64_t rows, int64_t ld, int batch,
                int64_t stride, uint32_t bx, uint32_t by, int* bmid) {
  *bmid = batch > 1 && stride < ld * rows ? 1 : 0;
  if (*bmid) {
    const uint64_t dims[3] = {static_cast<uint64_t>(inner), static_cast<uint64_t>(batch), static_cast<uint64_t>(rows)};
    const uint64_t str[2] = {static_cast<uint64_t>(stride) * 4, static_cast<uint64_t>(ld) * 4};
    const uint32_t box[3] = {bx, 1, by};
    return make_tmap_f32_3d(m, base, dims, str, box);
  }
  const uint64_t dims[3] = {static_cast<uint64_t>(inner), static_cast<uint64_t>(rows), static_cast<uint64_t>(batch)};
  const uint64_t str[2] = {static_cast<uint64_t>(ld) * 4,
                           static_cast<uint64_t>(batch > 1 ? stride : ld * rows) * 4};
  const uint32_t box[3] = {bx, by, 1};
  return make_tmap_f32_3d(m, base, dims, str, box);
}

template <int BN, bool AMN, bool BMN>
int launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g, int64_t units,
                cudaStream_t s) {
  auto k = gemm_tf32_kernel<BN, AMN, BMN>;
  // the stages, then 2 kGemmStages + 2 mbarriers, the TMEM slot and the abort flag
  const uint32_t smem = kGemmStages * (kAStage + BN * 128u) + (2 * kGemmStages + 2) * 8 + 16;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("gemm_tc smem: ") + cudaGetErrorString(e));
  k<<<static_cast<unsigned>(units), kGemmThreads, smem, s>>>(tmA, tmB, g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("gemm_tc launch: ") + cudaGetErrorString(e));
  return STCA_OK;
}

template <int BN>
int launch_gemm_bn(bool amn, bool bmn, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g,
                   int64_t units, cudaStream_t s) {
  if (amn && bmn) return launch_gemm<BN, true, true>(tmA, tmB, g, units, s);
  if (amn) return launch_gemm<BN, true, false>(tmA, tmB, g, units, s);
  if (bmn) return launch_gemm<BN, false, true>(tmA, tmB, g, units, s);
  return launch_gemm<BN, false, false>(tmA, tmB, g, units, s);
}

}  // namespace

int tc_gemm_tf32(bool ta, bool tb, int64_t m, int64_t n, int64_t k, const float* A, int64_t lda,
                 const float* B, int64_t ldb, float* C, int64_t ldc, float beta, float alpha, int batch,
                 int64_t sA, int64_t sB, int64_t sC, int num_sms, int* status, cudaStream_t s) {
  if (m <= 0 || n <= 0 || batch <= 0) return STCA_OK;
  // TF32 operands must be K-major: the tensor core reads 32-bit types only in
  // that layout (a transposed operand is declined here and runs elsewhere)
  if (ta || !tb) return set_error(STCA_EINVAL, "tensor-core TF32 GEMM: operands must be K-major");
  if (!al16(A) || !al16(B) || !st16(lda) || !st16(ldb) || (batch > 1 && (!st16(sA) || !st16(sB))))
    return set_error(STCA_EINVAL, "tensor-core GEMM: operands not 16-byte aligned");
  if (m > INT32_MAX || n > INT32_MAX || k > INT32_MAX) return set_error(STCA_EINVAL, "tensor-core GEMM: too large");
  const bool amn = ta, bmn = !tb;
  // tile width: 128 columns, or 64 / 32 for narrow outputs
  int BN = 128;
  while (BN > 32 && BN / 2 >= n) BN /= 2;
  GemmArgs g{};
  g.m = m;
  g.n = n;
  g.k = k;
  g.tiles_m = static_cast<int>((m + 127) / 128);
  g.tiles_n = static_cast<int>((n + BN - 1) / BN);
  g.C = C;
  g.ldc = ldc;
  g.sC = sC;
  g.alpha = alpha;
  g.beta = beta;
  g.status = status;
  // split a long K over CTAs when the output tiles alone cannot fill the GPU
  const int64_t tiles = static_cast<int64_t>(g.tiles_m) * g.tiles_n * batch;
  int ksplit = 1;
  if (k >= 4096 && tiles < num_sms) ksplit = static_cast<int>(std::min<int64_t>(num_sms / tiles, (k + 1023) / 1024));
  ksplit = std::max(ksplit, 1);
  g.k_per_split = ((k + ksplit - 1) / ksplit + 31) / 32 * 32;
  g.ksplit = static_cast<int>(std::max<int64_t>(1, (k + g.k_per_split - 1) / g.k_per_split));
  g.atomic = g.ksplit > 1;
  CUtensorMap tmA, tmB;
  // op(A): A^T stored k x m (MN-major) or A stored m x k (K-major);
  // op(B): B stored k x n (MN-major) or B^T stored n x k (K-major).
  // A map the driver declines is reported as STCA_EINVAL: nothing has run yet.
  if (operand_map(&tmA, A, amn ? m : k, amn ? k : m, lda, batch, sA, 32, amn ? 32u : 128u, &g.a_bmid) ||
      operand_map(&tmB, B, bmn ? n : k, bmn ? k : n, ldb, batch, sB, 32, bmn ? 32u : static_cast<uint32_t>(BN),
                  &g.b_bmid))
    return set_error(STCA_EINVAL, "tensor-core GEMM: operand layout not expressible as a tensor map");
  if (g.atomic) {
    // every split adds alpha times its part to C, which starts as beta C
    if (beta == 0.f) {
      for (int i = 0; i < batch; ++i)
        STCA_CUDA_TRY(cudaMemset2DAsync(C + i * sC, ldc * 4, 0, n * 4, m, s));
    } else if (beta != 1.f) {
      return set_error(STCA_EINVAL, "tensor-core GEMM: split K needs beta 0 or 1");
    }
  }
  const int64_t units = static_cast<int64_t>(g.tiles_m) * g.tiles_n * g.ksplit * batch;
  if (units > INT32_MAX) return set_error(STCA_EINVAL, "tensor-core GEMM: too many tiles");
  switch (BN) {
    case 128: return launch_gemm_bn<128>(amn, bmn, tmA, tmB, g, units, s);
    case 64: return launch_gemm_bn<64>(amn, bmn, tmA, tmB, g, units, s);
    default: return launch_gemm_bn<32>(amn, bmn, tmA, tmB, g, units, s);
  }
}


namespace {
// bf16 operand map: stored row-major `rows` x `inner` with row stride ld
// (elements), box bx x by.
int map16(CUtensorMap* m, const uint16_t* base, int64_t inner, int64_t rows, int64_t ld, uint32_t bx, uint32_t by) {
  return make_tmap_bf16_2d_strided(m, base, static_cast<uint64_t>(inner), static_cast<uint64_t>(rows),
                                   static_cast<uint64_t>(ld) * 2, bx, by);
}

template <int BN, int EPI>
int launch16(bool amn, bool bmn, const CUtensorMap& tmA, const CUtensorMap& tmB, const Gemm16Args& g,
             int64_t units, int num_sms, cudaStream_t s) {
  const uint32_t smem = kGemm16Stages * (kA16Stage + BN * 128u) + kGemm16Staging + (2 * kGemm16Stages + 5) * 8 + 16;
  static_assert(kGemm16Stages * (kA16Stage + 128u * 128u) + kGemm16Staging + (2 * kGemm16Stages + 5) * 8 + 16 <=
                    227u * 1024u, "bf16 GEMM shared memory");
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(units, std::max(num_sms, 1)));
  auto go = [&](auto kf) -> int {
    cudaError_t e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("gemm_bf16 smem: ") + cudaGetErrorString(e));
    kf<<<grid, kGemm16Threads, smem, s>>>(tmA, tmB, g);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("gemm_bf16 launch: ") + cudaGetErrorString(e));
    return STCA_OK;
  };
  if (amn && bmn) return go(gemm_bf16_kernel<BN, true, true, EPI>);
  if (amn) return go(gemm_bf16_kernel<BN, true, false, EPI>);
  if (bmn) return go(gemm_bf16_kernel<BN, false, true, EPI>);
  return go(gemm_bf16_kernel<BN, false, false, EPI>);
}
}  // namespace

int tc_gemm_bf16(bool ta, bool tb, int64_t m, int64_t n, int64_t k, const uint16_t* A, int64_t lda,
                 const uint16_t* B, int64_t ldb, float* C, int64_t ldc, float beta, int epi, uint16_t* A16,
                 uint16_t* G16, uint16_t* H16, int64_t ld16, int64_t ldh, int num_sms, int* status, cudaStream_t s) {
  if (m <= 0 || n <= 0) return STCA_OK;
  if (k <= 0) return set_error(STCA_EINVAL, "bf16 tensor-core GEMM: empty inner dimension");
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al(A) || !al(B) || (lda * 2) % 16 || (ldb * 2) % 16)
    return set_error(STCA_EINVAL, "bf16 tensor-core GEMM: operands not 16-byte aligned");
  const bool amn = ta, bmn = !tb;
  const int BN = (epi != kEpiStore || n > 64) ? 128 : 64;
  if (epi != kEpiStore && (n % 128 || !A16 || !G16 || (epi == kEpiSwigluF && !H16)))
    return set_error(STCA_EINVAL, "bf16 tensor-core GEMM: SwiGLU epilogue needs whole 128-column tiles");
  Gemm16Args g{};
  g.m = m;
  g.n = n;
  g.k = k;
  g.tiles_m = static_cast<int>((m + 127) / 128);
  g.tiles_n = static_cast<int>((n + BN - 1) / BN);
  g.C = C;
  g.ldc = ldc;
  g.alpha = 1.f;
  g.beta = beta;
  g.A16 = A16;
  g.G16 = G16;
  g.H16 = H16;
  g.ld16 = ld16;
  g.ldh = ldh;
  g.status = status;
  const int64_t tiles = static_cast<int64_t>(g.tiles_m) * g.tiles_n;
  int ksplit = 1;
  if (epi == kEpiStore && k >= 4096 && tiles < num_sms)
    ksplit = static_cast<int>(std::min<int64_t>(num_sms / tiles, (k + 2047) / 2048));
  ksplit = std::max(ksplit, 1);
  g.k_per_split = ((k + ksplit - 1) / ksplit + 63) / 64 * 64;
  g.ksplit = static_cast<int>(std::max<int64_t>(1, (k + g.k_per_split - 1) / g.k_per_split));
  g.atomic = g.ksplit > 1;
  CUtensorMap tmA, tmB;
  if (map16(&tmA, A, amn ? m : k, amn ? k : m, lda, 64, amn ? 64u : 128u) ||
      map16(&tmB, B, bmn ? n : k, bmn ? k : n, ldb, 64, bmn ? 64u : static_cast<uint32_t>(BN)))
    return set_error(STCA_EINVAL, "bf16 tensor-core GEMM: operand layout not expressible as a tensor map");
  if (g.atomic) {
    if (beta == 0.f) STCA_CUDA_TRY(cudaMemset2DAsync(C, ldc * 4, 0, n * 4, m, s));
    else if (beta != 1.f) return set_error(STCA_EINVAL, "bf16 tensor-core GEMM: split K needs beta 0 or 1");
  }
  const int64_t units = tiles * g.ksplit;
  if (units > INT32_MAX) return set_error(STCA_EINVAL, "bf16 tensor-core GEMM: too many tiles");
  if (BN == 64) return launch16<64, kEpiStore>(amn, bmn, tmA, tmB, g, units, num_sms, s);
  switch (epi) {
    case kEpiSwigluF: return launch16<128, kEpiSwigluF>(amn, bmn, tmA, tmB, g, units, num_sms, s);
    case kEpiSwigluB: return launch16<128, kEpiSwigluB>(amn, bmn, tmA, tmB, g, units, num_sms, s);
    default: return launch16<128, kEpiStore>(amn, bmn, tmA, tmB, g, units, num_sms, s);
  }
}

}  // namespace stca
