// Backward pass of the pieces of the STCA step ("Make It Long, Keep It Fast"
// digest §2.1; training with request-level batching, STCA blog §2.5), under a
// loss whose gradient is given:
//
//  * the history encoding X~ = LN(((X W_u) * SiLU(X W_g)) W_d) (Eqs. (1)-(2)),
//    and with the query weights the query init q(1) of Eq. (3):
//      dX, dW_u, dW_g, dW_d, dgamma, dbeta from dX~.  The products are plain
//      fp32 GEMMs run by cuBLASLt (TF32 tensor cores for bf16 handles, exact
//      fp32 otherwise); the SwiGLU and LayerNorm derivatives are two kernels here.
//  * the single-query attention of Eq. (13) on merged rows c = softmax(u X~^T) X~:
//      dU and dX~ from dC, with the softmax recomputed flash-style:
//        row kernel: per query row, pass 1 over the keys gives m, l and
//          delta = sum_l P_l dP_l (dP_l = dc . x~_l); pass 2 gives
//          dU = sum_l dS_l x~_l with dS_l = P_l (dP_l - delta);
//        key kernel: per key, dX~_l = sum_rows (P dc + dS u) over the request's rows.
//    Both run on the CUDA cores: a thread holds an eighth of a row's (or key's)
//    d features, and eight lanes reduce the dot products by shuffles; operands
//    are staged in shared memory with 16-byte loads.
//  * the projections around the attention (Eqs. (6), (13)): the output side
//    (W_V, W_O: dZ -> dC) and the query side (W_Q, W_K: dU -> dQ), plain
//    products with the per-head slices as strided batches;
//  * the fusion blocks of Eq. (7) and the head of Eq. (9),
//    SwiGLUFFN([o(1) || ... || o(b) || x_t] W): d[o(1..b)], dx_t and the weights'
//    gradients, the FFN forward recomputed.
#include <cublasLt.h>
#include <cuda_bf16.h>
#include <math.h>

#include <cmath>

#include <algorithm>
#include <string>
#include <vector>

#include "stca_internal.h"

namespace stca {
namespace {

constexpr int kLanes = 8;           // lanes per row (or key), each with d / 8 features
constexpr int kBwThreads = 128;     // 16 rows (or keys) x 8 lanes
constexpr int kBwBlock = kBwThreads / kLanes;
constexpr int kBwTile = 32;         // keys (or rows) staged per shared-memory tile

__device__ __forceinline__ float ld_x(const void* X, bool bf, int64_t i) {
  if (bf) return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(X)[i]) << 16);
  return static_cast<const float*>(X)[i];
}

// Stage n rows of d values of X (bf16 or fp32) as fp32 into s, 8 values per
// 16-byte load (d % 8 == 0, rows 16-byte aligned).
__device__ __forceinline__ void stage_rows(float* s, const void* X, bool bf, int64_t row0, int n, int d) {
  const int n8 = n * d / 8;
  for (int e = threadIdx.x; e < n8; e += blockDim.x) {
    float4 lo, hi;
    if (bf) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(X) + row0 * d) + e);
      lo = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
      hi = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u),
                       __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
    } else {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(X) + row0 * d) + 2 * e;
      lo = __ldg(src);
      hi = __ldg(src + 1);
    }
    reinterpret_cast<float4*>(s)[2 * e] = lo;
    reinterpret_cast<float4*>(s)[2 * e + 1] = hi;
  }
}

// Sum over the kLanes lanes that share a row (or key).
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  return v;
}

// Work unit of the attention backward: request, first row (or key) of the
// block, rows (or keys) in it.
struct BwUnit {
  int32_t req;
  int32_t n;
  int64_t first;
};

struct AttnBwArgs {
  const void* Xt;           // N x d (bf16 or fp32): X~ of the layer
  int xbf;
  const float* U;           // T h x d
  const float* dC;          // T h x d
  float* dU;                // T h x d
  float* dX;                // N x d
  float* stats;             // T h x 3: m, l, delta
  const int64_t* off;       // R + 1 (keys)
  const int64_t* qoff;      // R + 1 (query rows: toff * h)
  const BwUnit* units;
  int d;
};

// Row kernel: block of up to 16 query rows of one request; thread (row, eighth
// of the d = 8 DQ features).
template <int DQ>
__global__ void __launch_bounds__(kBwThreads) attn_bw_rows_kernel(AttnBwArgs a) {
  extern __shared__ float sk[];                 // kBwTile x d keys (fp32)
  const BwUnit un = a.units[blockIdx.x];
  constexpr int kMaxQ = DQ;
  const int d = kLanes * DQ, dq = DQ;
  const int tid = threadIdx.x, rl = tid / kLanes, qu = tid % kLanes;
  const bool active = rl < un.n;
  const int64_t row = un.first + rl;
  const int64_t k0 = a.off[un.req], L = a.off[un.req + 1] - k0;
  float u[kMaxQ], dc[kMaxQ], du[kMaxQ];
#pragma unroll
  for (int f = 0; f < kMaxQ; ++f) {
    u[f] = dc[f] = du[f] = 0.f;
    if (f < dq && active) {
      u[f] = a.U[row * d + f * kLanes + qu];      // features interleaved across the lanes:
      dc[f] = a.dC[row * d + f * kLanes + qu];    // conflict-free shared-memory reads
    }
  }
  float m = -INFINITY, l = 0.f, dl = 0.f;       // running max, sum, sum of P dP (unnormalised)
  for (int pass = 0; pass < 2; ++pass) {
    const float inv_l = pass ? 1.f / l : 0.f, delta = pass ? dl / l : 0.f;
    for (int64_t kt = 0; kt < L; kt += kBwTile) {
      const int nk = static_cast<int>(L - kt < kBwTile ? L - kt : kBwTile);
      __syncthreads();
      stage_rows(sk, a.Xt, a.xbf, k0 + kt, nk, d);
      __syncthreads();
      for (int k = 0; k < nk; ++k) {
        const float* xk = sk + k * d + qu;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int f = 0; f < kMaxQ; ++f)
          if (f < dq) {
            s = fmaf(u[f], xk[f * kLanes], s);
            dp = fmaf(dc[f], xk[f * kLanes], dp);
          }
        s = quad_sum(s);
        dp = quad_sum(dp);
        if (pass == 0) {
          if (s > m) {
            const float c = __expf(m - s);
            l *= c;
            dl *= c;
            m = s;
          }
          const float e = __expf(s - m);
          l += e;
          dl = fmaf(e, dp, dl);
        } else {
          const float p = __expf(s - m) * inv_l;
          const float ds = p * (dp - delta);
#pragma unroll
          for (int f = 0; f < kMaxQ; ++f)
            if (f < dq) du[f] = fmaf(ds, xk[f * kLanes], du[f]);
        }
      }
    }
  }
  if (!active) return;
#pragma unroll
  for (int f = 0; f < kMaxQ; ++f)
    if (f < dq) a.dU[row * d + f * kLanes + qu] = du[f];
  if (qu == 0) {
    a.stats[row * 3 + 0] = m;
    a.stats[row * 3 + 1] = l;
    a.stats[row * 3 + 2] = dl / l;
  }
}

// Key kernel: block of up to 16 keys of one request; thread (key, eighth).
template <int DQ>
__global__ void __launch_bounds__(kBwThreads) attn_bw_keys_kernel(AttnBwArgs a) {
  extern __shared__ float sr[];                 // kBwTile rows x (2 d + 3): u, dc, m l delta
  const BwUnit un = a.units[blockIdx.x];
  constexpr int kMaxQ = DQ;
  const int d = kLanes * DQ, dq = DQ, w = 2 * d + 3;
  const int tid = threadIdx.x, kl = tid / kLanes, qu = tid % kLanes;
  const bool active = kl < un.n;
  const int64_t key = un.first + kl;
  const int64_t r0 = a.qoff[un.req], R = a.qoff[un.req + 1] - r0;
  float x[kMaxQ], dx[kMaxQ];
#pragma unroll
  for (int f = 0; f < kMaxQ; ++f) {
    x[f] = dx[f] = 0.f;
    if (f < dq && active) x[f] = ld_x(a.Xt, a.xbf, key * d + f * kLanes + qu);
  }
  for (int64_t rt = 0; rt < R; rt += kBwTile) {
    const int nr = static_cast<int>(R - rt < kBwTile ? R - rt : kBwTile);
    __syncthreads();
    {
      // u and dc of the tile's rows as float4, then their statistics
      const int d4 = d / 4;
      for (int e = tid; e < nr * 2 * d4; e += kBwThreads) {
        const int r = e / (2 * d4), c4 = e - r * 2 * d4;
        const int64_t row = r0 + rt + r;
        const float4 v = c4 < d4 ? __ldg(reinterpret_cast<const float4*>(a.U + row * d) + c4)
                                 : __ldg(reinterpret_cast<const float4*>(a.dC + row * d) + c4 - d4);
        float* dst = sr + r * w + 4 * c4;
        dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
      }
      for (int e = tid; e < nr * 3; e += kBwThreads) {
        const int r = e / 3, c = e - r * 3;
        sr[r * w + 2 * d + c] = a.stats[(r0 + rt + r) * 3 + c];
      }
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      const float* ur = sr + r * w + qu;
      const float* cr = ur + d;
      const float m = sr[r * w + 2 * d], l = sr[r * w + 2 * d + 1], delta = sr[r * w + 2 * d + 2];
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int f = 0; f < kMaxQ; ++f)
        if (f < dq) {
          s = fmaf(ur[f * kLanes], x[f], s);
          dp = fmaf(cr[f * kLanes], x[f], dp);
        }
      s = quad_sum(s);
      dp = quad_sum(dp);
      const float p = __expf(s - m) / l;
      const float ds = p * (dp - delta);
#pragma unroll
      for (int f = 0; f < kMaxQ; ++f)
        if (f < dq) dx[f] = fmaf(p, cr[f * kLanes], fmaf(ds, ur[f * kLanes], dx[f]));
    }
  }
  if (!active) return;
#pragma unroll
  for (int f = 0; f < kMaxQ; ++f)
    if (f < dq) a.dX[key * d + f * kLanes + qu] = dx[f];
}

// ---------------------------------------------------------------- encoder
__device__ __forceinline__ float sigm(float z) { return 1.0f / (1.0f + __expf(-z)); }

// H = A * SiLU(G), elementwise over n values.
__global__ void swiglu_fwd_kernel(const float* __restrict__ A, const float* __restrict__ G,
                                  float* __restrict__ H, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float g = G[i];
    H[i] = A[i] * g * sigm(g);
  }
}

// dA = dH * SiLU(G), dG = dH * A * SiLU'(G), written over A and G.
__global__ void swiglu_bwd_kernel(float* __restrict__ A, float* __restrict__ G,
                                  const float* __restrict__ dH, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float g = G[i], a = A[i], dh = dH[i], sg = sigm(g);
    A[i] = dh * g * sg;
    G[i] = dh * a * sg * (1.0f + g * (1.0f - sg));
  }
}

// LayerNorm backward: a CTA of 8 warps takes kLnRows consecutive rows, one warp
// per row at a time.  Y holds y on entry and dy on exit (or, given dy16, dy goes
// there as bf16 and Y is left as it was).  Each lane keeps its
// columns' sums of dX~ * yhat and dX~ in registers over the CTA's rows, the
// warps add them in shared memory, and the CTA adds its totals to dgamma and
// dbeta with one atomic per column.
constexpr int kLnRows = 256;
constexpr int kLnMaxCols = 8;                  // d / 32, d <= 256

__global__ void __launch_bounds__(256) ln_bwd_kernel(float* __restrict__ Y, const float* __restrict__ dXt,
                                                     const float* __restrict__ gamma, float* __restrict__ dgamma,
                                                     float* __restrict__ dbeta, int64_t N, int d,
                                                     uint16_t* __restrict__ dy16 = nullptr) {
  __shared__ float sg[256], sb[256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int c = threadIdx.x; c < d; c += 256) sg[c] = sb[c] = 0.f;
  __syncthreads();
  float ag[kLnMaxCols], ab[kLnMaxCols];
#pragma unroll
  for (int j = 0; j < kLnMaxCols; ++j) ag[j] = ab[j] = 0.f;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kLnRows;
  for (int64_t row = r0 + warp; row < N && row < r0 + kLnRows; row += 8) {
    float* y = Y + row * d;
    const float* g = dXt + row * d;
    float yv[kLnMaxCols], gv[kLnMaxCols];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kLnMaxCols; ++j) {
      const int c = lane + 32 * j;
      yv[j] = c < d ? y[c] : 0.f;
      gv[j] = c < d ? g[c] : 0.f;
      s += yv[j];
    }
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mu = s / d;
    float v = 0.f;
#pragma unroll
    for (int j = 0; j < kLnMaxCols; ++j)
      if (lane + 32 * j < d) { const float t = yv[j] - mu; v = fmaf(t, t, v); }
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const float rstd = rsqrtf(v / d + 1e-5f);
    float m1 = 0.f, m2 = 0.f;                    // sums of dyh and dyh * yhat
#pragma unroll
    for (int j = 0; j < kLnMaxCols; ++j) {
      const int c = lane + 32 * j;
      if (c >= d) continue;
      const float yh = (yv[j] - mu) * rstd, dyh = gv[j] * gamma[c];
      m1 += dyh;
      m2 = fmaf(dyh, yh, m2);
      ag[j] = fmaf(gv[j], yh, ag[j]);
      ab[j] += gv[j];
    }
    for (int o = 16; o > 0; o >>= 1) {
      m1 += __shfl_xor_sync(0xffffffffu, m1, o);
      m2 += __shfl_xor_sync(0xffffffffu, m2, o);
    }
    m1 /= d;
    m2 /= d;
#pragma unroll
    for (int j = 0; j < kLnMaxCols; ++j) {
      const int c = lane + 32 * j;
      if (c >= d) continue;
      const float yh = (yv[j] - mu) * rstd, dyh = gv[j] * gamma[c];
      const float dy = rstd * (dyh - m1 - yh * m2);
      // the bf16 pipeline reads dy only as bf16: the fp32 copy is then not written
      if (dy16) dy16[row * d + c] = __bfloat16_as_ushort(__float2bfloat16_rn(dy));
      else y[c] = dy;
    }
  }
#pragma unroll
  for (int j = 0; j < kLnMaxCols; ++j) {
    const int c = lane + 32 * j;
    if (c < d) {
      atomicAdd(&sg[c], ag[j]);
      atomicAdd(&sb[c], ab[j]);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += 256) {
    atomicAdd(&dgamma[c], sg[c]);
    atomicAdd(&dbeta[c], sb[c]);
  }
}

// bf16 layouts of one SwiGLU FFN's weights for the tensor-core backward:
//   W1i (2rd x d): rows 128 c + j hold column 64 c + j of W_u (j < 64) or
//                  column 64 c + j - 64 of W_g: up and gate of 64 hidden units
//                  per 128-row tile (the recomputation's B operand, K-major);
//   WdT (d x rd) = W_d^T;  Wd16 (rd x d), Wu16, Wg16 (d x rd): row-major copies.
__global__ void ffn_weights16_kernel(const float* __restrict__ Wu, const float* __restrict__ Wg,
                                     const float* __restrict__ Wd, uint16_t* __restrict__ W1i,
                                     uint16_t* __restrict__ WdT, uint16_t* __restrict__ Wd16,
                                     uint16_t* __restrict__ Wu16, uint16_t* __restrict__ Wg16, int d, int rd) {
  const int64_t n = static_cast<int64_t>(d) * rd;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    auto bf = [](float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); };
    // i = k * rd + hcol (row-major d x rd index of W_u / W_g)
    const int64_t k = i / rd, hcol = i - k * rd;
    const int64_t c = hcol / 64, j = hcol - c * 64;
    W1i[(128 * c + j) * d + k] = bf(Wu[i]);
    W1i[(128 * c + 64 + j) * d + k] = bf(Wg[i]);
    // [W_u | W_g] side by side: row k of a d x 2 rd matrix
    Wu16[k * 2 * rd + hcol] = bf(Wu[i]);
    Wg16[k * 2 * rd + hcol] = bf(Wg[i]);
    // i as a row-major rd x d index of W_d: (h, nn)
    const int64_t h = i / d, nn = i - h * d;
    Wd16[i] = bf(Wd[i]);
    WdT[nn * rd + h] = bf(Wd[i]);
  }
}

__global__ void to_f32_kernel(const uint16_t* __restrict__ x, float* __restrict__ y, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = __uint_as_float(static_cast<uint32_t>(x[i]) << 16);
}

unsigned grid_for(int64_t n) { return static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 148 * 16)); }

// Row-major C (m x n) = op(A) op(B) (+ C when beta = 1), fp32, through cuBLASLt's
// column-major view C^T = op(B)^T op(A)^T.  ta / tb: A / B stored transposed.
int gemm_rm(stca_handle* H, bool ta, bool tb, int64_t m, int64_t n, int64_t k, const float* A,
            int64_t lda, const float* B, int64_t ldb, float* C, int64_t ldc, float beta,
            cudaStream_t s, float alpha = 1.f, int batch = 1, int64_t sA = 0, int64_t sB = 0,
            int64_t sC = 0) {
  // bf16 handles: TF32 products on the tensor cores by the library's own GEMM
  // (gemm_tc.cu); fp32 handles keep exact fp32 products (cuBLASLt, no TF32),
  // which the 1e-3 bound of the fp32 configuration needs
  // (a product whose operands TMA cannot address -- unaligned, or a tensor map
  // the driver declines -- is refused before anything is launched, and runs on
  // cuBLASLt instead)
  if (H->elem == 2 && H->opt_bw_gemm != 1) {
    const int rc = tc_gemm_tf32(ta, tb, m, n, k, A, lda, B, ldb, C, ldc, beta, alpha, batch, sA, sB, sC,
                                H->num_sms, H->status_d, s);
    if (rc != STCA_EINVAL) return rc;
  }
  if (!H->lt) {
    cublasLtHandle_t lt = nullptr;
    if (cublasLtCreate(&lt) != CUBLAS_STATUS_SUCCESS) return set_error(STCA_ECUDA, "cublasLtCreate failed");
    H->lt = lt;
  }
  constexpr size_t kWs = size_t(32) << 20;
  if (!H->lt_ws || H->lt_ws_cap < kWs) {
    cudaFree(H->lt_ws);
    H->lt_ws = nullptr;
    H->lt_ws_cap = 0;
    if (cudaMalloc(&H->lt_ws, kWs) != cudaSuccess) {
      cudaGetLastError();
      return set_error(STCA_ENOMEM, "cuBLASLt workspace");
    }
    H->lt_ws_cap = kWs;
  }
  cublasLtHandle_t lt = static_cast<cublasLtHandle_t>(H->lt);
  const cublasComputeType_t ct = H->elem == 2 ? CUBLAS_COMPUTE_32F_FAST_TF32 : CUBLAS_COMPUTE_32F;
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t l1 = nullptr, l2 = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  int rc = STCA_OK;
  // first cuBLAS operand: B (n x k after op), second: A (k x m after op)
  const cublasOperation_t o1 = tb ? CUBLAS_OP_T : CUBLAS_OP_N, o2 = ta ? CUBLAS_OP_T : CUBLAS_OP_N;
  if (cublasLtMatmulDescCreate(&op, ct, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &o1, sizeof(o1)) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &o2, sizeof(o2)) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&l1, CUDA_R_32F, tb ? k : n, tb ? n : k, ldb) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&l2, CUDA_R_32F, ta ? m : k, ta ? k : m, lda) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&lc, CUDA_R_32F, n, m, ldc) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS)
    rc = set_error(STCA_ECUDA, "cuBLASLt descriptor set-up failed");
  if (rc == STCA_OK && batch > 1) {
    // `batch` products, operand i at A + i sA, B + i sB, C + i sC
    const int64_t strides[3] = {sB, sA, sC};
    cublasLtMatrixLayout_t lays[3] = {l1, l2, lc};
    for (int i = 0; i < 3 && rc == STCA_OK; ++i)
      if (cublasLtMatrixLayoutSetAttribute(lays[i], CUBLASLT_MATRIX_LAYOUT_BATCH_COUNT, &batch, sizeof(batch)) !=
              CUBLAS_STATUS_SUCCESS ||
          cublasLtMatrixLayoutSetAttribute(lays[i], CUBLASLT_MATRIX_LAYOUT_STRIDED_BATCH_OFFSET, &strides[i],
                                           sizeof(strides[i])) != CUBLAS_STATUS_SUCCESS)
        rc = set_error(STCA_ECUDA, "cuBLASLt batch set-up failed");
  }
  cublasLtMatmulHeuristicResult_t heur{};
  int found = 0;
  if (rc == STCA_OK) {
    size_t ws = kWs;
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws, sizeof(ws));
    // operands may be column slices (one head's columns): tell the heuristic
    // their true alignment (of every batch member), which is below the 256
    // bytes it assumes by default
    auto align = [batch](const void* p, int64_t stride) {
      uint32_t a = 256;
      const uintptr_t step = batch > 1 ? static_cast<uintptr_t>(stride) * sizeof(float) : 0;
      while (a > 4 && (reinterpret_cast<uintptr_t>(p) % a || step % a)) a >>= 1;
      return a;
    };
    const uint32_t aA = align(B, sB), aB = align(A, sA), aC = align(C, sC);
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MIN_ALIGNMENT_A_BYTES, &aA, sizeof(aA));
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MIN_ALIGNMENT_B_BYTES, &aB, sizeof(aB));
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MIN_ALIGNMENT_C_BYTES, &aC, sizeof(aC));
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MIN_ALIGNMENT_D_BYTES, &aC, sizeof(aC));
    if (cublasLtMatmulAlgoGetHeuristic(lt, op, l1, l2, lc, lc, pref, 1, &heur, &found) !=
            CUBLAS_STATUS_SUCCESS || found < 1)
      rc = set_error(STCA_ECUDA, "cuBLASLt found no algorithm for a backward product");
  }
  if (rc == STCA_OK) {
    if (cublasLtMatmul(lt, op, &alpha, B, l1, A, l2, &beta, C, lc, C, lc, &heur.algo, H->lt_ws, kWs, s) !=
        CUBLAS_STATUS_SUCCESS)
      rc = set_error(STCA_ECUDA, "cuBLASLt backward product failed");
  }
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (l2) cublasLtMatrixLayoutDestroy(l2);
  if (l1) cublasLtMatrixLayoutDestroy(l1);
  if (op) cublasLtMatmulDescDestroy(op);
  return rc;
}

int ensure(void** p, size_t* cap, size_t bytes) {
  if (*cap >= bytes && *p) return STCA_OK;
  cudaFree(*p);
  *p = nullptr;
  *cap = 0;
  if (cudaMalloc(p, bytes) != cudaSuccess) {
    cudaGetLastError();
    return set_error(STCA_ENOMEM, "backward workspace allocation failed");
  }
  *cap = bytes;
  return STCA_OK;
}

}  // namespace
}  // namespace stca

using namespace stca;

namespace {

// The same backward for bf16 handles on the library's tensor-core GEMM, with
// bf16 intermediates: [A | G] = X [W_u | W_g] with H = A SiLU(G) formed in the
// GEMM's epilogue; Y = H W_d; the LayerNorm derivative (dy, also as bf16);
// dW_d = H^T dy; dH = dy W_d^T with the SwiGLU derivative in the epilogue
// (dA, dG over A, G); dW_u = X^T dA, dW_g = X^T dG; dX = [dA | dG] [W_u | W_g]^T,
// one product over K = 2 rd.  A and G share the rows of one N x 2 rd buffer
// (A in the first rd columns), so dA and dG are that product's left operand
// as they lie.  Products with K = N (the weight gradients) split K over CTAs.
int ffn_ln_backward16(stca_handle* H, const uint16_t* X, int64_t N, const float* dXt, float* dX,
                      const float* Wu, const float* Wg, const float* Wd, const float* gamma, float* dWu,
                      float* dWg, float* dWd, float* dgamma, float* dbeta, cudaStream_t s) {
  const int d = H->d, rd = H->rd;
  const size_t nd = static_cast<size_t>(N) * d, nr = static_cast<size_t>(N) * rd;
  const size_t wn = static_cast<size_t>(d) * rd;
  // workspace: AG (N x 2 rd bf16), H16 (N rd bf16), dy16 (N d bf16), Y (N d fp32), weights (6 d rd bf16)
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t oAG = 0, oH = a256(oAG + 2 * nr * 2), oDy = a256(oH + nr * 2);
  const size_t oY = a256(oDy + nd * 2), oW = a256(oY + nd * 4), total = a256(oW + 6 * wn * 2);
  if (int rc = ensure(&H->bw_ws, &H->bw_ws_cap, total)) return rc;
  char* w = static_cast<char*>(H->bw_ws);
  uint16_t* AG = reinterpret_cast<uint16_t*>(w + oAG);
  uint16_t* H16 = reinterpret_cast<uint16_t*>(w + oH);
  uint16_t* dy16 = reinterpret_cast<uint16_t*>(w + oDy);
  float* Y = reinterpret_cast<float*>(w + oY);
  uint16_t* W1i = reinterpret_cast<uint16_t*>(w + oW);      // 2 wn
  uint16_t* WdT = W1i + 2 * wn;
  uint16_t* Wd16 = WdT + wn;
  uint16_t* Wug = Wd16 + wn;                                  // d x 2 rd: [W_u | W_g]
  ffn_weights16_kernel<<<grid_for(static_cast<int64_t>(wn)), 256, 0, s>>>(Wu, Wg, Wd, W1i, WdT, Wd16, Wug,
                                                                          Wug + rd, d, rd);
  STCA_CUDA_TRY(cudaGetLastError());
  const int ns = H->num_sms;
  int* st = H->status_d;
  const int64_t ldag = 2 * static_cast<int64_t>(rd);
  // forward recomputation
  if (int rc = tc_gemm_bf16(false, true, N, 2 * rd, d, X, d, W1i, d, nullptr, 0, 0.f, 1, AG, AG + rd, H16, ldag,
                            rd, ns, st, s))
    return rc;
  if (int rc = tc_gemm_bf16(false, true, N, d, rd, H16, rd, WdT, rd, Y, d, 0.f, 0, nullptr, nullptr, nullptr, 0, 0,
                            ns, st, s))
    return rc;
  // LayerNorm: dy as bf16 (dy16); dgamma, dbeta
  STCA_CUDA_TRY(cudaMemsetAsync(dgamma, 0, d * sizeof(float), s));
  STCA_CUDA_TRY(cudaMemsetAsync(dbeta, 0, d * sizeof(float), s));
  ln_bwd_kernel<<<static_cast<unsigned>((N + kLnRows - 1) / kLnRows), 256, 0, s>>>(Y, dXt, gamma, dgamma,
                                                                                   dbeta, N, d, dy16);
  STCA_CUDA_TRY(cudaGetLastError());
  // dW_d = H^T dy
  if (int rc = tc_gemm_bf16(true, false, rd, d, N, H16, rd, dy16, d, dWd, d, 0.f, 0, nullptr, nullptr, nullptr, 0,
                            0, ns, st, s))
    return rc;
  // dH = dy W_d^T, then dA, dG over A, G
  if (int rc = tc_gemm_bf16(false, true, N, rd, d, dy16, d, Wd16, d, nullptr, 0, 0.f, 2, AG, AG + rd, nullptr,
                            ldag, 0, ns, st, s))
    return rc;
  // dW_u = X^T dA, dW_g = X^T dG
  if (int rc = tc_gemm_bf16(true, false, d, rd, N, X, d, AG, ldag, dWu, rd, 0.f, 0, nullptr, nullptr, nullptr, 0,
                            0, ns, st, s))
    return rc;
  if (int rc = tc_gemm_bf16(true, false, d, rd, N, X, d, AG + rd, ldag, dWg, rd, 0.f, 0, nullptr, nullptr, nullptr,
                            0, 0, ns, st, s))
    return rc;
  // dX = [dA | dG] [W_u | W_g]^T
  if (dX) {
    if (int rc = tc_gemm_bf16(false, true, N, d, 2 * rd, AG, ldag, Wug, ldag, dX, d, 0.f, 0, nullptr, nullptr,
                              nullptr, 0, 0, ns, st, s))
      return rc;
  }
  set_error(STCA_OK, "");
  return STCA_OK;
}

// Backward of Y = LN(((X W_u) * SiLU(X W_g)) W_d) with LN's scale gamma, for N
// rows of X (handle dtype): the history encoding of Eqs. (1)-(2) and, with the
// query weights, the query init of Eq. (3).  dX may be NULL.
int ffn_ln_backward(stca_handle* H, const void* X, int64_t N, const float* dXt, float* dX,
                    const float* Wu, const float* Wg, const float* Wd, const float* gamma, float* dWu,
                    float* dWg, float* dWd, float* dgamma, float* dbeta, cudaStream_t s) {
  const int d = H->d, rd = H->rd;
  if (d > 32 * kLnMaxCols) return set_error(STCA_EINVAL, "encoder backward needs d <= 256");
  // bf16 handles: the tensor-core pipeline, where its tiles fit the sizes
  if (H->elem == 2 && H->opt_bw_gemm != 1 && d % 64 == 0 && rd % 128 == 0 && N <= INT32_MAX)
    return ffn_ln_backward16(H, static_cast<const uint16_t*>(X), N, dXt, dX, Wu, Wg, Wd, gamma, dWu, dWg, dWd,
                             dgamma, dbeta, s);
  // workspace: Xf (N d), A (N rd), G (N rd), Hh (N rd), Y (N d)
  const size_t nd = static_cast<size_t>(N) * d, nr = static_cast<size_t>(N) * rd;
  if (int rc = ensure(&H->bw_ws, &H->bw_ws_cap, (2 * nd + 3 * nr) * sizeof(float))) return rc;
  float* Xf = static_cast<float*>(H->bw_ws);
  float* A = Xf + nd;
  float* G = A + nr;
  float* Hh = G + nr;
  float* Y = Hh + nr;
  if (H->elem == 2) {
    to_f32_kernel<<<grid_for(nd), 256, 0, s>>>(static_cast<const uint16_t*>(X), Xf, nd);
  } else {
    STCA_CUDA_TRY(cudaMemcpyAsync(Xf, X, nd * sizeof(float), cudaMemcpyDeviceToDevice, s));
  }
  // forward recomputation: A = X W_u, G = X W_g, H = A SiLU(G), Y = H W_d
  if (int rc = gemm_rm(H, false, false, N, rd, d, Xf, d, Wu, rd, A, rd, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, false, false, N, rd, d, Xf, d, Wg, rd, G, rd, 0.f, s)) return rc;
  swiglu_fwd_kernel<<<grid_for(nr), 256, 0, s>>>(A, G, Hh, nr);
  if (int rc = gemm_rm(H, false, false, N, d, rd, Hh, rd, Wd, d, Y, d, 0.f, s)) return rc;
  // LayerNorm: Y <- dy; dgamma, dbeta
  STCA_CUDA_TRY(cudaMemsetAsync(dgamma, 0, d * sizeof(float), s));
  STCA_CUDA_TRY(cudaMemsetAsync(dbeta, 0, d * sizeof(float), s));
  ln_bwd_kernel<<<static_cast<unsigned>((N + kLnRows - 1) / kLnRows), 256, 0, s>>>(Y, dXt, gamma, dgamma,
                                                                                   dbeta, N, d);
  // dW_d = H^T dy; dH = dy W_d^T (over H)
  if (int rc = gemm_rm(H, true, false, rd, d, N, Hh, rd, Y, d, dWd, d, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, false, true, N, rd, d, Y, d, Wd, d, Hh, rd, 0.f, s)) return rc;
  swiglu_bwd_kernel<<<grid_for(nr), 256, 0, s>>>(A, G, Hh, nr);
  // dW_u = X^T dA, dW_g = X^T dG; dX = dA W_u^T + dG W_g^T
  if (int rc = gemm_rm(H, true, false, d, rd, N, Xf, d, A, rd, dWu, rd, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, true, false, d, rd, N, Xf, d, G, rd, dWg, rd, 0.f, s)) return rc;
  if (dX) {
    if (int rc = gemm_rm(H, false, true, N, d, rd, A, rd, Wu, rd, dX, d, 0.f, s)) return rc;
    if (int rc = gemm_rm(H, false, true, N, d, rd, G, rd, Wg, rd, dX, d, 1.f, s)) return rc;
  }
  STCA_CUDA_TRY(cudaGetLastError());
  set_error(STCA_OK, "");
  return STCA_OK;
}

}  // namespace

extern "C" int stca_encode_backward(stca_handle* H, int layer, const void* X, int64_t N,
                                    const float* dXt, float* dX, float* dWu, float* dWg,
                                    float* dWd, float* dgamma, float* dbeta, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (layer < 0 || layer >= H->M) return set_error(STCA_EINVAL, "layer out of range");
  if (N < 1 || N > (int64_t(1) << 31)) return set_error(STCA_EINVAL, "N must be in [1, 2^31]");
  if (!X || !dXt || !dWu || !dWg || !dWd || !dgamma || !dbeta)
    return set_error(STCA_EINVAL, "stca_encode_backward: NULL argument");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != H->device) cudaSetDevice(H->device);
  const LayerW32& Wl = H->L32[layer];
  return ffn_ln_backward(H, X, N, dXt, dX, Wl.Wu, Wl.Wg, Wl.Wd, Wl.ln_g, dWu, dWg, dWd, dgamma, dbeta,
                         static_cast<cudaStream_t>(stream));
}

extern "C" int stca_query_init_backward(stca_handle* H, const void* targets, int64_t T, const float* dq,
                                        float* dxt, float* dWu, float* dWg, float* dWd, float* dgamma,
                                        float* dbeta, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (T < 1 || T > (int64_t(1) << 31)) return set_error(STCA_EINVAL, "T must be in [1, 2^31]");
  if (!targets || !dq || !dWu || !dWg || !dWd || !dgamma || !dbeta)
    return set_error(STCA_EINVAL, "stca_query_init_backward: NULL argument");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != H->device) cudaSetDevice(H->device);
  const LayerW32& W0 = H->L32[0];
  return ffn_ln_backward(H, targets, T, dq, dxt, W0.qWu, W0.qWg, W0.qWd, H->q_ln_g, dWu, dWg, dWd, dgamma,
                         dbeta, static_cast<cudaStream_t>(stream));
}

namespace {

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

// The tensor-core attention backward (attn_bw_tc.cu): the forward's work plan,
// bf16 copies of U (log2-scaled) and dC, the forward attention for c and the
// row statistics, delta = dC . c, then the backward kernel.
int attention_backward_tc(stca_handle* H, int layer, const float* U, const int64_t* toff, int64_t T,
                          const float* dC, float* dU, float* dXt, cudaStream_t s) {
  const int d = H->d, h = H->h;
  const int64_t R = H->R, N = H->N, rows = T * h;
  const int64_t* off = H->offsets_h.data();
  PlanHost P;
  build_plan_host(off, toff, R, h, 2, H->num_sms, 0, P, H->dh);
  if (int rc = check_plan(P, off, toff, R, h, 2)) return rc;
  bool split_pairs = false, shared_rows = false;
  for (size_t k = 0; k + 1 < P.pair_item_begin.size(); ++k)
    split_pairs |= P.pair_item_begin[k + 1] - P.pair_item_begin[k] > 1;
  for (int64_t r = 0; r < R; ++r) shared_rows |= P.req_pair_begin[r + 1] - P.req_pair_begin[r] != 1;
  const int64_t npairs = static_cast<int64_t>(P.pair_item_begin.size()) - 1;
  // plan arrays
  const size_t o_items = 0, o_cta = al256(P.items.size() * sizeof(AttnItem));
  const size_t o_pib = al256(o_cta + P.cta_begin.size() * sizeof(int32_t));
  const size_t o_rpb = al256(o_pib + P.pair_item_begin.size() * sizeof(int32_t));
  const size_t plan_bytes = al256(o_rpb + P.req_pair_begin.size() * sizeof(int32_t));
  if (int rc = ensure(&H->bw_plan, &H->bw_plan_cap, plan_bytes)) return rc;
  char* pl = static_cast<char*>(H->bw_plan);
  STCA_CUDA_TRY(cudaMemcpyAsync(pl + o_items, P.items.data(), P.items.size() * sizeof(AttnItem),
                                cudaMemcpyHostToDevice, s));
  STCA_CUDA_TRY(cudaMemcpyAsync(pl + o_cta, P.cta_begin.data(), P.cta_begin.size() * sizeof(int32_t),
                                cudaMemcpyHostToDevice, s));
  STCA_CUDA_TRY(cudaMemcpyAsync(pl + o_pib, P.pair_item_begin.data(),
                                P.pair_item_begin.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s));
  STCA_CUDA_TRY(cudaMemcpyAsync(pl + o_rpb, P.req_pair_begin.data(),
                                P.req_pair_begin.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s));
  // workspace: U', dC' (bf16), c, statistics, delta, the forward's partials and counters
  const size_t w_ub = 0, w_cb = al256(static_cast<size_t>(rows) * d * 2);
  const size_t w_c = al256(w_cb + static_cast<size_t>(rows) * d * 2);
  const size_t w_st = al256(w_c + static_cast<size_t>(rows) * d * 4);
  const size_t w_dl = al256(w_st + static_cast<size_t>(rows) * 2 * 4);
  const size_t w_part = al256(w_dl + static_cast<size_t>(rows) * 4);
  const size_t w_cnt = al256(w_part + static_cast<size_t>(std::max<int64_t>(P.G, 1)) * (d + 4) * 4);
  const size_t ws_bytes = al256(w_cnt + static_cast<size_t>(std::max<int64_t>(npairs, 1)) * 8 * 4);
  if (int rc = ensure(&H->bw_ws, &H->bw_ws_cap, ws_bytes)) return rc;
  char* w = static_cast<char*>(H->bw_ws);
  uint16_t* Ub = reinterpret_cast<uint16_t*>(w + w_ub);
  uint16_t* Cb = reinterpret_cast<uint16_t*>(w + w_cb);
  float* cbuf = reinterpret_cast<float*>(w + w_c);
  float* stats = reinterpret_cast<float*>(w + w_st);
  float* delta = reinterpret_cast<float*>(w + w_dl);
  float* part = reinterpret_cast<float*>(w + w_part);
  int* cnt = reinterpret_cast<int*>(w + w_cnt);
  CUtensorMap tmU, tmC;
  if (int rc = make_tmap_bf16_2d(&tmU, Ub, d, rows, 64, 128)) return rc;
  if (int rc = make_tmap_bf16_2d(&tmC, Cb, d, rows, 64, 128)) return rc;
  STCA_CUDA_TRY(cudaMemsetAsync(cnt, 0, static_cast<size_t>(std::max<int64_t>(npairs, 1)) * 8 * 4, s));
  launch_bw_prep(U, dC, Ub, Cb, rows * d, s);
  STCA_CUDA_TRY(cudaGetLastError());
  const AttnItem* items_d = reinterpret_cast<const AttnItem*>(pl + o_items);
  const int32_t* cta_d = reinterpret_cast<const int32_t*>(pl + o_cta);
  const int32_t* pib_d = reinterpret_cast<const int32_t*>(pl + o_pib);
  const int32_t* rpb_d = reinterpret_cast<const int32_t*>(pl + o_rpb);
  if (int rc = launch_attn_pp(d, tmU, H->tmXt[layer], items_d, cta_d, pib_d, P.grid, part, P.G, cbuf, cnt,
                              H->status_d, H->opt_stop_tiles, s, stats))
    return rc;
  launch_bw_delta(dC, cbuf, delta, rows, d, s);
  STCA_CUDA_TRY(cudaGetLastError());
  if (split_pairs) STCA_CUDA_TRY(cudaMemsetAsync(dU, 0, static_cast<size_t>(rows) * d * 4, s));
  // rows of requests without targets, or with several query tiles adding to them
  if (shared_rows) STCA_CUDA_TRY(cudaMemsetAsync(dXt, 0, static_cast<size_t>(N) * d * 4, s));
  if (int rc = launch_attn_bw_tc(d, tmU, tmC, H->tmXt[layer], items_d, cta_d, pib_d, rpb_d, P.grid, stats,
                                 delta, dU, dXt, H->status_d, H->opt_stop_tiles, s))
    return rc;
  // (the plan's copies are from pageable memory, which the runtime has staged
  // by the time each cudaMemcpyAsync returns)
  set_error(STCA_OK, "");
  return STCA_OK;
}

}  // namespace

extern "C" int stca_attention_backward(stca_handle* H, int layer, const float* U,
                                       const int64_t* target_offsets, int64_t T, const float* dC,
                                       float* dU, float* dXt, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (!H->encoded) return set_error(STCA_ESTATE, "stca_attention_backward before a successful stca_encode");
  if (layer < 0 || layer >= H->M) return set_error(STCA_EINVAL, "layer out of range");
  if (H->d != 64 && H->d != 128 && H->d != 256)
    return set_error(STCA_EINVAL, "attention backward needs d in {64, 128, 256}");
  if (int rc = stca_validate_offsets(target_offsets, H->R, T, 0)) return rc;
  if (!dXt || (T > 0 && (!U || !dC || !dU)))
    return set_error(STCA_EINVAL, "stca_attention_backward: NULL argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = H->d, h = H->h;
  const int64_t R = H->R, N = H->N;
  if (H->dtype == STCA_BF16 && attn_bw_tc_supported(d) && attn_pp_supported(d) && H->opt_attn_path != 1)
    return attention_backward_tc(H, layer, U, target_offsets, T, dC, dU, dXt, s);
  // work units and offsets, uploaded through the handle's backward plan buffer
  std::vector<BwUnit> rows, keys;
  std::vector<int64_t> offs(2 * (R + 1));
  for (int64_t r = 0; r <= R; ++r) {
    offs[r] = H->offsets_h[r];
    offs[R + 1 + r] = target_offsets[r] * h;
  }
  for (int64_t r = 0; r < R; ++r) {
    const int64_t q0 = target_offsets[r] * h, q1 = target_offsets[r + 1] * h;
    for (int64_t q = q0; q < q1; q += kBwBlock)
      rows.push_back({static_cast<int32_t>(r), static_cast<int32_t>(std::min<int64_t>(kBwBlock, q1 - q)), q});
    for (int64_t k = H->offsets_h[r]; k < H->offsets_h[r + 1]; k += kBwBlock)
      keys.push_back({static_cast<int32_t>(r),
                      static_cast<int32_t>(std::min<int64_t>(kBwBlock, H->offsets_h[r + 1] - k)), k});
  }
  const size_t b_off = offs.size() * sizeof(int64_t);
  const size_t b_rows = rows.size() * sizeof(BwUnit), b_keys = keys.size() * sizeof(BwUnit);
  const size_t bytes = b_off + b_rows + b_keys + static_cast<size_t>(std::max<int64_t>(T * h, 1)) * 3 * sizeof(float) + 64;
  if (int rc = ensure(&H->bw_plan, &H->bw_plan_cap, bytes)) return rc;
  char* p = static_cast<char*>(H->bw_plan);
  STCA_CUDA_TRY(cudaMemcpyAsync(p, offs.data(), b_off, cudaMemcpyHostToDevice, s));
  if (!rows.empty()) STCA_CUDA_TRY(cudaMemcpyAsync(p + b_off, rows.data(), b_rows, cudaMemcpyHostToDevice, s));
  if (!keys.empty())
    STCA_CUDA_TRY(cudaMemcpyAsync(p + b_off + b_rows, keys.data(), b_keys, cudaMemcpyHostToDevice, s));
  // the host vectors must outlive the copies: wait for them (a small upload)
  STCA_CUDA_TRY(cudaStreamSynchronize(s));
  AttnBwArgs a{};
  a.Xt = static_cast<const char*>(H->xt) + static_cast<size_t>(N) * d * H->elem * layer;
  a.xbf = H->elem == 2;
  a.U = U;
  a.dC = dC;
  a.dU = dU;
  a.dX = dXt;
  a.off = reinterpret_cast<const int64_t*>(p);
  a.qoff = a.off + R + 1;
  a.stats = reinterpret_cast<float*>(p + ((b_off + b_rows + b_keys + 15) & ~size_t(15)));
  a.d = d;
  auto run = [&](auto rows_k, auto keys_k) {
    if (!rows.empty()) {
      a.units = reinterpret_cast<const BwUnit*>(p + b_off);
      rows_k<<<static_cast<unsigned>(rows.size()), kBwThreads, kBwTile * d * sizeof(float), s>>>(a);
    }
    if (!keys.empty()) {
      a.units = reinterpret_cast<const BwUnit*>(p + b_off + b_rows);
      const size_t smem = static_cast<size_t>(kBwTile) * (2 * d + 3) * sizeof(float);
      cudaFuncSetAttribute(keys_k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      keys_k<<<static_cast<unsigned>(keys.size()), kBwThreads, smem, s>>>(a);
    }
  };
  if (d == 64) run(attn_bw_rows_kernel<8>, attn_bw_keys_kernel<8>);
  else if (d == 128) run(attn_bw_rows_kernel<16>, attn_bw_keys_kernel<16>);
  else run(attn_bw_rows_kernel<32>, attn_bw_keys_kernel<32>);
  STCA_CUDA_TRY(cudaGetLastError());
  set_error(STCA_OK, "");
  return STCA_OK;
}

namespace {

int projection_args(stca_handle* H, int layer, int64_t T, const void* a, const void* b,
                    const void* c, const void* w1, const void* w2, const char* who) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (layer < 0 || layer >= H->M) return set_error(STCA_EINVAL, "layer out of range");
  if (T < 0 || T > (int64_t(1) << 31)) return set_error(STCA_EINVAL, std::string(who) + ": T out of range");
  if (!w1 || !w2 || (T > 0 && (!a || !b || !c)))
    return set_error(STCA_EINVAL, std::string(who) + ": NULL argument");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != H->device) cudaSetDevice(H->device);
  return STCA_OK;
}

}  // namespace

extern "C" int stca_output_backward(stca_handle* H, int layer, const float* C, int64_t T,
                                    const float* dZ, float* dC, float* dWv, float* dWo, void* stream) {
  if (int rc = projection_args(H, layer, T, C, dZ, dC, dWv, dWo, "stca_output_backward")) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = H->d, h = H->h, dh = d / h;
  const size_t dd = static_cast<size_t>(d) * d;
  if (T == 0) {
    STCA_CUDA_TRY(cudaMemsetAsync(dWv, 0, dd * sizeof(float), s));
    STCA_CUDA_TRY(cudaMemsetAsync(dWo, 0, dd * sizeof(float), s));
    set_error(STCA_OK, "");
    return STCA_OK;
  }
  const LayerW32& Wl = H->L32[layer];
  // workspace: Oh = the heads' c_j W_V^j side by side (T x d), dOh = dZ W_O^T (T x d)
  const size_t td = static_cast<size_t>(T) * d;
  if (int rc = ensure(&H->bw_ws, &H->bw_ws_cap, 2 * td * sizeof(float))) return rc;
  float* Oh = static_cast<float*>(H->bw_ws);
  float* dOh = Oh + td;
  const int64_t hd = static_cast<int64_t>(h) * d;
  // per head j (one batched product each): operands step by d (C_j), d_h (column slices)
  // Oh[:, j] = C_j W_V[:, j]   (T x d_h)
  if (int rc = gemm_rm(H, false, false, T, dh, d, C, hd, Wl.Wv, d, Oh, d, 0.f, s, 1.f, h, d, dh, dh))
    return rc;
  // dW_O = Oh^T dZ, dOh = dZ W_O^T
  if (int rc = gemm_rm(H, true, false, d, d, T, Oh, d, dZ, d, dWo, d, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, false, true, T, d, d, dZ, d, Wl.Wo, d, dOh, d, 0.f, s)) return rc;
  // dC_j = dOh[:, j] W_V[:, j]^T  (T x d),  dW_V[:, j] = C_j^T dOh[:, j]  (d x d_h)
  if (int rc = gemm_rm(H, false, true, T, d, dh, dOh, d, Wl.Wv, d, dC, hd, 0.f, s, 1.f, h, dh, dh, d))
    return rc;
  if (int rc = gemm_rm(H, true, false, d, dh, T, C, hd, dOh, d, dWv, d, 0.f, s, 1.f, h, d, dh, dh))
    return rc;
  STCA_CUDA_TRY(cudaGetLastError());
  set_error(STCA_OK, "");
  return STCA_OK;
}

extern "C" int stca_query_backward(stca_handle* H, int layer, const float* Q, int64_t T,
                                   const float* dU, float* dQ, float* dWq, float* dWk, void* stream) {
  if (int rc = projection_args(H, layer, T, Q, dU, dQ, dWq, dWk, "stca_query_backward")) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = H->d, h = H->h, dh = d / h;
  const size_t dd = static_cast<size_t>(d) * d;
  if (T == 0) {
    STCA_CUDA_TRY(cudaMemsetAsync(dWq, 0, dd * sizeof(float), s));
    STCA_CUDA_TRY(cudaMemsetAsync(dWk, 0, dd * sizeof(float), s));
    set_error(STCA_OK, "");
    return STCA_OK;
  }
  const LayerW32& Wl = H->L32[layer];
  const float scale = 1.f / std::sqrt(static_cast<float>(dh));
  // workspace: P = Q W_Q (T x d, head j on columns j d_h ..), dP (T x d)
  const size_t td = static_cast<size_t>(T) * d;
  if (int rc = ensure(&H->bw_ws, &H->bw_ws_cap, 2 * td * sizeof(float))) return rc;
  float* P = static_cast<float*>(H->bw_ws);
  float* dP = P + td;
  const int64_t hd = static_cast<int64_t>(h) * d;
  if (int rc = gemm_rm(H, false, false, T, d, d, Q, d, Wl.Wq, d, P, d, 0.f, s)) return rc;
  // per head j, batched: W_K^j is stored transposed, WkT[j] (d_h x d) = W_K[:, j]^T,
  // WkT[j] = WkT + j d_h d.  dP[:, j] = scale dU_j W_K^j   (T x d_h)
  const int64_t wk_step = static_cast<int64_t>(dh) * d;
  if (int rc = gemm_rm(H, false, true, T, dh, d, dU, hd, Wl.WkT, d, dP, d, 0.f, s, scale, h, d, wk_step, dh))
    return rc;
  // dW_K[:, j] = scale dU_j^T P[:, j]   (d x d_h)
  if (int rc = gemm_rm(H, true, false, d, dh, T, dU, hd, P, d, dWk, d, 0.f, s, scale, h, d, dh, dh))
    return rc;
  // dQ = dP W_Q^T, dW_Q = Q^T dP
  if (int rc = gemm_rm(H, false, true, T, d, d, dP, d, Wl.Wq, d, dQ, d, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, true, false, d, d, T, Q, d, dP, d, dWq, d, 0.f, s)) return rc;
  STCA_CUDA_TRY(cudaGetLastError());
  set_error(STCA_OK, "");
  return STCA_OK;
}

extern "C" int stca_fusion_backward(stca_handle* H, int block, const float* Z, const void* targets, int64_t T,
                                    const float* dy, int accumulate, float* dZ, float* dxt, float* dW,
                                    float* dWu, float* dWg, float* dWd, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (block < 1 || block > H->M) return set_error(STCA_EINVAL, "block must be in [1, M]");
  if (block == H->M && !H->hWz32)
    return set_error(STCA_EINVAL, "block M is the prediction head: the handle has no head weights");
  if (T < 0 || T > (int64_t(1) << 31)) return set_error(STCA_EINVAL, "T out of range");
  if (!dW || !dWu || !dWg || !dWd || (T > 0 && (!Z || !targets || !dy || !dZ || !dxt)))
    return set_error(STCA_EINVAL, "stca_fusion_backward: NULL argument");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != H->device) cudaSetDevice(H->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = H->d, rd = H->rd, M = H->M;
  const int64_t bd = static_cast<int64_t>(block) * d, Md = static_cast<int64_t>(M) * d;
  // block b < M: W_C of layer b+1 (0-based b) with that layer's query FFN (Eq. (7));
  // block M: W_Z with the head's FFN (Eq. (9))
  const bool head = block == M;
  const float* W = head ? H->hWz32 : H->L32[block].Wc;
  const float* Wu = head ? H->hWu32 : H->L32[block].qWu;
  const float* Wg = head ? H->hWg32 : H->L32[block].qWg;
  const float* Wd = head ? H->hWd32 : H->L32[block].qWd;
  if (T == 0) {
    STCA_CUDA_TRY(cudaMemsetAsync(dW, 0, static_cast<size_t>(bd + d) * d * sizeof(float), s));
    STCA_CUDA_TRY(cudaMemsetAsync(dWu, 0, static_cast<size_t>(d) * rd * sizeof(float), s));
    STCA_CUDA_TRY(cudaMemsetAsync(dWg, 0, static_cast<size_t>(d) * rd * sizeof(float), s));
    STCA_CUDA_TRY(cudaMemsetAsync(dWd, 0, static_cast<size_t>(rd) * d * sizeof(float), s));
    set_error(STCA_OK, "");
    return STCA_OK;
  }
  // workspace: xf (T d), a (T d), da (T d), A, G, Hh (T rd each)
  const size_t nd = static_cast<size_t>(T) * d, nr = static_cast<size_t>(T) * rd;
  if (int rc = ensure(&H->bw_ws, &H->bw_ws_cap, (3 * nd + 3 * nr) * sizeof(float))) return rc;
  float* xf = static_cast<float*>(H->bw_ws);
  float* a = xf + nd;
  float* da = a + nd;
  float* A = da + nd;
  float* G = A + nr;
  float* Hh = G + nr;
  if (H->elem == 2) {
    to_f32_kernel<<<grid_for(nd), 256, 0, s>>>(static_cast<const uint16_t*>(targets), xf, nd);
  } else {
    STCA_CUDA_TRY(cudaMemcpyAsync(xf, targets, nd * sizeof(float), cudaMemcpyDeviceToDevice, s));
  }
  const float* Wx = W + bd * d;           // the rows of W that multiply x_t (the last block)
  // a = [o^(1) .. o^(b)] W[:b d] + x_t W[b d:]: the first b d columns of each Z row, then x_t
  if (int rc = gemm_rm(H, false, false, T, d, bd, Z, Md, W, d, a, d, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, false, false, T, d, d, xf, d, Wx, d, a, d, 1.f, s)) return rc;
  // the FFN forward recomputed: A = a W_u, G = a W_g, H = A SiLU(G)
  if (int rc = gemm_rm(H, false, false, T, rd, d, a, d, Wu, rd, A, rd, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, false, false, T, rd, d, a, d, Wg, rd, G, rd, 0.f, s)) return rc;
  swiglu_fwd_kernel<<<grid_for(nr), 256, 0, s>>>(A, G, Hh, nr);
  // dW_d = H^T dy; dH = dy W_d^T (over H); dA, dG (over A, G)
  if (int rc = gemm_rm(H, true, false, rd, d, T, Hh, rd, dy, d, dWd, d, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, false, true, T, rd, d, dy, d, Wd, d, Hh, rd, 0.f, s)) return rc;
  swiglu_bwd_kernel<<<grid_for(nr), 256, 0, s>>>(A, G, Hh, nr);
  // dW_u = a^T dA, dW_g = a^T dG, da = dA W_u^T + dG W_g^T
  if (int rc = gemm_rm(H, true, false, d, rd, T, a, d, A, rd, dWu, rd, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, true, false, d, rd, T, a, d, G, rd, dWg, rd, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, false, true, T, d, rd, A, rd, Wu, rd, da, d, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, false, true, T, d, rd, G, rd, Wg, rd, da, d, 1.f, s)) return rc;
  // dW = [Z[:, :b d] || x_t]^T da, by its two row blocks
  if (int rc = gemm_rm(H, true, false, bd, d, T, Z, Md, da, d, dW, d, 0.f, s)) return rc;
  if (int rc = gemm_rm(H, true, false, d, d, T, xf, d, da, d, dW + bd * d, d, 0.f, s)) return rc;
  // d[o^(1) .. o^(b)] = da W[:b d]^T into the first b d columns of dZ; dx_t = da W[b d:]^T
  const float beta = accumulate ? 1.f : 0.f;
  if (int rc = gemm_rm(H, false, true, T, bd, d, da, d, W, d, dZ, Md, beta, s)) return rc;
  if (int rc = gemm_rm(H, false, true, T, d, d, da, d, Wx, d, dxt, d, beta, s)) return rc;
  STCA_CUDA_TRY(cudaGetLastError());
  set_error(STCA_OK, "");
  return STCA_OK;
}
