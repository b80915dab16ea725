// CUDA-core kernels of the STCA forward: the row-wise SwiGLU+LayerNorm encoder
// and the split-L single-query attention.  They run the fp32 configuration
// (where tensor-core TF32 would not hold the 1e-3 bound) and the sizes the
// tensor-core kernels do not cover.  Sources: "Make
// It Long, Keep It Fast" digest §2.1, Eqs. (1)-(8) and (13).
#include <cuda_bf16.h>
#include <math.h>

#include "stca_internal.h"

namespace stca {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

template <bool BF>
__device__ __forceinline__ float ld_elem(const void* p, int64_t i) {
  if constexpr (BF) return bf16_to_f32(static_cast<const uint16_t*>(p)[i]);
  else return static_cast<const float*>(p)[i];
}

template <bool BF>
__device__ __forceinline__ void st_elem(void* p, int64_t i, float v) {
  if constexpr (BF) static_cast<uint16_t*>(p)[i] = f32_to_bf16(v);
  else static_cast<float*>(p)[i] = v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// SiLU(z) = z * sigmoid(z) with the accurate expf (CUDA-core path).
__device__ __forceinline__ float silu_acc(float z) { return z / (1.0f + expf(-z)); }

// ------------------------------------------------------------------ encoder
// Y[row] = LN?(((x W_u) * SiLU(x W_g)) W_d) for a block of kFfnRows rows.
// Eq. (1)-(2) (history) and Eq. (3) (query init).
constexpr int kFfnRows = 16;
constexpr int kFfnChunk = 64;

template <bool XBF, bool YBF, bool LN>
__global__ void __launch_bounds__(kThreads)
ffn_rows_kernel(const void* __restrict__ X, int64_t nrows, const float* __restrict__ Wu,
                const float* __restrict__ Wg, const float* __restrict__ Wd,
                const float* __restrict__ ln_g, const float* __restrict__ ln_b,
                void* __restrict__ Y, int d, int rd) {
  extern __shared__ float sm[];
  float* xs = sm;                       // kFfnRows x d
  float* ys = xs + kFfnRows * d;        // kFfnRows x d
  float* hs = ys + kFfnRows * d;        // kFfnRows x kFfnChunk
  const int tid = threadIdx.x;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kFfnRows;
  const int nr = nrows - row0 < kFfnRows ? static_cast<int>(nrows - row0) : kFfnRows;
  for (int e = tid; e < kFfnRows * d; e += kThreads) {
    const int rr = e / d, c = e - rr * d;
    xs[e] = rr < nr ? ld_elem<XBF>(X, (row0 + rr) * d + c) : 0.f;
    ys[e] = 0.f;
  }
  __syncthreads();
  const int c = tid & (kFfnChunk - 1), rg = tid / kFfnChunk;   // 4 row groups of 4 rows
  for (int h0 = 0; h0 < rd; h0 += kFfnChunk) {
    float au[4] = {0.f, 0.f, 0.f, 0.f}, ag[4] = {0.f, 0.f, 0.f, 0.f};
    const int hc = h0 + c;
    if (hc < rd) {
      for (int k = 0; k < d; ++k) {
        const float wu = Wu[static_cast<int64_t>(k) * rd + hc];
        const float wg = Wg[static_cast<int64_t>(k) * rd + hc];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float x = xs[(rg * 4 + q) * d + k];
          au[q] = fmaf(x, wu, au[q]);
          ag[q] = fmaf(x, wg, ag[q]);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      hs[(rg * 4 + q) * kFfnChunk + c] = hc < rd ? au[q] * silu_acc(ag[q]) : 0.f;
    __syncthreads();
    const int kmax = min(kFfnChunk, rd - h0);
    for (int e = tid; e < kFfnRows * d; e += kThreads) {
      const int rr = e / d, n = e - rr * d;
      float acc = ys[e];
      for (int k = 0; k < kmax; ++k)
        acc = fmaf(hs[rr * kFfnChunk + k], Wd[static_cast<int64_t>(h0 + k) * d + n], acc);
      ys[e] = acc;
    }
    __syncthreads();
  }
  const int warp = tid >> 5, lane = tid & 31;
  for (int rr = warp; rr < nr; rr += kThreads / 32) {
    const float* y = ys + rr * d;
    float mean = 0.f, rstd = 1.f;
    if (LN) {
      float s = 0.f;
      for (int k = lane; k < d; k += 32) s += y[k];
      mean = warp_sum(s) / d;
      float v = 0.f;
      for (int k = lane; k < d; k += 32) { const float t = y[k] - mean; v = fmaf(t, t, v); }
      rstd = 1.0f / sqrtf(warp_sum(v) / d + 1e-5f);
    }
    for (int k = lane; k < d; k += 32) {
      const float o = LN ? (y[k] - mean) * rstd * ln_g[k] + ln_b[k] : y[k];
      st_elem<YBF>(Y, (row0 + rr) * d + k, o);
    }
  }
}

// ---------------------------------------------------------------- attention
// One CTA per (work item, target): the target's h scaled query rows u_j
// (Eq. (13)) against the item's key range, online softmax per head, partial
// (max, sum, sum p * x~) written for the split combine.
constexpr int kAttnWarps = 4;
constexpr int kMaxPerLane = 32;   // d <= 1024

template <bool XBF>
__global__ void __launch_bounds__(kAttnWarps * 32)
attn_simt_kernel(const void* __restrict__ Xt, const float* __restrict__ U,
                 const AttnItem* __restrict__ items, const int32_t* __restrict__ pairs,
                 const int64_t* __restrict__ toff, float* __restrict__ pacc,
                 float* __restrict__ pm, float* __restrict__ pl, int d, int h) {
  extern __shared__ float sm[];
  float* us = sm;                                  // h x d
  float* acc = us + h * d;                         // warps x h x d
  float* ms = acc + kAttnWarps * h * d;            // warps x h
  float* ls = ms + kAttnWarps * h;                 // warps x h
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int w_item = pairs[2 * blockIdx.x], tl = pairs[2 * blockIdx.x + 1];
  const AttnItem it = items[w_item];
  const int64_t t = toff[it.req] + tl;
  for (int e = tid; e < h * d; e += blockDim.x) us[e] = U[t * h * d + e];
  for (int e = tid; e < kAttnWarps * h * d; e += blockDim.x) acc[e] = 0.f;
  for (int e = tid; e < kAttnWarps * h; e += blockDim.x) { ms[e] = -INFINITY; ls[e] = 0.f; }
  __syncthreads();
  const int nper = (d + 31) / 32;
  float* wacc = acc + warp * h * d;
  float* wm = ms + warp * h;
  float* wl = ls + warp * h;
  for (int key = warp; key < it.nkeys; key += kAttnWarps) {
    const int64_t row = it.key0 + key;
    float xv[kMaxPerLane];
#pragma unroll
    for (int e = 0; e < kMaxPerLane; ++e)
      xv[e] = (e < nper && lane + 32 * e < d) ? ld_elem<XBF>(Xt, row * d + lane + 32 * e) : 0.f;
    for (int j = 0; j < h; ++j) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < kMaxPerLane; ++e)
        if (e < nper && lane + 32 * e < d) s = fmaf(us[j * d + lane + 32 * e], xv[e], s);
      s = warp_sum(s);
      const float mo = wm[j];
      const float mn = fmaxf(mo, s);
      const float corr = expf(mo - mn);
      const float p = expf(s - mn);
#pragma unroll
      for (int e = 0; e < kMaxPerLane; ++e)
        if (e < nper && lane + 32 * e < d) {
          float* a = wacc + j * d + lane + 32 * e;
          *a = fmaf(*a, corr, p * xv[e]);
        }
      __syncwarp();
      if (lane == 0) { wm[j] = mn; wl[j] = fmaf(wl[j], corr, p); }
      __syncwarp();
    }
  }
  __syncthreads();
  // merge the warps' states and write this item's partial rows
  for (int e = tid; e < h * d; e += blockDim.x) {
    const int j = e / d, k = e - j * d;
    float mx = -INFINITY;
    for (int w = 0; w < kAttnWarps; ++w) mx = fmaxf(mx, ms[w * h + j]);
    float a = 0.f, l = 0.f;
    for (int w = 0; w < kAttnWarps; ++w) {
      const float f = expf(ms[w * h + j] - mx);   // warps with no key: exp(-inf) = 0
      a = fmaf(acc[(w * h + j) * d + k], f, a);
      l = fmaf(ls[w * h + j], f, l);
    }
    const int64_t g = it.row_base + static_cast<int64_t>(tl) * h + j;
    pacc[g * d + k] = a;
    if (k == 0) { pm[g] = mx; pl[g] = l; }
  }
}

}  // namespace

// ------------------------------------------------------------------ launchers
void launch_ffn_rows(const void* X, int x_is_bf16, int64_t nrows, const LayerW32& w,
                     bool history_ffn, const float* ln_g, const float* ln_b, void* Y,
                     int y_is_bf16, int d, int rd, cudaStream_t s) {
  if (nrows <= 0) return;
  const float* Wu = history_ffn ? w.Wu : w.qWu;
  const float* Wg = history_ffn ? w.Wg : w.qWg;
  const float* Wd = history_ffn ? w.Wd : w.qWd;
  const size_t smem = (2 * kFfnRows * d + kFfnRows * kFfnChunk) * sizeof(float);
  const unsigned grid = static_cast<unsigned>((nrows + kFfnRows - 1) / kFfnRows);
  const bool ln = ln_g != nullptr;
#define STCA_FFN(XB, YB, LNB)                                                                \
  do {                                                                                       \
    auto k = ffn_rows_kernel<XB, YB, LNB>;                                                   \
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
    k<<<grid, kThreads, smem, s>>>(X, nrows, Wu, Wg, Wd, ln_g, ln_b, Y, d, rd);              \
  } while (0)
  if (x_is_bf16) {
    if (y_is_bf16) { if (ln) STCA_FFN(true, true, true); else STCA_FFN(true, true, false); }
    else { if (ln) STCA_FFN(true, false, true); else STCA_FFN(true, false, false); }
  } else {
    if (y_is_bf16) { if (ln) STCA_FFN(false, true, true); else STCA_FFN(false, true, false); }
    else { if (ln) STCA_FFN(false, false, true); else STCA_FFN(false, false, false); }
  }
#undef STCA_FFN
}

size_t attn_simt_smem(const stca_handle* H) {
  return (static_cast<size_t>(H->h) * H->d * (1 + kAttnWarps) + 2 * kAttnWarps * H->h) *
         sizeof(float);
}

void launch_attn_simt(const stca_handle* H, int layer, const void* xt_layer,
                      const AttnItem* items_d, const int32_t* pairs_d, int64_t npairs,
                      const int64_t* toff_d, cudaStream_t s) {
  (void)layer;
  if (npairs <= 0) return;
  const size_t smem = attn_simt_smem(H);
  const int64_t G = H->last_G;
  float* pacc = H->part;
  float* pm = pacc + G * H->d;
  float* pl = pm + G;
  if (H->elem == 2) {
    cudaFuncSetAttribute(attn_simt_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    attn_simt_kernel<true><<<static_cast<unsigned>(npairs), kAttnWarps * 32, smem, s>>>(
        xt_layer, H->U, items_d, pairs_d, toff_d, pacc, pm, pl, H->d, H->h);
  } else {
    cudaFuncSetAttribute(attn_simt_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    attn_simt_kernel<false><<<static_cast<unsigned>(npairs), kAttnWarps * 32, smem, s>>>(
        xt_layer, H->U, items_d, pairs_d, toff_d, pacc, pm, pl, H->d, H->h);
  }
}

}  // namespace stca
