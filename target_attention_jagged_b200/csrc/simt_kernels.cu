// CUDA-core kernels of the STCA forward: the row-wise SwiGLU+LayerNorm encoder,
// the split-L single-query attention and the per-target step (split combine,
// W_V / W_O epilogue, Eq. (7) query fusion, the u = (q W_Q) W_K^T projection).
//
// These run the fp32 configuration (where tensor-core TF32 would not hold the
// 1e-3 bound) and the per-target work of every configuration.  Sources: "Make
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

// ---------------------------------------------------------------- per-target
// The per-target step after layer `layer`'s attention (layer >= 0): merge the
// split partials into c_j = alpha_j X~ (Eq. (13)), o = [c_j W_V^j]_j W_O (Eq. (6)),
// Z[t, layer, :] = o (Eq. (8)); then, unless layer is the last, the Eq. (7)
// query fusion of layer+1 and its u projection.  layer == -1 computes
// q(1) = LN(FFN_1(x_t)) (Eq. (3)) and the u projection of layer 0.
constexpr int kTB = 4;   // targets per CTA

struct StepArgs {
  int layer, M, d, h, dh, rd;
  int64_t T;
  const void* targets;
  StepPlan plan;
  const float *pacc, *pm, *pl;
  float* Z;
  float* U;
  uint16_t* Ubf;      // optional bf16 copy of U (tensor-core attention)
  float uscale;       // folded into U: 1/sqrt(d_h), times log2(e) for exp2 kernels
  LayerW32 cur, nxt;  // weights of `layer` (post) and `layer+1` (prep)
  const float *q_ln_g, *q_ln_b;
  int wa;             // width of buffer A per target
  int wb;             // width of buffer B per target
};

// out[b][c] = sum_k in[b][k] * W[k][c] for c < n, b < nb.
__device__ __forceinline__ void rows_matmul(const float* in, int ldin, int K, const float* W,
                                            int64_t ldw, float* out, int ldout, int n, int nb) {
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    float acc[kTB];
#pragma unroll
    for (int b = 0; b < kTB; ++b) acc[b] = 0.f;
    for (int k = 0; k < K; ++k) {
      const float w = W[static_cast<int64_t>(k) * ldw + c];
#pragma unroll
      for (int b = 0; b < kTB; ++b) acc[b] = fmaf(in[b * ldin + k], w, acc[b]);
    }
    for (int b = 0; b < nb; ++b) out[b * ldout + c] = acc[b];
  }
}

// x (nb rows of width d in `in`) -> SwiGLU FFN -> out (width d); scratch: 2rd + rd.
__device__ void rows_ffn(const float* in, int ldin, const float* Wu, const float* Wg,
                         const float* Wd, float* tmp2, float* tmp1, float* out, int ldout,
                         int d, int rd, int nb) {
  rows_matmul(in, ldin, d, Wu, rd, tmp2, 2 * rd, rd, nb);
  rows_matmul(in, ldin, d, Wg, rd, tmp2 + rd, 2 * rd, rd, nb);
  __syncthreads();
  for (int e = threadIdx.x; e < nb * rd; e += blockDim.x) {
    const int b = e / rd, c = e - b * rd;
    tmp1[b * rd + c] = tmp2[b * 2 * rd + c] * silu_acc(tmp2[b * 2 * rd + rd + c]);
  }
  __syncthreads();
  rows_matmul(tmp1, rd, rd, Wd, d, out, ldout, d, nb);
  __syncthreads();
}

template <bool XBF>
__global__ void __launch_bounds__(kThreads) target_step_kernel(StepArgs a) {
  extern __shared__ float sm[];
  const int d = a.d, h = a.h, dh = a.dh, rd = a.rd;
  float* xs = sm;                       // kTB x d: raw x_t
  float* A = xs + kTB * d;              // kTB x wa
  float* B = A + kTB * a.wa;            // kTB x wb
  float* C = B + kTB * a.wb;            // kTB x d
  float* D = C + kTB * d;               // kTB x 2rd, then kTB x rd (FFN scratch)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTB;
  const int nb = a.T - t0 < kTB ? static_cast<int>(a.T - t0) : kTB;
  for (int e = tid; e < kTB * d; e += blockDim.x) {
    const int b = e / d, k = e - b * d;
    xs[e] = b < nb ? ld_elem<XBF>(a.targets, (t0 + b) * d + k) : 0.f;
  }
  __syncthreads();
  const int layer = a.layer;
  if (layer >= 0) {
    // split combine: c_j = sum_w e^{m_w - m} acc_w / sum_w e^{m_w - m} l_w
    const StepPlan& P = a.plan;
    for (int pr = warp; pr < nb * h; pr += blockDim.x / 32) {
      const int b = pr / h, j = pr - b * h;
      const int64_t t = t0 + b;
      const int r = P.treq[t];
      const int64_t qrow = (t - P.toff[r]) * h + j;
      const int64_t mt = qrow / P.mtile_rows;
      const int64_t row = qrow - mt * P.mtile_rows;
      const int pair = P.req_pair_begin[r] + static_cast<int>(mt);
      const int w0 = P.pair_item_begin[pair], w1 = P.pair_item_begin[pair + 1];
      float mx = -INFINITY;
      for (int w = w0; w < w1; ++w) mx = fmaxf(mx, a.pm[P.items[w].row_base + row]);
      float l = 0.f;
      for (int w = w0; w < w1; ++w) {
        const int64_t g = P.items[w].row_base + row;
        const float f = P.log2_partials ? exp2f(a.pm[g] - mx) : expf(a.pm[g] - mx);
        l = fmaf(a.pl[g], f, l);
      }
      const float inv = 1.0f / l;
      for (int k = lane; k < d; k += 32) {
        float v = 0.f;
        for (int w = w0; w < w1; ++w) {
          const int64_t g = P.items[w].row_base + row;
          const float f = P.log2_partials ? exp2f(a.pm[g] - mx) : expf(a.pm[g] - mx);
          v = fmaf(a.pacc[g * d + k], f, v);
        }
        A[b * a.wa + j * d + k] = v * inv;
      }
    }
    __syncthreads();
    // o_head[b][j dh + c] = sum_k c_j[k] W_V[k][j dh + c]
    for (int cc = tid; cc < d; cc += blockDim.x) {
      const int j = cc / dh;
      float acc[kTB];
#pragma unroll
      for (int b = 0; b < kTB; ++b) acc[b] = 0.f;
      for (int k = 0; k < d; ++k) {
        const float w = a.cur.Wv[static_cast<int64_t>(k) * d + cc];
#pragma unroll
        for (int b = 0; b < kTB; ++b) acc[b] = fmaf(A[b * a.wa + j * d + k], w, acc[b]);
      }
      for (int b = 0; b < nb; ++b) B[b * a.wb + cc] = acc[b];
    }
    __syncthreads();
    rows_matmul(B, a.wb, d, a.cur.Wo, d, C, d, d, nb);
    __syncthreads();
    for (int e = tid; e < nb * d; e += blockDim.x) {
      const int b = e / d, k = e - b * d;
      a.Z[((t0 + b) * a.M + layer) * d + k] = C[b * d + k];
    }
    __syncthreads();
    if (layer + 1 >= a.M) return;
    // Eq. (7): [o(1) || ... || o(layer+1) || x_t] W_C^(layer+2)
    const int wcat = (layer + 2) * d;
    for (int e = tid; e < nb * wcat; e += blockDim.x) {
      const int b = e / wcat, k = e - b * wcat;
      const int blk = k / d, kk = k - blk * d;
      float v;
      if (blk < layer) v = a.Z[((t0 + b) * a.M + blk) * d + kk];
      else if (blk == layer) v = C[b * d + kk];
      else v = xs[b * d + kk];
      A[b * a.wa + k] = v;
    }
    __syncthreads();
    rows_matmul(A, a.wa, wcat, a.nxt.Wc, d, B, a.wb, d, nb);
    __syncthreads();
    rows_ffn(B, a.wb, a.nxt.qWu, a.nxt.qWg, a.nxt.qWd, D, D + kTB * 2 * rd, C, d, d, rd, nb);
  } else {
    rows_ffn(xs, d, a.nxt.qWu, a.nxt.qWg, a.nxt.qWd, D, D + kTB * 2 * rd, C, d, d, rd, nb);
    // LayerNorm of Eq. (3)
    for (int b = warp; b < nb; b += blockDim.x / 32) {
      float s = 0.f;
      for (int k = lane; k < d; k += 32) s += C[b * d + k];
      const float mean = warp_sum(s) / d;
      float v = 0.f;
      for (int k = lane; k < d; k += 32) { const float u = C[b * d + k] - mean; v = fmaf(u, u, v); }
      const float rstd = 1.0f / sqrtf(warp_sum(v) / d + 1e-5f);
      __syncwarp();
      for (int k = lane; k < d; k += 32)
        C[b * d + k] = (C[b * d + k] - mean) * rstd * a.q_ln_g[k] + a.q_ln_b[k];
    }
    __syncthreads();
  }
  // P = q W_Q of the next layer; u_j = P_j W_K^j^T, scaled (Eq. (13))
  rows_matmul(C, d, d, a.nxt.Wq, d, B, a.wb, d, nb);
  __syncthreads();
  for (int cc = tid; cc < h * d; cc += blockDim.x) {
    const int j = cc / d, k = cc - j * d;
    float acc[kTB];
#pragma unroll
    for (int b = 0; b < kTB; ++b) acc[b] = 0.f;
    const float* wk = a.nxt.WkT + static_cast<int64_t>(j) * dh * d + k;
    for (int c = 0; c < dh; ++c) {
      const float w = wk[static_cast<int64_t>(c) * d];
#pragma unroll
      for (int b = 0; b < kTB; ++b) acc[b] = fmaf(B[b * a.wb + j * dh + c], w, acc[b]);
    }
    for (int b = 0; b < nb; ++b) {
      const float u = acc[b] * a.uscale;
      const int64_t gi = (t0 + b) * h * d + cc;
      if (a.U) a.U[gi] = u;
      if (a.Ubf) a.Ubf[gi] = f32_to_bf16(u);
    }
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

static void step_widths(const stca_handle* H, int* wa, int* wb) {
  const int d = H->d;
  *wa = std::max(std::max(H->h * d, (H->M + 1) * d), d);
  *wb = d;
}

size_t target_step_smem(const stca_handle* H) {
  int wa, wb;
  step_widths(H, &wa, &wb);
  return static_cast<size_t>(kTB) * (H->d + wa + wb + H->d + 3 * H->rd) * sizeof(float);
}

void launch_target_step(const stca_handle* H, int layer, const void* targets, int64_t T,
                        const StepPlan& plan, float* Z, cudaStream_t s) {
  if (T <= 0) return;
  StepArgs a{};
  a.layer = layer;
  a.M = H->M; a.d = H->d; a.h = H->h; a.dh = H->dh; a.rd = H->rd;
  a.T = T;
  a.targets = targets;
  a.plan = plan;
  const int64_t G = H->last_G;
  a.pacc = H->part;
  a.pm = H->part + G * H->d;
  a.pl = a.pm + G;
  a.Z = Z;
  const bool tc = plan.log2_partials != 0;
  a.U = tc ? nullptr : H->U;
  a.Ubf = tc ? H->Ubf : nullptr;
  // fold 1/sqrt(d_h) (and log2(e) for the exp2-based tensor-core kernel) into u
  a.uscale = (tc ? 1.4426950408889634f : 1.0f) / sqrtf(static_cast<float>(H->dh));
  if (layer >= 0) a.cur = H->L32[layer];
  if (layer + 1 < H->M) a.nxt = H->L32[layer + 1];
  a.q_ln_g = H->q_ln_g;
  a.q_ln_b = H->q_ln_b;
  step_widths(H, &a.wa, &a.wb);
  const size_t smem = target_step_smem(H);
  const unsigned grid = static_cast<unsigned>((T + kTB - 1) / kTB);
  if (H->elem == 2) {
    cudaFuncSetAttribute(target_step_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    target_step_kernel<true><<<grid, kThreads, smem, s>>>(a);
  } else {
    cudaFuncSetAttribute(target_step_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    target_step_kernel<false><<<grid, kThreads, smem, s>>>(a);
  }
}

// Same launch as launch_target_step for the tensor-core partial layout, with
// the bf16 query rows and the split partials in caller-given buffers.
void launch_target_step_ws(const stca_handle* H, int layer, const void* targets, int64_t T,
                           const StepPlan& plan, float* Z, uint16_t* Ubf, float* part,
                           int64_t G, cudaStream_t s) {
  if (T <= 0) return;
  StepArgs a{};
  a.layer = layer;
  a.M = H->M; a.d = H->d; a.h = H->h; a.dh = H->dh; a.rd = H->rd;
  a.T = T;
  a.targets = targets;
  a.plan = plan;
  a.pacc = part;
  a.pm = part + G * H->d;
  a.pl = a.pm + G;
  a.Z = Z;
  a.U = nullptr;
  a.Ubf = Ubf;
  a.uscale = 1.4426950408889634f / sqrtf(static_cast<float>(H->dh));
  if (layer >= 0) a.cur = H->L32[layer];
  if (layer + 1 < H->M) a.nxt = H->L32[layer + 1];
  a.q_ln_g = H->q_ln_g;
  a.q_ln_b = H->q_ln_b;
  step_widths(H, &a.wa, &a.wb);
  const size_t smem = target_step_smem(H);
  const unsigned grid = static_cast<unsigned>((T + kTB - 1) / kTB);
  cudaFuncSetAttribute(target_step_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  target_step_kernel<true><<<grid, kThreads, smem, s>>>(a);
}

}  // namespace stca
