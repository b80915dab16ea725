// Per-target step of the STCA forward, between two attention layers:
//   split combine   c_j = sum_w 2^{m_w - m} acc_w / sum_w 2^{m_w - m} l_w       (Eq. (13) alpha X~)
//   output          o = [c_1 W_V^1 || ... || c_h W_V^h] W_O; Z[t, i, :] = o   (Eqs. (6), (8))
//   query fusion    q = SwiGLUFFN_{i+1}([o(1) || ... || o(i+1) || x_t] W_C)  (Eq. (7))
//   u projection    u_j = (q W_Q^j) W_K^j^T, scaled for the next attention     (Eq. (13))
// and, before the first layer, q(1) = LN(SwiGLUFFN_1(x_t)) (Eq. (3)) and its u;
// after the last layer, optionally, the prediction-head token
//   z = SwiGLUFFN_z([o(1) || ... || o(M) || x_t] W_Z)                         (Eq. (9)).
// Sources: "Make It Long, Keep It Fast" digest §2.1.
//
// A CTA takes kTB targets and runs the whole chain for them with fp32
// activations in shared memory.  Every matrix product streams its weight
// matrix (bf16 for bf16 handles, fp32 otherwise) through a 4-stage ring of
// bulk TMA copies, and gives each thread a pair of output columns for all kTB
// rows; narrow outputs split the K range over thread groups and reduce in
// shared memory.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <vector>

#include "stca_internal.h"
#include "tc_common.cuh"

namespace stca {
namespace {

constexpr int kThreads = 512;
constexpr int kNB = 512;               // output columns per GEMM block (256 pairs)
constexpr int kChunk = 16384;          // weight bytes per pipeline stage
constexpr int kStages = 4;             // weight chunks in flight

using stca::tc::smem_u32;

// Weight ring: kStages shared-memory stages filled by bulk TMA copies (one per
// row segment, or one per stage when the rows are contiguous), each stage
// completing on its own mbarrier.  Chunk q of the kernel's whole sequence of
// products lands in stage q % kStages; its phase parity is (q / kStages) & 1.
struct Ring {
  unsigned char* buf;     // kStages x stage bytes
  uint64_t* bar;          // kStages mbarriers
  int* status;            // device status word (bounded waits)
  uint32_t q;             // chunks consumed so far in this kernel
};

__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Issue chunk q: `rows` rows of `row_bytes` from src (row pitch src_pitch) to
// stage q % kStages (row pitch dst_pitch).  Called by every thread; thread 0 issues.
__device__ __forceinline__ void ring_issue(Ring& R, uint32_t q, int stage_bytes, const unsigned char* src,
                                           int rows, int row_bytes, int64_t src_pitch, int dst_pitch) {
  if (threadIdx.x != 0) return;
  const int st = q % kStages;
  unsigned char* dst = R.buf + st * stage_bytes;
  uint64_t* bar = &R.bar[st];
  stca::tc::mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows * row_bytes));
  if (src_pitch == row_bytes && dst_pitch == row_bytes) {
    bulk_copy(dst, src, static_cast<uint32_t>(rows * row_bytes), bar);
  } else {
    for (int r = 0; r < rows; ++r)
      bulk_copy(dst + r * dst_pitch, src + r * src_pitch, static_cast<uint32_t>(row_bytes), bar);
  }
}

// Wait until chunk q has landed (bounded; a timeout is reported and skipped).
__device__ __forceinline__ void ring_wait(Ring& R, uint32_t q) {
  uint64_t* bar = &R.bar[q % kStages];
  const uint32_t parity = (q / kStages) & 1;
  if (stca::tc::mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = stca::tc::globaltimer();
  while (!stca::tc::mbar_try_wait(bar, parity)) {
    if (stca::tc::globaltimer() - t0 > stca::tc::kWaitTimeoutNs) {
      atomicOr(R.status, kStatusStepTimeout);
      return;
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float silu_acc(float z) { return z / (1.0f + expf(-z)); }

template <typename WT>
__device__ __forceinline__ float2 load_pair(const unsigned char* p);
template <>
__device__ __forceinline__ float2 load_pair<uint16_t>(const unsigned char* p) {
  const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}
template <>
__device__ __forceinline__ float2 load_pair<float>(const unsigned char* p) {
  return *reinterpret_cast<const float2*>(p);
}

template <bool BF>
__device__ __forceinline__ float ld_elem(const void* p, int64_t i) {
  if constexpr (BF) return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16);
  else return static_cast<const float*>(p)[i];
}

// out[b][n] = sum_{k < K} in[b * ldin + (n / hc) * hs + k] * W[k * N + n], b < kTB, n < N.
// `hc` columns share one input slice (a head), placed `hs` floats apart; a plain
// product has hc = N, hs = 0.  W is row-major K x N in global memory.  Every
// thread of the CTA must call this; it ends with the CTA synchronised.
template <typename WT, int kTB, int NT>
__device__ void gemm_tb(const float* in, int ldin, int hc, int hs, int K, const WT* W, int N,
                        float* out, int ldout, Ring& R, float* red) {
  unsigned char* wbuf = R.buf;
  const int tid = threadIdx.x;
  const bool vec4 = (ldin % 4 == 0) && (hs % 4 == 0) && (reinterpret_cast<uintptr_t>(in) % 16 == 0);
  for (int n0 = 0; n0 < N; n0 += kNB) {
    const int nb = min(kNB, N - n0);
    const int np = nb >> 1;
    const int gk = max(1, NT / np);                        // K groups
    const int p = tid % np, g = tid / np;
    const bool active = g < gk;
    const int row_bytes = nb * static_cast<int>(sizeof(WT));
    const int rows = max(1, kChunk / row_bytes);
    const int nchunks = (K + rows - 1) / rows;
    auto issue = [&](int c) {
      if (c >= nchunks) return;
      const int k0 = c * rows, kr = min(rows, K - k0);
      ring_issue(R, R.q + c, kChunk,
                 reinterpret_cast<const unsigned char*>(W + static_cast<int64_t>(k0) * N + n0), kr,
                 row_bytes, static_cast<int64_t>(N) * sizeof(WT), row_bytes);
    };
    float acc[kTB][2];
#pragma unroll
    for (int b = 0; b < kTB; ++b) acc[b][0] = acc[b][1] = 0.f;
    const int col = n0 + 2 * p;
    const float* inb = in + (col / hc) * hs;
    for (int c = 0; c < kStages - 1; ++c) issue(c);
    for (int c = 0; c < nchunks; ++c) {
      issue(c + kStages - 1);
      ring_wait(R, R.q + c);
      const unsigned char* wb = wbuf + ((R.q + c) % kStages) * kChunk + p * 2 * sizeof(WT);
      const int k0 = c * rows, kr = min(rows, K - k0);
      if (active) {
        // group g takes a contiguous slice of the chunk's rows, in steps of 4
        const int per = ((kr + gk - 1) / gk + 3) & ~3;
        const int kb = g * per, ke = min(kr, kb + per);
        int kk = kb;
        if (vec4 && ((k0 + kb) & 3) == 0) {
          for (; kk + 4 <= ke; kk += 4) {
            float2 w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) w[u] = load_pair<WT>(wb + (kk + u) * row_bytes);
#pragma unroll
            for (int b = 0; b < kTB; ++b) {
              const float4 x = *reinterpret_cast<const float4*>(inb + b * ldin + k0 + kk);
              acc[b][0] = fmaf(x.x, w[0].x, acc[b][0]);
              acc[b][1] = fmaf(x.x, w[0].y, acc[b][1]);
              acc[b][0] = fmaf(x.y, w[1].x, acc[b][0]);
              acc[b][1] = fmaf(x.y, w[1].y, acc[b][1]);
              acc[b][0] = fmaf(x.z, w[2].x, acc[b][0]);
              acc[b][1] = fmaf(x.z, w[2].y, acc[b][1]);
              acc[b][0] = fmaf(x.w, w[3].x, acc[b][0]);
              acc[b][1] = fmaf(x.w, w[3].y, acc[b][1]);
            }
          }
        }
        for (; kk < ke; ++kk) {
          const float2 w = load_pair<WT>(wb + kk * row_bytes);
#pragma unroll
          for (int b = 0; b < kTB; ++b) {
            const float x = inb[b * ldin + k0 + kk];
            acc[b][0] = fmaf(x, w.x, acc[b][0]);
            acc[b][1] = fmaf(x, w.y, acc[b][1]);
          }
        }
      }
      __syncthreads();
    }
    R.q += nchunks;
    if (gk > 1) {
      if (active) {
#pragma unroll
        for (int b = 0; b < kTB; ++b) {
          red[(g * kTB + b) * nb + 2 * p] = acc[b][0];
          red[(g * kTB + b) * nb + 2 * p + 1] = acc[b][1];
        }
      }
      __syncthreads();
      for (int e = tid; e < kTB * nb; e += NT) {
        const int b = e / nb, n = e - b * nb;
        float s = 0.f;
        for (int q = 0; q < gk; ++q) s += red[(q * kTB + b) * nb + n];
        out[b * ldout + n0 + n] = s;
      }
    } else if (active) {
#pragma unroll
      for (int b = 0; b < kTB; ++b) {
        out[b * ldout + col] = acc[b][0];
        out[b * ldout + col + 1] = acc[b][1];
      }
    }
    __syncthreads();
  }
}

template <typename WT, int kTB>
__device__ __forceinline__ void gemm(const float* in, int ldin, int hc, int hs, int K, const void* W,
                                     int N, float* out, int ldout, Ring& R, float* red) {
  gemm_tb<WT, kTB, kThreads>(in, ldin, hc, hs, K, static_cast<const WT*>(W), N, out, ldout, R, red);
}

// ---------------------------------------------------------------- split combine
// c_j = sum_w s_w acc_w / sum_w s_w l_w with s_w = e^(m_w - m) (2^ for the
// tensor-core partials) over the items w that cover query row (t, j): the
// attention-weighted history alpha_j X~ of Eq. (13).  One warp per query row,
// eight rows per CTA: the lanes first read the items' (m, l), one item per
// lane, and turn them into weights; then each lane owns 4 columns (a float4)
// of every 128 and sums the items' partial rows, one coalesced 16-byte load
// per lane and item.
constexpr int kCombineThreads = 256;
constexpr int kCombineRows = kCombineThreads / 32;

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(StepPlan P, const float* __restrict__ pacc, const float* __restrict__ pm,
               const float* __restrict__ pl, float* __restrict__ out, int d, int h, int64_t nq) {
  const int lane = threadIdx.x & 31;
  const int64_t qr = static_cast<int64_t>(blockIdx.x) * kCombineRows + (threadIdx.x >> 5);
  tc::pdl_wait();
  if (qr >= nq) return;                   // target t, head j: row t * h + j of U
  const int64_t t = qr / h;
  const int j = static_cast<int>(qr - t * h);
  const int r = P.treq[t];
  const int64_t qrow = (t - P.toff[r]) * h + j;
  const int64_t mt = qrow / P.mtile_rows;
  const int64_t row = qrow - mt * P.mtile_rows;
  const int pair = P.req_pair_begin[r] + static_cast<int>(mt);
  const int w0 = P.pair_item_begin[pair], nw = P.pair_item_begin[pair + 1] - w0;
  // the row's maximum and normaliser over all items, 32 items at a time
  float mx = -INFINITY;
  for (int b = 0; b < nw; b += 32)
    if (b + lane < nw) mx = fmaxf(mx, pm[P.items[w0 + b + lane].row_base + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float ls = 0.f;
  for (int b = 0; b < nw; b += 32)
    if (b + lane < nw) {
      const int64_t g = P.items[w0 + b + lane].row_base + row;
      const float m = pm[g];
      ls = fmaf(pl[g], P.log2_partials ? exp2f(m - mx) : expf(m - mx), ls);
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  const float inv = 1.0f / ls;
  float* orow = out + qr * d;
  for (int b = 0; b < nw; b += 32) {
    // item b + lane: its partial row and weight, handed round the warp below
    int64_t g = 0;
    float f = 0.f;
    if (b + lane < nw) {
      g = P.items[w0 + b + lane].row_base + row;
      const float m = pm[g];
      f = (P.log2_partials ? exp2f(m - mx) : expf(m - mx)) * inv;
    }
    const int n = min(32, nw - b);
    for (int k0 = 0; k0 < d; k0 += 128) {      // the whole warp walks the same k0 (shuffles)
      const int k = k0 + 4 * lane;
      const bool on = k < d;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (on && b > 0) acc = *reinterpret_cast<const float4*>(orow + k);
      for (int w = 0; w < n; ++w) {
        const int64_t gw = __shfl_sync(0xffffffffu, g, w);
        const float fw = __shfl_sync(0xffffffffu, f, w);
        if (on) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(pacc + gw * d + k));
          acc.x = fmaf(fw, v.x, acc.x);
          acc.y = fmaf(fw, v.y, acc.y);
          acc.z = fmaf(fw, v.z, acc.z);
          acc.w = fmaf(fw, v.w, acc.w);
        }
      }
      if (on) *reinterpret_cast<float4*>(orow + k) = acc;
    }
  }
  tc::pdl_trigger();
}

// Naive-form merge (Eq. (12) with projected K, V): o_j[t] = sum_w s_w acc_w / sum_w
// s_w l_w over the items of head j's row of target t, where acc_w holds the
// tile's 64 head-group features of alpha V and head j owns d_h of them.  One
// warp per (target, head) query row, eight per CTA; writes o_head[t][j d_h + c].
__global__ void __launch_bounds__(kCombineThreads)
combine_naive_kernel(StepPlan P, const float* __restrict__ pacc, const float* __restrict__ pm,
                     const float* __restrict__ pl, float* __restrict__ out, int d, int h, int dh,
                     int G, int Tq, int64_t nq) {
  const int lane = threadIdx.x & 31;
  const int64_t qr = static_cast<int64_t>(blockIdx.x) * kCombineRows + (threadIdx.x >> 5);
  if (qr >= nq) return;
  const int64_t t = qr / h;
  const int j = static_cast<int>(qr - t * h);
  const int r = P.treq[t];
  const int64_t tl = t - P.toff[r], Tr = P.toff[r + 1] - P.toff[r];
  const int64_t nslots = (Tr + Tq - 1) / Tq, qs = tl / Tq, tt = tl - qs * Tq;
  const int jg = j / G, sl = j - jg * G;
  const int64_t row = static_cast<int64_t>(sl) * Tq + tt;
  const int pair = P.req_pair_begin[r] + static_cast<int>(jg * nslots + qs);
  const int w0 = P.pair_item_begin[pair], nw = P.pair_item_begin[pair + 1] - w0;
  float mx = -INFINITY;
  for (int b = 0; b < nw; b += 32)
    if (b + lane < nw) mx = fmaxf(mx, pm[P.items[w0 + b + lane].row_base + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float ls = 0.f;
  for (int b = 0; b < nw; b += 32)
    if (b + lane < nw) {
      const int64_t g = P.items[w0 + b + lane].row_base + row;
      ls = fmaf(pl[g], exp2f(pm[g] - mx), ls);
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  const float inv = 1.0f / ls;
  float* orow = out + t * d + static_cast<int64_t>(j) * dh;
  for (int b = 0; b < nw; b += 32) {
    int64_t g = 0;
    float f = 0.f;
    if (b + lane < nw) {
      g = P.items[w0 + b + lane].row_base + row;
      f = exp2f(pm[g] - mx) * inv;
    }
    const int n = min(32, nw - b);
    for (int c0 = 0; c0 < dh; c0 += 32) {      // warp-uniform: the shuffles below
      const int c = c0 + lane;
      const bool on = c < dh;
      float acc = (on && b > 0) ? orow[c] : 0.f;
      for (int w = 0; w < n; ++w) {
        const int64_t gw = __shfl_sync(0xffffffffu, g, w);
        const float fw = __shfl_sync(0xffffffffu, f, w);
        if (on) acc = fmaf(fw, __ldg(pacc + gw * 64 + sl * dh + c), acc);
      }
      if (on) orow[c] = acc;
    }
  }
}

struct StepArgs {
  int layer, M, d, h, dh, rd;
  int64_t T;
  const void* targets;
  const float* cmerged;   // T x h x d: c_j = alpha_j X~ of the layer just attended
  float* Z;
  int* status;        // device status word
  float* U;           // fp32 query rows (CUDA-core attention) or NULL
  uint16_t* Ubf;      // bf16 query rows (tensor-core attention) or NULL
  float uscale;       // 1/sqrt(d_h), times log2(e) for the exp2 kernels
  LayerStep cur, nxt; // weights of `layer` (output) and `layer + 1` (query)
  const float *q_ln_g, *q_ln_b;
  int wa, wb;         // widths of buffers A and B per target
};

template <bool XBF, typename WT, int kTB>
__global__ void __launch_bounds__(kThreads) target_step_kernel(StepArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int d = a.d, h = a.h, dh = a.dh, rd = a.rd;
  const int ldd = d + 8;     // padded row strides spread rows over the shared-memory banks
  constexpr int kRing = kStages * kChunk;
  constexpr int kRed = kTB * 2 * kThreads;
  unsigned char* wbuf = smem;                                 // weight ring
  uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + kRing); // kStages ring mbarriers
  float* red = reinterpret_cast<float*>(smem + kRing + 128);  // K-split partials
  float* xs = red + kRed;                                     // kTB x ldd: raw x_t
  float* A = xs + kTB * ldd;                                  // kTB x wa
  float* B = A + kTB * a.wa;                                  // kTB x wb
  float* C = B + kTB * a.wb;                                  // kTB x ldd
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) stca::tc::mbar_init(&rbar[i], 1);
    stca::tc::fence_mbar_init();
  }
  Ring R{wbuf, rbar, a.status, 0};
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTB;
  const int nb = a.T - t0 < kTB ? static_cast<int>(a.T - t0) : kTB;
  for (int e = tid; e < kTB * d; e += blockDim.x) {
    const int b = e / d, k = e - b * d;
    xs[b * ldd + k] = b < nb ? ld_elem<XBF>(a.targets, (t0 + b) * d + k) : 0.f;
  }
  __syncthreads();
  const int layer = a.layer;
  if (layer >= 0) {
    // c_j rows of these targets (merged by combine_kernel) into A[b][j * d + k]
    const int hd = h * d;
    for (int e = tid * 4; e < kTB * hd; e += blockDim.x * 4) {
      const int b = e / hd, c = e - b * hd;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (b < nb) v = *reinterpret_cast<const float4*>(a.cmerged + (t0 + b) * hd + c);
      *reinterpret_cast<float4*>(A + b * a.wa + c) = v;
    }
    __syncthreads();
    // o_head[b][j dh + c] = c_j . W_V[:, j dh + c]; o = o_head W_O
    gemm<WT, kTB>(A, a.wa, dh, d, d, a.cur.Wv, d, B, a.wb, R, red);
    gemm<WT, kTB>(B, a.wb, d, 0, d, a.cur.Wo, d, C, ldd, R, red);
    for (int e = tid; e < nb * d; e += blockDim.x) {
      const int b = e / d, k = e - b * d;
      a.Z[((t0 + b) * a.M + layer) * d + k] = C[b * ldd + k];
    }
    if (layer + 1 >= a.M) return;
    // Eq. (7): [o(1) || ... || o(layer+1) || x_t] W_C^(layer+2), then SwiGLU
    const int wcat = (layer + 2) * d;
    __syncthreads();
    for (int e = tid; e < kTB * wcat; e += blockDim.x) {
      const int b = e / wcat, k = e - b * wcat;
      const int blk = k / d, kk = k - blk * d;
      float v = 0.f;
      if (b < nb) {
        if (blk < layer) v = a.Z[((t0 + b) * a.M + blk) * d + kk];
        else if (blk == layer) v = C[b * ldd + kk];
        else v = xs[b * ldd + kk];
      }
      A[b * a.wa + k] = v;
    }
    __syncthreads();
    gemm<WT, kTB>(A, a.wa, wcat, 0, wcat, a.nxt.Wc, d, B, a.wb, R, red);
    gemm<WT, kTB>(B, a.wb, 2 * rd, 0, d, a.nxt.Wug, 2 * rd, A, a.wa, R, red);
  } else {
    gemm<WT, kTB>(xs, ldd, 2 * rd, 0, d, a.nxt.Wug, 2 * rd, A, a.wa, R, red);
  }
  // gate: B[b][c] = u * SiLU(g); then the down projection into C
  for (int e = tid; e < kTB * rd; e += blockDim.x) {
    const int b = e / rd, c = e - b * rd;
    B[b * a.wb + c] = A[b * a.wa + c] * silu_acc(A[b * a.wa + rd + c]);
  }
  __syncthreads();
  gemm<WT, kTB>(B, a.wb, d, 0, rd, a.nxt.Wd, d, C, ldd, R, red);
  if (layer < 0) {
    // LayerNorm of Eq. (3)
    for (int b = warp; b < kTB; b += blockDim.x / 32) {
      float s = 0.f;
      for (int k = lane; k < d; k += 32) s += C[b * ldd + k];
      const float mean = warp_sum(s) / d;
      float v = 0.f;
      for (int k = lane; k < d; k += 32) { const float u = C[b * ldd + k] - mean; v = fmaf(u, u, v); }
      const float rstd = 1.0f / sqrtf(warp_sum(v) / d + 1e-5f);
      __syncwarp();
      for (int k = lane; k < d; k += 32)
        C[b * ldd + k] = (C[b * ldd + k] - mean) * rstd * a.q_ln_g[k] + a.q_ln_b[k];
    }
    __syncthreads();
  }
  // P = q W_Q (into B); u_j = P_j W_K^j^T (into A, [b][j][k]); store scaled
  gemm<WT, kTB>(C, ldd, d, 0, d, a.nxt.Wq, d, B, a.wb, R, red);
  gemm<WT, kTB>(B, a.wb, d, dh, dh, a.nxt.WkT, h * d, A, a.wa, R, red);
  for (int e = tid; e < nb * h * d; e += blockDim.x) {
    const int b = e / (h * d), cc = e - b * (h * d);
    const float u = A[b * a.wa + cc] * a.uscale;
    const int64_t gi = (t0 + b) * h * d + cc;
    if (a.U) a.U[gi] = u;
    if (a.Ubf) a.Ubf[gi] = __bfloat16_as_ushort(__float2bfloat16_rn(u));
  }
}

// ---------------------------------------------------------------- prediction head
// z = ((v W_Z) zW_u * SiLU((v W_Z) zW_g)) zW_d with v = [o(1) || ... || o(M) || x_t]
// (Eq. (9)).  Row t of Z already holds o(1..M) back to back, so v is that row
// followed by x_t.  Organised like the step: kTB targets per CTA, fp32
// activations in shared memory, each weight matrix streamed once per CTA.
struct HeadArgs {
  int M, d, rd;
  int64_t T;
  const void* targets;
  const float* Z;
  float* zout;
  int* status;
  const void *Wz, *Wug, *Wd;
  int wa, wb;         // widths of buffers A and B per target
};

template <bool XBF, typename WT, int kTB>
__global__ void __launch_bounds__(kThreads) head_kernel(HeadArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int kRing = kStages * kChunk;
  constexpr int kRed = kTB * 2 * kThreads;
  unsigned char* wbuf = smem;                                 // weight ring
  uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + kRing); // kStages ring mbarriers
  float* red = reinterpret_cast<float*>(smem + kRing + 128);  // K-split partials
  float* A = red + kRed;        // kTB x wa: v, then [u | g], then z
  float* B = A + kTB * a.wa;    // kTB x wb: v W_Z, then u * SiLU(g)
  const int tid = threadIdx.x;
  const int d = a.d, rd = a.rd, md = a.M * d, vd = md + d;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) stca::tc::mbar_init(&rbar[i], 1);
    stca::tc::fence_mbar_init();
  }
  Ring R{wbuf, rbar, a.status, 0};
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTB;
  const int nb = a.T - t0 < kTB ? static_cast<int>(a.T - t0) : kTB;
  for (int e = tid; e < kTB * vd; e += blockDim.x) {
    const int b = e / vd, k = e - b * vd;
    float v = 0.f;
    if (b < nb) v = k < md ? a.Z[(t0 + b) * md + k] : ld_elem<XBF>(a.targets, (t0 + b) * d + k - md);
    A[b * a.wa + k] = v;
  }
  __syncthreads();
  gemm<WT, kTB>(A, a.wa, d, 0, vd, a.Wz, d, B, a.wb, R, red);
  gemm<WT, kTB>(B, a.wb, 2 * rd, 0, d, a.Wug, 2 * rd, A, a.wa, R, red);
  for (int e = tid; e < kTB * rd; e += blockDim.x) {
    const int b = e / rd, c = e - b * rd;
    B[b * a.wb + c] = A[b * a.wa + c] * silu_acc(A[b * a.wa + rd + c]);
  }
  __syncthreads();
  gemm<WT, kTB>(B, a.wb, d, 0, rd, a.Wd, d, A, a.wa, R, red);
  for (int e = tid; e < nb * d; e += blockDim.x) {
    const int b = e / d, k = e - b * d;
    a.zout[(t0 + b) * d + k] = A[b * a.wa + k];
  }
}

void head_widths(const stca_handle* H, int* wa, int* wb) {
  *wa = std::max((H->M + 1) * H->d, 2 * H->rd) + 8;
  *wb = std::max(H->d, H->rd) + 8;
}

size_t head_smem(const stca_handle* H, int tb) {
  int wa, wb;
  head_widths(H, &wa, &wb);
  return static_cast<size_t>(kStages) * kChunk + 128 +
         static_cast<size_t>(tb) * 2 * kThreads * sizeof(float) +
         static_cast<size_t>(tb) * (wa + wb) * sizeof(float);
}

template <int TB>
void launch_head_tb(const stca_handle* H, const HeadArgs& a, cudaStream_t s) {
  const size_t smem = head_smem(H, TB);
  const unsigned grid = static_cast<unsigned>((a.T + TB - 1) / TB);
  if (H->elem == 2) {
    auto k = head_kernel<true, uint16_t, TB>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, s>>>(a);
  } else {
    auto k = head_kernel<false, float, TB>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, s>>>(a);
  }
}

// Convert fp32 host values (bf16-exact for bf16 handles) to the handle's
// element type and copy them to a new device allocation.
int upload_elems(const stca_handle* H, const std::vector<float>& host, void** dst, const char* what) {
  const size_t n = host.size();
  const size_t esz = H->elem == 2 ? 2 : 4;
  std::vector<unsigned char> bytes(n * esz);
  if (esz == 2) {
    uint16_t* out = reinterpret_cast<uint16_t*>(bytes.data());
    for (size_t k = 0; k < n; ++k) {
      uint32_t u;
      memcpy(&u, &host[k], 4);
      out[k] = static_cast<uint16_t>(u >> 16);
    }
  } else {
    memcpy(bytes.data(), host.data(), n * 4);
  }
  if (cudaMalloc(dst, bytes.size()) != cudaSuccess) {
    cudaGetLastError();
    *dst = nullptr;
    return set_error(STCA_ENOMEM, std::string(what) + " weight allocation failed");
  }
  STCA_CUDA_TRY(cudaMemcpy(*dst, bytes.data(), bytes.size(), cudaMemcpyHostToDevice));
  return STCA_OK;
}

void step_widths(const stca_handle* H, int* wa, int* wb) {
  const int d = H->d;
  *wa = std::max(std::max(H->h * d, H->M * d), 2 * H->rd) + 8;
  *wb = std::max(d, H->rd) + 8;
}

size_t smem_for(const stca_handle* H, int tb) {
  int wa, wb;
  step_widths(H, &wa, &wb);
  return static_cast<size_t>(kStages) * kChunk + 128 +
         static_cast<size_t>(tb) * 2 * kThreads * sizeof(float) +
         static_cast<size_t>(tb) * (2 * (H->d + 8) + wa + wb) * sizeof(float);
}

// Targets per CTA: 8, or 4 when 8 do not fit in shared memory.
int choose_tb(const stca_handle* H) { return smem_for(H, 8) <= 227 * 1024 ? 8 : 4; }

template <int TB>
void launch_tb(const stca_handle* H, const StepArgs& a, cudaStream_t s) {
  const size_t smem = smem_for(H, TB);
  const unsigned grid = static_cast<unsigned>((a.T + TB - 1) / TB);
  if (H->elem == 2) {
    auto k = target_step_kernel<true, uint16_t, TB>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, s>>>(a);
  } else {
    auto k = target_step_kernel<false, float, TB>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, s>>>(a);
  }
}

void launch(const stca_handle* H, const StepArgs& a0, cudaStream_t s) {
  StepArgs a = a0;
  step_widths(H, &a.wa, &a.wb);
  if (choose_tb(H) == 8) launch_tb<8>(H, a, s);
  else launch_tb<4>(H, a, s);
}

StepArgs base_args(const stca_handle* H, int layer, const void* targets, int64_t T,
                   const float* cmerged, float* Z) {
  StepArgs a{};
  a.layer = layer;
  a.M = H->M; a.d = H->d; a.h = H->h; a.dh = H->dh; a.rd = H->rd;
  a.T = T;
  a.targets = targets;
  a.cmerged = cmerged;
  a.Z = Z;
  a.status = H->status_d;
  if (layer >= 0) a.cur = H->Lstep[layer];
  if (layer + 1 < H->M) a.nxt = H->Lstep[layer + 1];
  a.q_ln_g = H->q_ln_g;
  a.q_ln_b = H->q_ln_b;
  return a;
}

}  // namespace

size_t target_step_smem(const stca_handle* H) { return smem_for(H, 4); }

void launch_combine(const stca_handle* H, const StepPlan& plan, const float* part, int64_t G,
                    int64_t T, float* out, cudaStream_t s) {
  if (T <= 0) return;
  const float* pacc = part;
  const float* pm = part + G * H->d;
  const float* pl = pm + G;
  const int64_t nq = T * H->h;
  tc::launch_pdl(combine_kernel, dim3(static_cast<unsigned>((nq + kCombineRows - 1) / kCombineRows)),
                 dim3(kCombineThreads), 0, s, plan, pacc, pm, pl, out, H->d, H->h, nq);
}

void launch_combine_proj(const stca_handle* H, const StepPlan& plan, const float* part, int64_t G,
                         int64_t T, float* out, cudaStream_t s) {
  if (T <= 0) return;
  // rows d_h wide: row t h + j of the merged output is o_head[t][j d_h ..]
  const float* pacc = part;
  const float* pm = part + G * H->d;
  const float* pl = pm + G;
  const int64_t nq = T * H->h;
  tc::launch_pdl(combine_kernel, dim3(static_cast<unsigned>((nq + kCombineRows - 1) / kCombineRows)),
                 dim3(kCombineThreads), 0, s, plan, pacc, pm, pl, out, H->dh, H->h, nq);
}

void launch_combine_naive(const stca_handle* H, const StepPlan& plan, const float* part, int64_t G,
                          int64_t T, float* out, cudaStream_t s) {
  if (T <= 0) return;
  const NaiveLayout NL = naive_layout(H->dh);
  const float* pacc = part;
  const float* pm = part + G * 64;
  const float* pl = pm + G;
  const int64_t nq = T * H->h;
  combine_naive_kernel<<<static_cast<unsigned>((nq + kCombineRows - 1) / kCombineRows),
                         kCombineThreads, 0, s>>>(plan, pacc, pm, pl, out, H->d, H->h, H->dh, NL.G,
                                                  NL.Tq, nq);
}

void launch_target_step(const stca_handle* H, int layer, const void* targets, int64_t T,
                        const StepPlan& plan, const float* cmerged, float* Z, cudaStream_t s) {
  if (T <= 0) return;
  StepArgs a = base_args(H, layer, targets, T, cmerged, Z);
  const bool tc = plan.log2_partials != 0;
  a.U = tc ? nullptr : H->U;
  a.Ubf = tc ? H->Ubf : nullptr;
  a.uscale = (tc ? 1.4426950408889634f : 1.0f) / sqrtf(static_cast<float>(H->dh));
  launch(H, a, s);
}

void launch_target_step_ws(const stca_handle* H, int layer, const void* targets, int64_t T,
                           const float* cmerged, float* Z, uint16_t* Ubf, cudaStream_t s) {
  if (T <= 0) return;
  StepArgs a = base_args(H, layer, targets, T, cmerged, Z);
  a.U = nullptr;
  a.Ubf = Ubf;
  a.uscale = 1.4426950408889634f / sqrtf(static_cast<float>(H->dh));
  launch(H, a, s);
}

// Lay out the per-target weights of every layer in the handle's element type:
// W_Q, W_K^T per head as one [d_h x h d] matrix, W_V, W_O, W_C, the query
// SwiGLU up/gate as one [d x 2rd] matrix [W_u | W_g], and W_d.
int step_weights_setup(stca_handle* H, const std::vector<StepHostW>& layers) {
  const int d = H->d, h = H->h, dh = H->dh, rd = H->rd, M = H->M;
  auto pad = [](size_t n) { return (n + 15) & ~size_t(15); };
  std::vector<float> host;
  struct Off { size_t Wq, WkT, Wv, Wo, Wc, Wug, Wd; };
  std::vector<Off> offs(M);
  for (int i = 0; i < M; ++i) {
    const StepHostW& L = layers[i];
    Off& o = offs[i];
    auto put = [&](const float* src, size_t n) {
      const size_t at = host.size();
      host.resize(at + pad(n), 0.f);
      if (src) std::copy(src, src + n, host.begin() + at);
      return at;
    };
    o.Wq = put(L.Wq, static_cast<size_t>(d) * d);
    o.WkT = put(nullptr, static_cast<size_t>(dh) * h * d);
    for (int c = 0; c < dh; ++c)          // WkT[c][j d + k] = W_K[k][j dh + c]
      for (int j = 0; j < h; ++j)
        for (int k = 0; k < d; ++k)
          host[o.WkT + static_cast<size_t>(c) * h * d + j * d + k] = L.Wk[static_cast<size_t>(k) * d + j * dh + c];
    o.Wv = put(L.Wv, static_cast<size_t>(d) * d);
    o.Wo = put(L.Wo, static_cast<size_t>(d) * d);
    o.Wc = i > 0 ? put(L.Wc, static_cast<size_t>(i + 1) * d * d) : 0;
    o.Wug = put(nullptr, static_cast<size_t>(d) * 2 * rd);
    for (int k = 0; k < d; ++k)
      for (int c = 0; c < rd; ++c) {
        host[o.Wug + static_cast<size_t>(k) * 2 * rd + c] = L.qWu[static_cast<size_t>(k) * rd + c];
        host[o.Wug + static_cast<size_t>(k) * 2 * rd + rd + c] = L.qWg[static_cast<size_t>(k) * rd + c];
      }
    o.Wd = put(L.qWd, static_cast<size_t>(rd) * d);
  }
  const size_t esz = H->elem == 2 ? 2 : 4;
  if (int rc = upload_elems(H, host, &H->wstep, "per-target")) return rc;
  H->Lstep.resize(M);
  const unsigned char* base = static_cast<const unsigned char*>(H->wstep);
  for (int i = 0; i < M; ++i) {
    const Off& o = offs[i];
    LayerStep& L = H->Lstep[i];
    L.Wq = base + o.Wq * esz;
    L.WkT = base + o.WkT * esz;
    L.Wv = base + o.Wv * esz;
    L.Wo = base + o.Wo * esz;
    L.Wc = i > 0 ? base + o.Wc * esz : nullptr;
    L.Wug = base + o.Wug * esz;
    L.Wd = base + o.Wd * esz;
  }
  return STCA_OK;
}

// Head weights in the handle's element type: W_Z, [zW_u | zW_g] as one
// [d x 2rd] matrix, zW_d; each starts on a 64-byte boundary.
int head_weights_setup(stca_handle* H, const float* Wz, const float* zWu, const float* zWg,
                       const float* zWd) {
  const int d = H->d, rd = H->rd;
  if (head_smem(H, 4) > 227 * 1024)
    return set_error(STCA_EINVAL, "prediction head needs more than 227 KB shared memory for these sizes");
  auto pad = [](size_t n) { return (n + 15) & ~size_t(15); };
  const size_t nz = static_cast<size_t>(H->M + 1) * d * d, nug = static_cast<size_t>(d) * 2 * rd,
               nd = static_cast<size_t>(rd) * d;
  const size_t oz = 0, oug = pad(nz), od = oug + pad(nug);
  std::vector<float> host(od + pad(nd), 0.f);
  std::copy(Wz, Wz + nz, host.begin() + oz);
  for (int k = 0; k < d; ++k)
    for (int c = 0; c < rd; ++c) {
      host[oug + static_cast<size_t>(k) * 2 * rd + c] = zWu[static_cast<size_t>(k) * rd + c];
      host[oug + static_cast<size_t>(k) * 2 * rd + rd + c] = zWg[static_cast<size_t>(k) * rd + c];
    }
  std::copy(zWd, zWd + nd, host.begin() + od);
  if (int rc = upload_elems(H, host, &H->whead, "prediction-head")) return rc;
  const size_t esz = H->elem == 2 ? 2 : 4;
  const unsigned char* base = static_cast<const unsigned char*>(H->whead);
  H->hWz = base + oz * esz;
  H->hWug = base + oug * esz;
  H->hWd = base + od * esz;
  return STCA_OK;
}

// Targets per CTA: 8, else 4.  Four always fit when the step's four-target
// layout does (stca_init checks that): the head's widths are (M+1)d and
// max(d, rd) against the step's 2d + max(hd, Md, 2rd) + max(d, rd).
void launch_head(const stca_handle* H, const void* targets, int64_t T, const float* Z, float* zout,
                 cudaStream_t s) {
  if (T <= 0) return;
  HeadArgs a{};
  a.M = H->M; a.d = H->d; a.rd = H->rd;
  a.T = T;
  a.targets = targets;
  a.Z = Z;
  a.zout = zout;
  a.status = H->status_d;
  a.Wz = H->hWz; a.Wug = H->hWug; a.Wd = H->hWd;
  head_widths(H, &a.wa, &a.wb);
  constexpr size_t kMax = 227 * 1024;
  if (head_smem(H, 8) <= kMax) launch_head_tb<8>(H, a, s);
  else launch_head_tb<4>(H, a, s);
}

}  // namespace stca
