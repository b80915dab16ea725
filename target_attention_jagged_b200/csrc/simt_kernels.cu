// CUDA-core kernels of the STCA forward: the row-wise SwiGLU+LayerNorm encoder
// and the split-L single-query attention.  They run the fp32 configuration
// (where tensor-core TF32 would not hold the 1e-3 bound) and the sizes the
// tensor-core kernels do not cover.  Sources: "Make
// It Long, Keep It Fast" digest §2.1, Eqs. (1)-(8) and (13).
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "softmax_exp.cuh"
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
// CUDA-core split-L single-query attention ("Make It Long, Keep It Fast"
// digest §2.1, Eq. (13)), for batches whose query rows per request (T_r h) are
// too few for a tensor-core tile, and for the fp32 configuration.  This
// key-per-group form serves the widths that the feature-per-lane kernel
// further down does not (d outside {32, 64, 128, 256}).
//
// One CTA takes one work item (a request's key range, at most a few thousand
// keys) and a block of up to kRowsPerCta(NCH) of the request's query rows, so
// the key range is read once for all of them.  The keys reach shared memory
// as whole tiles -- a request's history rows are contiguous, so one tile is
// one cp.async.bulk copy, completed on an mbarrier -- double-buffered so the
// next tile lands while this one is used.  A warp's lanes form groups of GL
// lanes (GL a power of two, at most 32); a group takes one key at a time and
// each lane holds NCH 4-feature chunks of it (16-byte shared loads for fp32,
// 8-byte for bf16); the dot products with the block's rows (kept in registers)
// are reduced over the group by warp shuffles.  Each group keeps its own online
// softmax state per row -- maximum m and sum l in log2 units, accumulator
// chunks -- rescaled lazily (only when a score exceeds m by more than 8); the
// groups' states are merged through shared memory at the end and written as
// the item's partial rows (accumulator, m, l in natural-log units) for the
// split combine.
constexpr int kSimtWarps = 4;
constexpr int kSimtThreads = 32 * kSimtWarps;
constexpr int kSimtStages = 2;

__host__ __device__ constexpr int simt_rows_per_cta(int nch) { return nch >= 8 ? 1 : 8 / nch; }

__device__ __forceinline__ void load_chunk_f32(const uint8_t* row, int c, float (&x)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(row + 16 * c);
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}

__device__ __forceinline__ void load_chunk_bf16(const uint8_t* row, int c, float (&x)[4]) {
  const uint2 v = *reinterpret_cast<const uint2*>(row + 8 * c);
  x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
  x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
}

__device__ __forceinline__ bool simt_wait(uint64_t* bar, uint32_t parity, int* status) {
  uint32_t ok;
  const long long t0 = clock64();
  for (;;) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))), "r"(parity)
        : "memory");
    if (ok) return true;
    if (clock64() - t0 > (1ll << 32)) {       // about two seconds
      atomicOr(status, kStatusAttnTimeout);
      return false;
    }
  }
}

template <bool XBF, int NCH>
__global__ void __launch_bounds__(kSimtThreads, 4)
attn_simt_kernel(const void* __restrict__ Xt, const float* __restrict__ U,
                 const AttnItem* __restrict__ items, const int32_t* __restrict__ pairs,
                 float* __restrict__ pacc, float* __restrict__ pm, float* __restrict__ pl, int d,
                 int GL, int kt, int us_off, int* status) {
  constexpr int RB = simt_rows_per_cta(NCH);
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ __align__(128) uint8_t smem_simt[];
  const int es = XBF ? 2 : 4;
  const int rowb = d * es;                                   // bytes per key row (multiple of 16)
  const size_t stage_bytes = static_cast<size_t>(kt) * rowb;
  uint8_t* stages = smem_simt;                                      // later: the merge area
  float* us = reinterpret_cast<float*>(smem_simt + us_off);                          // RB x d
  uint64_t* full = reinterpret_cast<uint64_t*>(us + RB * d);                  // kSimtStages
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item_i = pairs[2 * blockIdx.x], row0 = pairs[2 * blockIdx.x + 1];
  const AttnItem it = items[item_i];
  const int nrows = min(RB, it.rows - row0);
  const int ntiles = (it.nkeys + kt - 1) / kt;
  const uint8_t* src0 = static_cast<const uint8_t*>(Xt) + it.key0 * rowb;
  if (tid == 0) {
    for (int s = 0; s < kSimtStages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(
          static_cast<uint32_t>(__cvta_generic_to_shared(&full[s]))));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  auto issue = [&](int t) {           // thread 0: tile t into stage t % 2, one bulk copy
    const int s = t % kSimtStages;
    const int nk = min(kt, it.nkeys - t * kt);
    const uint32_t bytes = static_cast<uint32_t>(nk) * rowb;
    const uint32_t bar = static_cast<uint32_t>(__cvta_generic_to_shared(&full[s]));
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            static_cast<uint32_t>(__cvta_generic_to_shared(stages + s * stage_bytes))),
        "l"(src0 + static_cast<int64_t>(t) * stage_bytes), "r"(bytes), "r"(bar)
        : "memory");
  };
  if (tid == 0)
    for (int t = 0; t < min(ntiles, kSimtStages); ++t) issue(t);
  // the block's query rows, fp32, into shared memory and then registers
  for (int e = tid; e < RB * d; e += kSimtThreads) {
    const int r = e / d;
    us[e] = r < nrows ? U[(it.qrow0 + row0 + r) * d + (e - r * d)] : 0.f;
  }
  __syncthreads();
  const int gq = lane / GL, li = lane % GL;        // group within the warp, lane within the group
  const int kpw = 32 / GL;                         // keys per warp step
  const int nch = d / 4;                           // 4-feature chunks in a row
  float ur[RB][NCH][4];
#pragma unroll
  for (int r = 0; r < RB; ++r)
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = li + GL * i;
#pragma unroll
      for (int k = 0; k < 4; ++k) ur[r][i][k] = c < nch ? us[r * d + 4 * c + k] : 0.f;
    }
  float m[RB], l[RB], acc[RB][NCH][4];
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[r][i][k] = 0.f;
  }
  bool ok = true;
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % kSimtStages;
    if (ok) ok = simt_wait(&full[s], (t / kSimtStages) & 1, status);
    ok = __syncthreads_and(ok) != 0;      // one decision for the whole CTA (the loop below shuffles)
    const int nk = min(kt, it.nkeys - t * kt);
    const uint8_t* tile = stages + s * stage_bytes;
    if (ok) {
      // warp-uniform trip count: every lane of the warp takes part in the
      // shuffles below; a group whose key lies past the tile's end computes on
      // zeros and leaves its state unchanged
      for (int kb = warp * kpw; kb < nk; kb += kSimtWarps * kpw) {
        const int k = kb + gq;
        const bool valid = k < nk;
        const uint8_t* xrow = tile + static_cast<size_t>(valid ? k : 0) * rowb;
        float x[NCH][4];
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int c = li + GL * i;
          if (valid && c < nch) {
            if constexpr (XBF) load_chunk_bf16(xrow, c, x[i]);
            else load_chunk_f32(xrow, c, x[i]);
          } else {
            x[i][0] = x[i][1] = x[i][2] = x[i][3] = 0.f;
          }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          float sc = 0.f;
#pragma unroll
          for (int i = 0; i < NCH; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) sc = fmaf(ur[r][i][q], x[i][q], sc);
          for (int o = GL >> 1; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
          if (!valid) continue;
          const float s2 = sc * kLog2e;              // log2 units
          if (s2 > m[r] + 8.0f) {                    // lazy rescale (always on the first key)
            const float corr = sx::ex2(m[r] - s2);    // 0 from m = -inf
            l[r] *= corr;
#pragma unroll
            for (int i = 0; i < NCH; ++i)
#pragma unroll
              for (int q = 0; q < 4; ++q) acc[r][i][q] *= corr;
            m[r] = s2;
          }
          const float p = sx::ex2(s2 - m[r]);
          l[r] += p;
#pragma unroll
          for (int i = 0; i < NCH; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[r][i][q] = fmaf(p, x[i][q], acc[r][i][q]);
        }
      }
    }
    __syncthreads();                      // every warp is done with stage s
    if (tid == 0 && ok && t + kSimtStages < ntiles) issue(t + kSimtStages);
  }
  // let copies still in flight (after a failed wait) land before the stages are reused
  // (on the normal path these phases are complete and the waits return at once)
  if (tid == 0)
    for (int t = max(0, ntiles - kSimtStages); t < ntiles; ++t)
      simt_wait(&full[t % kSimtStages], (t / kSimtStages) & 1, status);
  __syncthreads();
  // merge the groups' states: state g = (warp, group) -> [RB rows][d + 2] floats
  const int ngroups = kSimtWarps * kpw;
  float* st = reinterpret_cast<float*>(smem_simt);            // the stages are free now
  const int g = warp * kpw + gq;
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    float* row = st + (static_cast<size_t>(g) * RB + r) * (d + 2);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = li + GL * i;
      if (c < nch)
#pragma unroll
        for (int q = 0; q < 4; ++q) row[4 * c + q] = acc[r][i][q];
    }
    if (li == 0) { row[d] = m[r]; row[d + 1] = l[r]; }
  }
  __syncthreads();
  for (int e = tid; e < nrows * d; e += kSimtThreads) {
    const int r = e / d, f = e - r * d;
    float mx = -INFINITY;
    for (int q = 0; q < ngroups; ++q) mx = fmaxf(mx, st[(static_cast<size_t>(q) * RB + r) * (d + 2) + d]);
    float a = 0.f, lsum = 0.f;
    for (int q = 0; q < ngroups; ++q) {
      const float* row = st + (static_cast<size_t>(q) * RB + r) * (d + 2);
      const float w = row[d + 1] > 0.f ? sx::ex2(row[d] - mx) : 0.f;   // a group with no key: 0
      a = fmaf(w, row[f], a);
      lsum = fmaf(w, row[d + 1], lsum);
    }
    const int64_t gr = it.row_base + row0 + r;
    pacc[gr * d + f] = a;
    if (f == 0) {
      pm[gr] = mx * 0.6931471805599453f;              // natural-log units for the combine
      pl[gr] = lsum;
    }
  }
}

// ---------------------------------------------------------------------------
// The same attention for d in {32, 64, 128, 256} (F = d / 32 features per
// lane), built so that the history is read at close to HBM speed when a
// request has few query rows.
//
// One CTA of 8 warps takes a work item and a block of up to 16 of the
// request's query rows (QB, the smallest of 4, 8, 16 that holds the batch's
// largest block).  Key tiles arrive as before, one bulk copy per tile into a
// double-buffered ring.  A warp takes KG keys at a time (16; 8 for d = 256)
// and keeps them in registers, F features per lane: lane l holds features
// l F .. l F + F - 1 of every key, read as one contiguous shared-memory row
// per key.  Per query row it forms the KG partial dot products of its lane's
// features, and a reduce-scatter over the lanes (KG - 1 shuffles, then one
// per remaining lane bit) leaves lane l with the whole score of key
// l mod KG.  With QB = 4 the kernel is held to 128 registers, so two CTAs
// share an SM.  The online softmax (maximum m and sum in log2 units) then needs
// one max-reduction per group, and the P-weighted sum over the group's keys
// broadcasts each key's weight from the lane that holds it.  The warps'
// states are merged through shared memory at the end and written as the
// item's partial rows, as above.
constexpr int kS2Warps = 8;
constexpr int kS2Threads = 32 * kS2Warps;
constexpr int kS2Stages = 2;
constexpr int kS2MaxRows = 16;

template <bool XBF, int F>
__device__ __forceinline__ void s2_load_key(const uint8_t* row, int lane, float (&x)[F]) {
  if constexpr (XBF) {
    const uint8_t* p = row + lane * (2 * F);
    if constexpr (F == 1) {
      x[0] = __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p)) << 16);
    } else if constexpr (F == 2) {
      const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
      x[0] = __uint_as_float(v << 16); x[1] = __uint_as_float(v & 0xFFFF0000u);
    } else if constexpr (F == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
      x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
    } else {
      const uint4 v = *reinterpret_cast<const uint4*>(p);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
  } else {
    const float* p = reinterpret_cast<const float*>(row) + lane * F;
    if constexpr (F == 1) {
      x[0] = p[0];
    } else if constexpr (F == 2) {
      const float2 v = *reinterpret_cast<const float2*>(p);
      x[0] = v.x; x[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < F / 4; ++i) {
        const float4 v = reinterpret_cast<const float4*>(p)[i];
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
      }
    }
  }
}

// v[k] holds this lane's partial sum for key k of the group (k < KG).  Returns
// the sum over all 32 lanes for key (lane mod KG).  Round b (KG/2, ..., 1):
// the lane keeps the half of its values whose key bit b equals its own lane
// bit b, and adds the partner's (lane ^ b) copy of that half; after the
// rounds, the lanes of an aligned group of KG hold the group's sums, and the
// remaining lane bits are summed by plain butterflies.
template <int KG>
__device__ __forceinline__ float s2_reduce_scatter(float (&v)[KG], int lane) {
#pragma unroll
  for (int b = KG / 2; b >= 1; b >>= 1) {
    const bool hi = (lane & b) != 0;
#pragma unroll
    for (int j = 0; j < b; ++j) {
      const float keep = hi ? v[j + b] : v[j];
      const float send = hi ? v[j] : v[j + b];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, b);
    }
  }
  float s = v[0];
#pragma unroll
  for (int o = KG; o < 32; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

template <bool XBF, int F, int QB>
__global__ void __launch_bounds__(kS2Threads, QB <= 4 ? 2 : 1)
attn_simt2_kernel(const void* __restrict__ Xt, const float* __restrict__ U,
                  const AttnItem* __restrict__ items, const int32_t* __restrict__ pairs,
                  float* __restrict__ pacc, float* __restrict__ pm, float* __restrict__ pl, int kt,
                  int us_off, int* status) {
  constexpr int D = 32 * F;
  constexpr int KG = F >= 8 ? 8 : 16;                  // keys per warp step
  constexpr int ROWB = D * (XBF ? 2 : 4);              // bytes per key row (a multiple of 16)
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ __align__(128) uint8_t smem_s2[];
  const size_t stage_bytes = static_cast<size_t>(kt) * ROWB;
  uint8_t* stages = smem_s2;                                        // later: the merge area
  float* us = reinterpret_cast<float*>(smem_s2 + us_off);           // QB x D query rows
  uint64_t* full = reinterpret_cast<uint64_t*>(us + QB * D);        // kS2Stages
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item_i = pairs[2 * blockIdx.x], row0 = pairs[2 * blockIdx.x + 1];
  const AttnItem it = items[item_i];
  const int nrows = min(QB, it.rows - row0);
  const int ntiles = (it.nkeys + kt - 1) / kt;
  const uint8_t* src0 = static_cast<const uint8_t*>(Xt) + it.key0 * ROWB;
  if (tid == 0) {
    for (int s = 0; s < kS2Stages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(
          static_cast<uint32_t>(__cvta_generic_to_shared(&full[s]))));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  auto issue = [&](int t) {           // thread 0: tile t into stage t % 2, one bulk copy
    const int s = t % kS2Stages;
    const int nk = min(kt, it.nkeys - t * kt);
    const uint32_t bytes = static_cast<uint32_t>(nk) * ROWB;
    const uint32_t bar = static_cast<uint32_t>(__cvta_generic_to_shared(&full[s]));
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            static_cast<uint32_t>(__cvta_generic_to_shared(stages + s * stage_bytes))),
        "l"(src0 + static_cast<int64_t>(t) * stage_bytes), "r"(bytes), "r"(bar)
        : "memory");
  };
  if (tid == 0)
    for (int t = 0; t < min(ntiles, kS2Stages); ++t) issue(t);
  for (int e = tid; e < QB * D; e += kS2Threads) {
    const int r = e / D;
    us[e] = r < nrows ? U[(it.qrow0 + row0 + r) * D + (e - r * D)] : 0.f;
  }
  __syncthreads();
  float m[QB], lsum[QB], acc[QB][F];
#pragma unroll
  for (int q = 0; q < QB; ++q) {
    m[q] = -INFINITY;
    lsum[q] = 0.f;
#pragma unroll
    for (int f = 0; f < F; ++f) acc[q][f] = 0.f;
  }
  const int myk = lane & (KG - 1);      // the key of the group whose score this lane ends with
  bool ok = true;
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % kS2Stages;
    if (ok) ok = simt_wait(&full[s], (t / kS2Stages) & 1, status);
    ok = __syncthreads_and(ok) != 0;      // one decision for the whole CTA (the loop below shuffles)
    const int nk = min(kt, it.nkeys - t * kt);
    const uint8_t* tile = stages + s * stage_bytes;
    if (ok) {
      for (int g0 = warp * KG; g0 < nk; g0 += kS2Warps * KG) {   // warp-uniform trip count
        float x[KG][F];
#pragma unroll
        for (int k = 0; k < KG; ++k) {
          if (g0 + k < nk) {
            s2_load_key<XBF, F>(tile + static_cast<size_t>(g0 + k) * ROWB, lane, x[k]);
          } else {
#pragma unroll
            for (int f = 0; f < F; ++f) x[k][f] = 0.f;
          }
        }
        const bool kvalid = g0 + myk < nk;
#pragma unroll
        for (int q = 0; q < QB; ++q) {
          if (q >= nrows) break;                              // CTA-uniform
          float uq[F];
#pragma unroll
          for (int f = 0; f < F; ++f) uq[f] = us[q * D + lane * F + f];
          float v[KG];
#pragma unroll
          for (int k = 0; k < KG; ++k) {
            float a = 0.f;
#pragma unroll
            for (int f = 0; f < F; ++f) a = fmaf(uq[f], x[k][f], a);
            v[k] = a;
          }
          const float sc = s2_reduce_scatter<KG>(v, lane);
          const float s2 = kvalid ? sc * kLog2e : -INFINITY;   // log2 units
          float gm = s2;
#pragma unroll
          for (int o = 1; o < KG; o <<= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
          if (gm > m[q]) {                                      // warp-uniform
            const float corr = sx::ex2(m[q] - gm);              // 0 from m = -inf
            lsum[q] *= corr;
#pragma unroll
            for (int f = 0; f < F; ++f) acc[q][f] *= corr;
            m[q] = gm;
          }
          const float p = kvalid ? sx::ex2(s2 - m[q]) : 0.f;
          if (lane < KG) lsum[q] += p;                          // one copy of each key's weight
#pragma unroll
          for (int k = 0; k < KG; ++k) {
            const float pk = __shfl_sync(0xffffffffu, p, k);
#pragma unroll
            for (int f = 0; f < F; ++f) acc[q][f] = fmaf(pk, x[k][f], acc[q][f]);
          }
        }
      }
    }
    __syncthreads();                      // every warp is done with stage s
    if (tid == 0 && ok && t + kS2Stages < ntiles) issue(t + kS2Stages);
  }
  // let copies still in flight (after a failed wait) land before the stages are reused
  if (tid == 0)
    for (int t = max(0, ntiles - kS2Stages); t < ntiles; ++t)
      simt_wait(&full[t % kS2Stages], (t / kS2Stages) & 1, status);
  __syncthreads();
  // merge the warps' states: warp w, row q -> [D + 2] floats (accumulator, m, l)
  float* st = reinterpret_cast<float*>(smem_s2);              // the stages are free now
#pragma unroll
  for (int q = 0; q < QB; ++q) {
    if (q >= nrows) break;
    float* row = st + (static_cast<size_t>(warp) * QB + q) * (D + 2);
#pragma unroll
    for (int f = 0; f < F; ++f) row[lane * F + f] = acc[q][f];
    float ls = lsum[q];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    if (lane == 0) { row[D] = m[q]; row[D + 1] = ls; }
  }
  __syncthreads();
  for (int e = tid; e < nrows * D; e += kS2Threads) {
    const int r = e / D, f = e - r * D;
    float mx = -INFINITY;
    for (int w = 0; w < kS2Warps; ++w) mx = fmaxf(mx, st[(static_cast<size_t>(w) * QB + r) * (D + 2) + D]);
    float a = 0.f, lt = 0.f;
    for (int w = 0; w < kS2Warps; ++w) {
      const float* row = st + (static_cast<size_t>(w) * QB + r) * (D + 2);
      const float wt = row[D + 1] > 0.f ? sx::ex2(row[D] - mx) : 0.f;   // a warp with no key: 0
      a = fmaf(wt, row[f], a);
      lt = fmaf(wt, row[D + 1], lt);
    }
    const int64_t gr = it.row_base + row0 + r;
    pacc[gr * D + f] = a;
    if (f == 0) {
      pm[gr] = mx * 0.6931471805599453f;              // natural-log units for the combine
      pl[gr] = lt;
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

namespace {
// Launch geometry of the CUDA-core attention for width d: NCH chunks of 4
// features per lane, GL lanes per key (a power of two), kt keys per tile.
struct SimtGeom {
  int nch, gl, kt, rb;
  size_t us_off, smem;
};

SimtGeom simt_geom(int d, int elem) {
  SimtGeom g{};
  const int chunks = d / 4;
  g.nch = 1;
  while (g.nch * 32 < chunks) g.nch *= 2;                  // 1, 2, 4, 8 (d <= 1024)
  g.gl = 1;
  while (g.gl * g.nch < chunks && g.gl < 32) g.gl *= 2;
  g.rb = simt_rows_per_cta(g.nch);
  const int rowb = d * elem;
  g.kt = std::max(8, std::min(256, (24 << 10) / rowb) / 8 * 8);   // up to 24 KB per stage
  const size_t stages = static_cast<size_t>(kSimtStages) * g.kt * rowb;
  const size_t merge = static_cast<size_t>(kSimtWarps) * (32 / g.gl) * g.rb * (d + 2) * sizeof(float);
  // the stages, reused as the merge area at the end; then the query rows and
  // the mbarriers
  g.us_off = (std::max(stages, merge) + 15) / 16 * 16;
  g.smem = g.us_off + static_cast<size_t>(g.rb) * d * sizeof(float) + 64;
  return g;
}
}  // namespace

namespace {
// The feature-per-lane kernel covers d in {32, 64, 128, 256}; other widths
// take the key-per-group kernel above.
bool simt2_supported(int d) { return d == 32 || d == 64 || d == 128 || d == 256; }

struct Simt2Geom {
  int kt;
  size_t us_off, smem;
};

// kt keys per tile (at most 32 KB a stage); shared memory for QB rows: the
// stages (reused as the warps' merge area), the query rows, the mbarriers
Simt2Geom simt2_geom(int d, int elem, int qb) {
  Simt2Geom g{};
  const int rowb = d * elem;
  g.kt = std::max(8, std::min(256, (32 << 10) / rowb) / 8 * 8);
  const size_t stages = static_cast<size_t>(kS2Stages) * g.kt * rowb;
  const size_t merge = static_cast<size_t>(kS2Warps) * qb * (d + 2) * sizeof(float);
  g.us_off = (std::max(stages, merge) + 15) / 16 * 16;
  g.smem = g.us_off + static_cast<size_t>(qb) * d * sizeof(float) + 64;
  return g;
}
}  // namespace

int attn_simt_rows_per_cta(int d) { return simt2_supported(d) ? kS2MaxRows : simt_geom(d, 4).rb; }

size_t attn_simt_smem(const stca_handle* H) {
  return simt2_supported(H->d) ? simt2_geom(H->d, H->elem, kS2MaxRows).smem : simt_geom(H->d, H->elem).smem;
}

void launch_attn_simt(const stca_handle* H, int layer, const void* xt_layer,
                      const AttnItem* items_d, const int32_t* pairs_d, int64_t npairs,
                      const int64_t* toff_d, cudaStream_t s) {
  (void)layer;
  (void)toff_d;
  if (npairs <= 0) return;
  const int64_t G = H->last_G;
  float* pacc = H->part;
  float* pm = pacc + G * H->d;
  float* pl = pm + G;
  if (simt2_supported(H->d)) {
    // QB: the smallest of 4, 8, 16 rows that holds every (item, row block)
    int64_t most = 1;
    for (size_t r = 0; r + 1 < H->last_toff.size(); ++r)
      most = std::max<int64_t>(most, (H->last_toff[r + 1] - H->last_toff[r]) * H->h);
    const int qb = most <= 4 ? 4 : most <= 8 ? 8 : kS2MaxRows;
    const Simt2Geom g = simt2_geom(H->d, H->elem, qb);
#define STCA_SIMT2(XB, FF, QQ)                                                                      \
  do {                                                                                              \
    auto k = attn_simt2_kernel<XB, FF, QQ>;                                                         \
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.smem);              \
    k<<<static_cast<unsigned>(npairs), kS2Threads, g.smem, s>>>(xt_layer, H->U, items_d, pairs_d,   \
                                                                pacc, pm, pl, g.kt, (int)g.us_off,  \
                                                                H->status_d);                       \
  } while (0)
#define STCA_SIMT2_Q(XB, FF)                        \
  do {                                              \
    if (qb == 4) STCA_SIMT2(XB, FF, 4);             \
    else if (qb == 8) STCA_SIMT2(XB, FF, 8);        \
    else STCA_SIMT2(XB, FF, kS2MaxRows);            \
  } while (0)
    const bool bf = H->elem == 2;
    switch (H->d) {
      case 32: if (bf) STCA_SIMT2_Q(true, 1); else STCA_SIMT2_Q(false, 1); break;
      case 64: if (bf) STCA_SIMT2_Q(true, 2); else STCA_SIMT2_Q(false, 2); break;
      case 128: if (bf) STCA_SIMT2_Q(true, 4); else STCA_SIMT2_Q(false, 4); break;
      default: if (bf) STCA_SIMT2_Q(true, 8); else STCA_SIMT2_Q(false, 8); break;
    }
#undef STCA_SIMT2_Q
#undef STCA_SIMT2
    return;
  }
  const SimtGeom g = simt_geom(H->d, H->elem);
#define STCA_SIMT(XB, NC)                                                                          \
  do {                                                                                             \
    auto k = attn_simt_kernel<XB, NC>;                                                             \
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.smem);             \
    k<<<static_cast<unsigned>(npairs), kSimtThreads, g.smem, s>>>(xt_layer, H->U, items_d, pairs_d, \
                                                                  pacc, pm, pl, H->d, g.gl, g.kt,  \
                                                                  (int)g.us_off, H->status_d);     \
  } while (0)
  const bool bf = H->elem == 2;
  switch (g.nch) {
    case 1: if (bf) STCA_SIMT(true, 1); else STCA_SIMT(false, 1); break;
    case 2: if (bf) STCA_SIMT(true, 2); else STCA_SIMT(false, 2); break;
    case 4: if (bf) STCA_SIMT(true, 4); else STCA_SIMT(false, 4); break;
    default: if (bf) STCA_SIMT(true, 8); else STCA_SIMT(false, 8); break;
  }
#undef STCA_SIMT
}

}  // namespace stca
