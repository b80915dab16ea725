// Tensor-core per-target step of the STCA forward, between two attention
// layers ("Make It Long, Keep It Fast" digest §2.1):
//   output          o = [c_1 W_V^1 || ... || c_h W_V^h] W_O; Z[t, i, :] = o   (Eqs. (6), (8), (13))
//   query fusion    q = SwiGLUFFN_{i+1}([o(1) || ... || o(i+1) || x_t] W_C)  (Eq. (7))
//   u projection    u_j = (q W_Q^j) W_K^j^T, scaled for the next attention     (Eq. (13))
// and, before the first layer, q(1) = LN(SwiGLUFFN_1(x_t)) (Eq. (3)) and its u.
//
// A CTA takes 16 targets.  The dense products run on the tensor cores in
// transposed form, Y^T[features x 16] = W^T[features x K] X^T[K x 16]: one
// tcgen05.mma is a 128-feature block x 16 targets x 16 inputs, so a handful of
// targets still fills the MMA's M side (features) and the 16 targets are its N.
// The weights are laid out once, at set-up, as a stream of ready-made A tiles
// ([128 features x 64 inputs] bf16, 128-byte swizzle, 16 KB) in the order the
// kernel consumes them, and reach shared memory by plain bulk copies through a
// ring.  The activations X^T are written by the worker warps, as bf16, straight
// into the B-operand layout ([16 targets x 64 inputs] tiles, 2 KB); outputs
// come back from TMEM one feature per lane, 16 targets per lane.  The
// per-head products c_j W_V^j and P_j W_K^j^T are too narrow for an MMA (d_h
// columns) and stay on the CUDA cores.
//
// Warp roles (320 threads): warp 0 streams the weight tiles, warp 1 owns TMEM
// and issues the MMAs (one thread), warps 2-9 are workers (prologue,
// epilogues, the CUDA-core products).  Worker warp w reads TMEM lane quarter
// w % 4 and target columns 8 ((w - 2) / 4) .. +7.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "attn_tc_dev.cuh"
#include "stca_internal.h"
#include "tc_common.cuh"

namespace stca {
namespace {

using namespace tc;

constexpr int kTgt = 16;                  // targets per CTA (the MMA's N)
constexpr int kWorkers = 8;               // worker warps
constexpr int kStepThreads = 32 * (2 + kWorkers);
constexpr uint32_t kATile = 128u * 128u;  // A tile: 128 rows x 64 bf16
constexpr uint32_t kBTile = kTgt * 128u;  // B tile: 16 rows x 64 bf16
constexpr int kMaxRing = 10;              // A tiles in flight, at most (what fits is used)

// Byte offset of element (row r, column c) of a K-major tile whose rows hold
// 64 bf16 (128 B) with the 128-byte swizzle: 8-row atoms of 1024 B, the
// 16-byte chunk j of row r stored at chunk j ^ (r % 8).
__host__ __device__ inline uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((((c >> 3) ^ r) & 7) << 4) +
                               (c & 7) * 2);
}

}  // namespace

// ------------------------------------------------------------------ set-up
// A tiles of Y^T = W^T X^T for a row-major W [K x N] (K inputs, N outputs):
// tile (m, kc) holds output features r in [0, 128) of block m and inputs k in
// [64 kc, 64 kc + 64).  Block m is read from columns col0 .. col0 + 127 of the
// matrix src (row length ld): element (r, c) = src[(64 kc + c) ld + col0 + r].
namespace {
struct ColBlock {
  const float* src;
  int ld, col0;
};

TcGemm put_tiles(std::vector<uint16_t>& out, int K, const std::vector<ColBlock>& blocks) {
  TcGemm g;
  g.mb = static_cast<int>(blocks.size());
  g.kc = K / 64;
  g.tile0 = static_cast<int64_t>(out.size() / (kATile / 2));
  for (const ColBlock& b : blocks)
    for (int kc = 0; kc < g.kc; ++kc) {
      const size_t base = out.size();
      out.resize(base + kATile / 2, 0);
      uint16_t* t = out.data() + base;
      for (int r = 0; r < 128; ++r)
        for (int c = 0; c < 64; ++c) {
          const float f = b.src[static_cast<size_t>(kc * 64 + c) * b.ld + b.col0 + r];
          uint32_t u;
          memcpy(&u, &f, 4);
          t[sw128_off(r, c) / 2] = static_cast<uint16_t>(u >> 16);   // bf16-exact values
        }
    }
  return g;
}

std::vector<ColBlock> col_blocks(const float* W, int N) {
  std::vector<ColBlock> v;
  for (int m = 0; m < N / 128; ++m) v.push_back({W, N, 128 * m});
  return v;
}
}  // namespace

bool step_tc_supported(const stca_handle* H) {
  // d: one or two 128-feature blocks; rd <= 512: the FFN's 2 rd / 128 blocks
  // of 16 columns fit the 128 TMEM columns; M <= 8 bounds the W_C operand
  return H->elem == 2 && (H->d == 128 || H->d == 256) && H->rd % 128 == 0 && H->rd <= 512 &&
         H->d % H->h == 0 && H->dh % 2 == 0 && H->M <= 8;
}

// Lay out, per layer i, the A tiles of W_O, W_C (i >= 1), the query FFN
// (W_u and W_g blocks interleaved: block 2m = u features 128m.., block 2m+1 =
// g features of the same range, so one TMEM lane holds a matching u, g pair)
// and W_d, and W_Q.
int step_tc_setup(stca_handle* H, const std::vector<StepHostW>& layers, const HeadHostW& head) {
  const int d = H->d, rd = H->rd, M = H->M;
  std::vector<uint16_t> tiles;
  H->tcO.assign(M, TcGemm());
  H->tcC.assign(M, TcGemm());
  H->tcUG.assign(M, TcGemm());
  H->tcD.assign(M, TcGemm());
  H->tcQ.assign(M, TcGemm());
  H->tcK.assign(M, TcGemm());
  // u_j = P_j W_K^j^T on the tensor cores: d = 128 (one feature block) and
  // 16 h <= 128 (the (target, head) columns of one accumulator)
  const bool wk_tc = d == 128 && H->h <= 8;
  std::vector<float> wkt(wk_tc ? static_cast<size_t>(d) * d : 0);
  for (int i = 0; i < M; ++i) {
    const StepHostW& L = layers[i];
    H->tcO[i] = put_tiles(tiles, d, col_blocks(L.Wo, d));
    if (i > 0) H->tcC[i] = put_tiles(tiles, (i + 1) * d, col_blocks(L.Wc, d));
    std::vector<ColBlock> ug;
    for (int m = 0; m < rd / 128; ++m) {
      ug.push_back({L.qWu, rd, 128 * m});
      ug.push_back({L.qWg, rd, 128 * m});
    }
    H->tcUG[i] = put_tiles(tiles, d, ug);
    H->tcD[i] = put_tiles(tiles, rd, col_blocks(L.qWd, d));
    H->tcQ[i] = put_tiles(tiles, d, col_blocks(L.Wq, d));
    if (wk_tc) {
      // as a [inputs x outputs] matrix: input (j, c) = column j d_h + c of W_K, output feature f
      for (int f = 0; f < d; ++f)
        for (int k = 0; k < d; ++k) wkt[static_cast<size_t>(k) * d + f] = L.Wk[static_cast<size_t>(f) * d + k];
      H->tcK[i] = put_tiles(tiles, d, {ColBlock{wkt.data(), d, 0}});
    }
  }
  if (head.Wz) {
    // prediction head of Eq. (9), run by the last layer's step: W_Z over the
    // (M+1) d inputs [o(1) .. o(M) | x_t], its SwiGLU up/gate (blocks
    // interleaved as for the query FFN) and down projection
    H->tcZC = put_tiles(tiles, (M + 1) * d, col_blocks(head.Wz, d));
    std::vector<ColBlock> ug;
    for (int m = 0; m < rd / 128; ++m) {
      ug.push_back({head.zWu, rd, 128 * m});
      ug.push_back({head.zWg, rd, 128 * m});
    }
    H->tcZUG = put_tiles(tiles, d, ug);
    H->tcZD = put_tiles(tiles, rd, col_blocks(head.zWd, d));
    H->head_tc = true;
  }
  if (cudaMalloc(&H->wstep_tc, tiles.size() * 2) != cudaSuccess) {
    cudaGetLastError();
    return set_error(STCA_ENOMEM, "tensor-core step weight allocation failed");
  }
  STCA_CUDA_TRY(cudaMemcpy(H->wstep_tc, tiles.data(), tiles.size() * 2, cudaMemcpyHostToDevice));
  H->step_tc_ready = true;
  return STCA_OK;
}

// ------------------------------------------------------------------ kernel
namespace {

// kZ: the head's down product; kK: u_j = P_j W_K^j^T on the tensor cores,
// U^T[d features x (target, head)] = [W_K] Pblk, where Pblk (16 h rows x d) holds
// row (t, j) = P[t] on head j's d_h inputs and zeros elsewhere (Eq. (13))
enum : int { kO = 0, kC = 1, kUG = 2, kD = 3, kQ = 4, kZ = 5, kK = 6 };

struct StepTcArgs {
  int layer, M, d, h, dh, rd;
  int64_t T;
  const uint16_t* targets;      // T x d
  const float* cmerged;         // T x h x d: c_j = alpha_j X~ of the layer just attended,
                                // or NULL: merge the split partials here (plan, pacc, pm, pl)
  StepPlan plan;
  const float *pacc, *pm, *pl;  // split partials: G x d, G, G (log2 units)
  float* Z;                     // T x M x d
  uint16_t* Ubf;                // T x h x d: scaled u rows for the next attention
  const uint16_t* tiles;        // A-tile stream
  const uint16_t* Wv;           // d x d (this layer), layer >= 0
  const uint16_t* WkT;          // d_h x h d (next layer), layer < M - 1
  const float *q_ln_g, *q_ln_b;
  float uscale;
  int* status;
  int ng;                       // products in this launch
  TcGemm g[8];
  int kind[8];
  int nring;                    // A-tile ring stages
  int kch;                      // inputs per W_V staging chunk
  int naive;                    // naive form: cmerged is o_head (T x d); write packed q rows
  int nG, nTq;                  // its layout (NaiveLayout)
  const int64_t* qbase;         // first packed row of each request
  uint16_t* upk;                // packed query rows [rows x 64] bf16
  float* zout;                  // prediction head z (T x d) when the last layer runs it, or NULL
  int head_only;                // the head alone: its operand [o(1) .. o(M) | x_t] all from Z
  int proj;                     // the attention projected its rows by W_V already: 1 cmerged
                                // is o_head (T x d, merged); 2 merge the d_h-wide partials here
  const float* qml;             // proj 2: the attention's per-row slots (QslotBufs; pacc too)
  const int* qn;
  int wk_tc;                    // the W_K products run on the tensor cores (product kind kK)
  int qtot;                     // A tiles of this launch (kK's Pblk takes the next two ring slots)
  int defer_wait;               // query init right after this library's encoder launch: wait for
                                // the predecessor at the end, not the start (see launch_step_tc)
};

// Shared memory, in bytes (1024-aligned base): the A-tile ring, then the
// B-operand buffers of the five products, an fp32 scratch of d x 16 (the
// query projection P^T, features by targets), a reduction scratch, then the
// mbarriers.  bU .. the end of the scratch are not in use before the output
// product, so the W_V prologue stages its operands there.
struct StepLayout {
  uint32_t ring, bO, bC, bU, bH, bQ, scr, red, cw, bar, total;
};

// Split partials merged in the step: at most kMaxItems items per query row.
// For query row (t, j) of the CTA: cw_g[q][w] = partial row of item w (this
// row of it), cw_f[q][w] = its weight 2^(m_w - m) / L, cw_n[q] = items.  With
// more items per row the merge reads more partial rows than the separate
// combine kernel (spread over every SM) takes to read and merge them, so the
// host keeps that kernel then.
constexpr int kMaxItems = 2;
// With partials already projected by W_V (d_h floats per row) the merge reads
// d / d_h times less, and up to kCwItems items per row are merged here.
constexpr int kCwItems = 8;

__host__ __device__ inline StepLayout step_layout(int d, int rd, int M, int h, int nring) {
  StepLayout L;
  L.ring = 0;
  L.bO = L.ring + nring * kATile;
  L.bC = L.bO + (d / 64) * kBTile;
  L.bU = L.bC + ((M + 1) * d / 64) * kBTile;     // fusion inputs, up to the head's M + 1 blocks
  L.bH = L.bU + (d / 64) * kBTile;
  L.bQ = L.bH + (rd / 64) * kBTile;
  L.scr = L.bQ + (d / 64) * kBTile;
  L.red = L.scr + kTgt * d * 4;
  L.cw = L.red + 2 * 2 * 4 * 8 * 4;              // [2 stats][2 halves][4 quarters][8 targets]
  L.bar = L.cw + kTgt * h * (kCwItems * 8 + 4);
  L.bar = (L.bar + 7) & ~7u;
  L.total = L.bar + (2 * kMaxRing + 4) * 8 + 16;
  return L;
}

// Worker-only barrier (the 256 worker threads; id 1).  Every worker executes
// the same sequence of these, whatever its mbarrier waits returned.
__device__ __forceinline__ void workers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kWorkers) : "memory");
}

// Write a worker thread's 8 fp32 values (targets t8 .. t8 + 7 of input feature
// f of the next product) into the bf16 B-operand buffer `b` (tiles of 16
// targets x 64 inputs).  Lanes f and f ^ 1 pair up into bf16x2 words: the even
// lane stores targets t8 .. t8 + 3, the odd one t8 + 4 .. t8 + 7.
__device__ __forceinline__ void put_b8(uint8_t* b, int f, int t8, const float (&v)[8], int lane) {
  const bool even = (lane & 1) == 0;
  const int f0 = f & ~1;
  uint8_t* tile = b + (f0 >> 6) * kBTile;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
    const float lo = even ? v[j] : other, hi = even ? other : v[j];
    if ((j < 4) == even) {
      const uint32_t w = pack_bf16x2(lo, hi);
      *reinterpret_cast<uint32_t*>(tile + sw128_off(t8 + j, f0 & 63)) = w;
    }
  }
}

// Element (target t, input k) of a B buffer, bf16.
__device__ __forceinline__ void put_b1(uint8_t* b, int t, int k, float v) {
  *reinterpret_cast<__nv_bfloat16*>(b + (k >> 6) * kBTile + sw128_off(t, k & 63)) =
      __float2bfloat16_rn(v);
}

__device__ __forceinline__ float bf2f(uint16_t u) { return __uint_as_float(static_cast<uint32_t>(u) << 16); }

__device__ __forceinline__ bool step_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kWaitTimeoutNs) {
      atomicOr(status, kStatusStepTimeout);
      return false;
    }
  return true;
}

// The kernel's body for CTA `cta` of its grid (targets 16 cta ..), on dynamic
// shared memory smem_raw (its layout plus 1024 bytes of alignment slack).  The
// calling kernel may have more than kStepThreads threads: the extra warps
// take no part but the CTA-wide barriers.
__device__ __forceinline__ void step_tc_body(const StepTcArgs& a, uint8_t* smem_raw, int cta) {
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int d = a.d, h = a.h, dh = a.dh, rd = a.rd, L = a.layer;
  const int R = a.nring;
  const StepLayout Y = step_layout(d, rd, a.M, h, R);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Y.bar);
  uint64_t* empty = full + R;
  uint64_t* bready = empty + R;   // the workers have written a product's B operand
  uint64_t* aready = bready + 1;      // a product's MMAs are complete
  uint64_t* mdrain = aready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdrain + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(cta) * kTgt;
  const int nb = a.T - t0 < kTgt ? static_cast<int>(a.T - t0) : kTgt;
  uint8_t* bufs[6] = {sm + Y.bO, sm + Y.bC, sm + Y.bU, sm + Y.bH, sm + Y.bQ, sm + Y.bH};

  if (threadIdx.x == 0) {
    for (int i = 0; i < R; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(bready, kWorkers);
    mbar_init(aready, 1);
    mbar_init(mdrain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (!a.defer_wait) pdl_wait();       // the predecessor's results are visible from here on

  if (warp == 0) {
    // ------------------------------------------------------------ weight streamer
    if (lane == 0) {
      uint32_t q = 0;
      bool ok = true;
      for (int gi = 0; ok && gi < a.ng; ++gi) {
        const TcGemm G = a.g[gi];
        const int n = G.mb * G.kc;
        for (int t = 0; ok && t < n; ++t, ++q) {
          const int s = q % R;
          if (!(ok = step_wait(&empty[s], ((q / R) & 1) ^ 1, a.status))) break;
          mbar_arrive_expect_tx(&full[s], kATile);
          const uint16_t* src = a.tiles + (G.tile0 + t) * (kATile / 2);
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  smem_u32(sm + Y.ring + s * kATile)),
              "l"(src), "r"(kATile), "r"(smem_u32(&full[s]))
              : "memory");
        }
      }
      // let the copies in flight land before the CTA can exit
      for (uint32_t c = q > static_cast<uint32_t>(R) ? q - R : 0; c < q; ++c)
        step_wait(&full[c % R], (c / R) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, kTgt);
      uint32_t q = 0;
      bool ok = true;
      for (int gi = 0; ok && gi < a.ng; ++gi) {
        const TcGemm G = a.g[gi];
        if (!(ok = step_wait(bready, gi & 1, a.status))) break;
        tc_fence_after();
        const bool wk = a.kind[gi] == kK;
        const uint32_t bbase = wk ? 0u : smem_u32(bufs[a.kind[gi]]);
        const uint32_t id = wk ? idesc_bf16(128, kTgt * h) : idesc;
        for (int m = 0; ok && m < G.mb; ++m) {
          const uint32_t acc = tmem + m * kTgt;
          for (int kc = 0; kc < G.kc; ++kc, ++q) {
            const int s = q % R;
            if (!(ok = step_wait(&full[s], (q / R) & 1, a.status))) break;
            tc_fence_after();
            const uint32_t aaddr = smem_u32(sm + Y.ring + s * kATile);
            // kK: K tile kc of Pblk sits in ring slot (qtot + kc) % R
            const uint32_t baddr = wk ? smem_u32(sm + Y.ring + ((a.qtot + kc) % R) * kATile) : bbase + kc * kBTile;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              mma_bf16_ss(acc, sdesc_sw128(aaddr + k4 * 32, 16, 1024),
                          sdesc_sw128(baddr + k4 * 32, 16, 1024), id, (kc | k4) != 0);
            mma_commit(&empty[s]);
          }
        }
        if (!ok) break;
        mma_commit(aready);
      }
      mma_commit(mdrain);
      step_wait(mdrain, 0, a.status);
    }
  } else if (warp < 2 + kWorkers) {
    // ------------------------------------------------------------ workers
    const int wid = warp - 2;                 // 0..7
    const int tid = threadIdx.x - 64;         // 0..255
    const int q4 = warp & 3;                  // TMEM lane quarter
    const int t8 = 8 * (wid >> 2);            // target columns t8 .. t8 + 7
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    float* scr = reinterpret_cast<float*>(sm + Y.scr);
    float* red = reinterpret_cast<float*>(sm + Y.red);
    const int M = a.M;
    bool ok = true;
    const int nq = kTgt * h;                  // query rows of this CTA
    int32_t* cw_g = reinterpret_cast<int32_t*>(sm + Y.cw);
    float* cw_f = reinterpret_cast<float*>(cw_g + nq * kCwItems);
    int32_t* cw_n = reinterpret_cast<int32_t*>(cw_f + nq * kCwItems);
    // [o(1) .. o(L) | o(L+1): by the output epilogue | x_t] of Eq. (7), or of
    // the head's Eq. (9) after the last layer: the B operand of W_C (W_Z).
    // 8 inputs (one 16-byte chunk of a B row) per item, 4 items per thread and
    // batch.  The first batch's loads are issued before the combine tables are
    // built and stored after the first product has been released (unless this
    // operand is the first one, the head alone), so they overlap the tables
    // and W_O; the output epilogue fills block L.
    const int wcat8 = (L + 2) * d / 8, d8 = d / 8, ne_cat = L >= 0 ? kTgt * wcat8 : 0;
    auto concat_load = [&](int e0, uint4 (&v)[4]) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * 32 * kWorkers;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (e >= ne_cat) continue;
        const int t = e / wcat8, k8 = e - t * wcat8;
        const int blk = k8 / d8, kk = 8 * (k8 - blk * d8);
        if (t >= nb || (blk == L && !a.head_only)) continue;
        if (blk < L || (blk == L && a.head_only)) {
          const float4* z = reinterpret_cast<const float4*>(a.Z + ((t0 + t) * M + blk) * d + kk);
          const float4 z0 = z[0], z1 = z[1];
          v[u] = make_uint4(pack_bf16x2(z0.x, z0.y), pack_bf16x2(z0.z, z0.w),
                            pack_bf16x2(z1.x, z1.y), pack_bf16x2(z1.z, z1.w));
        } else {
          v[u] = *reinterpret_cast<const uint4*>(a.targets + (t0 + t) * d + kk);
        }
      }
    };
    auto concat_store = [&](int e0, const uint4 (&v)[4]) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * 32 * kWorkers;
        if (e >= ne_cat) break;
        const int t = e / wcat8, k8 = e - t * wcat8;
        if (k8 / d8 == L && !a.head_only) continue;
        *reinterpret_cast<uint4*>(bufs[kC] + (8 * k8 >> 6) * kBTile + sw128_off(t, (8 * k8) & 63)) = v[u];
      }
    };
    auto build_concat_rest = [&]() {       // batches after the first
      for (int e0 = tid + 4 * 32 * kWorkers; e0 < ne_cat; e0 += 4 * 32 * kWorkers) {
        uint4 v[4];
        concat_load(e0, v);
        concat_store(e0, v);
      }
    };
    const bool concat = L >= 0 && (L + 1 < M || a.zout);
    uint4 cat0[4];
    if (concat) concat_load(tid, cat0);
    if (L >= 0 && a.cmerged == nullptr && !a.head_only && a.proj != 2) {
      // split combine of Eq. (13)'s alpha_j X~: c_j = sum_w 2^(m_w - m) acc_w / L,
      // L = sum_w 2^(m_w - m) l_w, over the items w that cover query row (t, j)
      for (int qi = tid; qi < nq; qi += 32 * kWorkers) {
        const int t = qi / h, j = qi - t * h;
        int n = 0;
        if (t < nb) {
          const StepPlan& P = a.plan;
          const int r = P.treq[t0 + t];
          const int64_t qrow = (t0 + t - P.toff[r]) * h + j;
          const int64_t mt = qrow / P.mtile_rows, row = qrow - mt * P.mtile_rows;
          const int pair = P.req_pair_begin[r] + static_cast<int>(mt);
          const int w0 = P.pair_item_begin[pair];
          n = min(P.pair_item_begin[pair + 1] - w0, kCwItems);   // the host keeps n <= kCwItems
          float mw[kCwItems], lw[kCwItems], mx = -INFINITY;
#pragma unroll
          for (int w = 0; w < kCwItems; ++w)
            if (w < n) {
              const int64_t g = P.items[w0 + w].row_base + row;
              cw_g[qi * kCwItems + w] = static_cast<int32_t>(g);
              mw[w] = a.pm[g];
              lw[w] = a.pl[g];
              mx = fmaxf(mx, mw[w]);
            }
          float ls = 0.f;
#pragma unroll
          for (int w = 0; w < kCwItems; ++w)
            if (w < n) {
              mw[w] = exp2f(mw[w] - mx);
              ls = fmaf(lw[w], mw[w], ls);
            }
#pragma unroll
          for (int w = 0; w < kCwItems; ++w)
            if (w < n) cw_f[qi * kCwItems + w] = mw[w] / ls;
        }
        cw_n[qi] = n;
      }
      workers_sync();
    }
    // ---- prologue: the B operand of the launch's first product
    if (L < 0) {
      for (int e = tid; e < kTgt * d; e += 32 * kWorkers) {
        const int t = e / d, k = e - t * d;
        put_b1(bufs[kUG], t, k, t < nb ? bf2f(__ldcg(a.targets + (t0 + t) * d + k)) : 0.f);
      }
    } else {
      if (concat && a.head_only) {
        concat_store(tid, cat0);
        build_concat_rest();
      }
      if (a.head_only) {
        // nothing more: the head's operand is complete
      } else if (a.proj == 2) {
        // o_head[t][j d_h + c] = sum_w f_w po_w[c]: the items' rows, already
        // projected by W_V^j in the attention, merged into the B operand of W_O
        // a task is 4 columns of one query row (t, j), global row q = (t0 + t) h + j
        // of the attention's per-row slots: the row's item count, then every
        // item's (m, l) and 16 bytes of its projected partial, all in flight
        // at once; the weights 2^(m_w - m) / L are formed here
        const int dhh = a.dh, c4n = dhh / 4, ntask = nq * c4n;
        constexpr int kU = 2;
        for (int e0 = tid; e0 < ntask; e0 += kU * 32 * kWorkers) {
          int n[kU];
          int64_t qrow[kU];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int e = e0 + u * 32 * kWorkers;
            const int qi = e / c4n, t = qi / h;
            qrow[u] = (t0 + t) * h + (qi - t * h);
            n[u] = e < ntask && t < nb ? min(a.qn[qrow[u]], kQslots) : 0;
          }
          float4 v[kU][kQslots];
          float2 ml[kU][kQslots];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int e = e0 + u * 32 * kWorkers;
            const int c4 = e % c4n;
#pragma unroll
            for (int w = 0; w < kQslots; ++w) {
              const int64_t slot = qrow[u] * kQslots + w;
              v[u][w] = w < n[u] ? __ldg(reinterpret_cast<const float4*>(a.pacc + slot * dhh) + c4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
              ml[u][w] = w < n[u] ? __ldg(reinterpret_cast<const float2*>(a.qml) + slot) : make_float2(-INFINITY, 0.f);
            }
          }
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int e = e0 + u * 32 * kWorkers;
            if (e >= ntask) break;
            const int qi = e / c4n, c4 = e - qi * c4n;
            const int t = qi / h, j = qi - t * h;
            float mx = -INFINITY;
#pragma unroll
            for (int w = 0; w < kQslots; ++w) mx = fmaxf(mx, ml[u][w].x);
            float ls = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kQslots; ++w)
              if (w < n[u]) {
                const float f = exp2f(ml[u][w].x - mx);
                ls = fmaf(ml[u][w].y, f, ls);
                acc.x = fmaf(f, v[u][w].x, acc.x);
                acc.y = fmaf(f, v[u][w].y, acc.y);
                acc.z = fmaf(f, v[u][w].z, acc.z);
                acc.w = fmaf(f, v[u][w].w, acc.w);
              }
            const float inv = n[u] > 0 ? 1.0f / ls : 0.f;
            // 4 bf16 of row t, inputs j d_h + 4 c4 .. + 3 (8 bytes inside one 16-byte chunk)
            const int k = j * dhh + 4 * c4;
            *reinterpret_cast<uint2*>(bufs[kO] + (k >> 6) * kBTile + sw128_off(t, k & 63)) =
                make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
          }
        }
      } else if (a.naive || a.proj == 1) {
        // naive form: the per-head outputs o_head[t] (already alpha V per head)
        // are the B operand of W_O as they are
        const int d8 = d / 8;
        for (int e = tid; e < kTgt * d8; e += 32 * kWorkers) {
          const int t = e / d8, k8 = e - t * d8;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (t < nb) {
            const float4* z = reinterpret_cast<const float4*>(a.cmerged + (t0 + t) * d + 8 * k8);
            const float4 z0 = z[0], z1 = z[1];
            v = make_uint4(pack_bf16x2(z0.x, z0.y), pack_bf16x2(z0.z, z0.w),
                           pack_bf16x2(z1.x, z1.y), pack_bf16x2(z1.z, z1.w));
          }
          *reinterpret_cast<uint4*>(bufs[kO] + (8 * k8 >> 6) * kBTile + sw128_off(t, (8 * k8) & 63)) = v;
        }
      } else {
      // o_head = c_j W_V^j into the B operand of W_O.  Output column n belongs
      // to head n / d_h; a thread owns blocks of 4 targets x 2 columns and
      // accumulates them over the d inputs, which arrive in chunks of kch:
      // cs[j][k][t] (all heads' c_j, 16 targets contiguous) and ws[k][n]
      // (rows of W_V), staged in the buffers the later products use.
      const int kch = a.kch;
      float* cs = reinterpret_cast<float*>(sm + Y.bU);
      uint16_t* ws = reinterpret_cast<uint16_t*>(sm + Y.bU + kTgt * h * kch * 4);
      constexpr int kMaxBlk = 2;                      // 2 d / 256 blocks per thread, d <= 256
      float acc[kMaxBlk][4][2];
#pragma unroll
      for (int bi = 0; bi < kMaxBlk; ++bi)
#pragma unroll
        for (int t = 0; t < 4; ++t) acc[bi][t][0] = acc[bi][t][1] = 0.f;
      const int nblk = 2 * d;                         // (16 / 4) x (d / 2) blocks
      // per thread and chunk: at most kMaxC float4 of c_j and kMaxW uint4 of
      // W_V, all loaded before any is stored so the loads overlap
      constexpr int kMaxC = 8, kMaxW = 4;
      const int nc = kTgt * h * (kch / 4), nw = kch * d / 8;
      // the items of this thread are the same in every chunk: their source
      // offsets (at k0 = 0) and destinations, once; -1 marks no item
      int c_src[kMaxC], c_dst[kMaxC], c_q[kMaxC], c_k[kMaxC], w_src[kMaxW], w_dst[kMaxW];
#pragma unroll
      for (int i = 0; i < kMaxC; ++i) {
        const int e = tid + i * 32 * kWorkers;
        const int t = e % kTgt, rest = e / kTgt;
        const int j = rest % h, k4 = rest / h;
        c_dst[i] = e < nc ? (j * kch + 4 * k4) * kTgt + t : -1;
        c_src[i] = e < nc && t < nb ? (t * h + j) * d + 4 * k4 : -1;   // from this CTA's rows
        c_q[i] = t * h + j;                                            // its query row
        c_k[i] = 4 * k4;
      }
      const bool fused = a.cmerged == nullptr;
#pragma unroll
      for (int i = 0; i < kMaxW; ++i) {
        const int e = tid + i * 32 * kWorkers;
        const int k = e / (d / 8), c8 = e - k * (d / 8);
        w_src[i] = e < nw ? k * d + 8 * c8 : -1;
        w_dst[i] = w_src[i];
      }
      const float* cm = fused ? nullptr : a.cmerged + t0 * h * d;
      // chunk k0's operands into registers; with merged rows (no in-step merge)
      // the next chunk's loads are issued before this chunk's products, so they
      // are in flight while the products run
      float4 cv[kMaxC];
      uint4 wv[kMaxW];
      auto load_chunk = [&](int k0) {
#pragma unroll
        for (int i = 0; i < kMaxC; ++i) {
          cv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (c_src[i] < 0) continue;
          if (!fused) {
            cv[i] = __ldg(reinterpret_cast<const float4*>(cm + c_src[i] + k0));
          } else {
            const int q = c_q[i], n = cw_n[q];
            const int koff = c_k[i] + k0;
#pragma unroll
            for (int w = 0; w < kMaxItems; ++w)
              if (w < n) {
                const float f = cw_f[q * kCwItems + w];
                const float4 v = __ldg(reinterpret_cast<const float4*>(
                    a.pacc + static_cast<int64_t>(cw_g[q * kCwItems + w]) * d + koff));
                cv[i].x = fmaf(f, v.x, cv[i].x);
                cv[i].y = fmaf(f, v.y, cv[i].y);
                cv[i].z = fmaf(f, v.z, cv[i].z);
                cv[i].w = fmaf(f, v.w, cv[i].w);
              }
          }
        }
#pragma unroll
        for (int i = 0; i < kMaxW; ++i)
          if (w_src[i] >= 0) wv[i] = __ldg(reinterpret_cast<const uint4*>(a.Wv + k0 * d + w_src[i]));
      };
      if (!fused) load_chunk(0);
      for (int k0 = 0; k0 < d; k0 += kch) {
        if (fused) load_chunk(k0);
        // c_j[t][k0 .. k0 + kch) as cs[j][k][t]
#pragma unroll
        for (int i = 0; i < kMaxC; ++i)
          if (c_dst[i] >= 0) {
            float* dst = cs + c_dst[i];
            dst[0] = cv[i].x;
            dst[kTgt] = cv[i].y;
            dst[2 * kTgt] = cv[i].z;
            dst[3 * kTgt] = cv[i].w;
          }
        // W_V rows k0 .. k0 + kch
#pragma unroll
        for (int i = 0; i < kMaxW; ++i)
          if (w_dst[i] >= 0) *reinterpret_cast<uint4*>(ws + w_dst[i]) = wv[i];
        workers_sync();
        if (!fused && k0 + kch < d) load_chunk(k0 + kch);
#pragma unroll
        for (int bi = 0; bi < kMaxBlk; ++bi) {
          const int b = tid + bi * 32 * kWorkers;
          if (b < nblk) {
            const int t4 = b & 3, n = 2 * (b >> 2), j = n / dh;
            const float* cp = cs + j * kch * kTgt + 4 * t4;
            const uint16_t* wp = ws + n;
#pragma unroll 8
            for (int k = 0; k < kch; ++k) {
              const float4 c = *reinterpret_cast<const float4*>(cp + k * kTgt);
              const uint32_t w2 = *reinterpret_cast<const uint32_t*>(wp + k * d);
              const float w0 = __uint_as_float(w2 << 16), w1 = __uint_as_float(w2 & 0xFFFF0000u);
              acc[bi][0][0] = fmaf(c.x, w0, acc[bi][0][0]); acc[bi][0][1] = fmaf(c.x, w1, acc[bi][0][1]);
              acc[bi][1][0] = fmaf(c.y, w0, acc[bi][1][0]); acc[bi][1][1] = fmaf(c.y, w1, acc[bi][1][1]);
              acc[bi][2][0] = fmaf(c.z, w0, acc[bi][2][0]); acc[bi][2][1] = fmaf(c.z, w1, acc[bi][2][1]);
              acc[bi][3][0] = fmaf(c.w, w0, acc[bi][3][0]); acc[bi][3][1] = fmaf(c.w, w1, acc[bi][3][1]);
            }
          }
        }
        workers_sync();
      }
#pragma unroll
      for (int bi = 0; bi < kMaxBlk; ++bi) {
        const int b = tid + bi * 32 * kWorkers;
        if (b < nblk) {
          const int t4 = b & 3, n = 2 * (b >> 2);
          uint8_t* tile = bufs[kO] + (n >> 6) * kBTile;
#pragma unroll
          for (int t = 0; t < 4; ++t)
            *reinterpret_cast<uint32_t*>(tile + sw128_off(4 * t4 + t, n & 63)) =
                pack_bf16x2(acc[bi][t][0], acc[bi][t][1]);
        }
      }
      }   // reordered form
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bready);
    // the W_C operand, while W_O runs (its epilogue's fence covers these stores)
    if (concat && !a.head_only) {
      concat_store(tid, cat0);
      build_concat_rest();
    }

    // ---- epilogues
    for (int gi = 0; gi < a.ng; ++gi) {
      const int kind = a.kind[gi];
      const TcGemm G = a.g[gi];
      if (ok) ok = step_wait(aready, gi & 1, a.status);
      if (kind == kQ && a.wk_tc) {
        // Pblk's two ring slots (their last tiles' MMAs are complete): zero
        // them, then the epilogue below scatters P into its blocks
        for (int e = tid; e < 2 * static_cast<int>(kATile / 16); e += 32 * kWorkers)
          *reinterpret_cast<uint4*>(sm + Y.ring + ((a.qtot + e / (kATile / 16)) % R) * kATile +
                                    (e % (kATile / 16)) * 16) = make_uint4(0u, 0u, 0u, 0u);
        workers_sync();
      }
      __syncwarp();
      tc_fence_after();
      float vals[2][8];                       // up to two blocks of 128 features (d <= 256)
      if (kind == kK) {
        // U^T: lane = feature f, column n = t h + j; this warp takes columns
        // [64 hf, 64 hf + 64) (the rows (t, j) of U for targets t < nb).  The
        // warp's 64 x 32 block goes through shared memory (Pblk's ring slots,
        // free once these products are done) so that U's rows are written in
        // 16-byte pieces
        const int ncol = kTgt * h, hf = wid >> 2;
        uint16_t* stg = reinterpret_cast<uint16_t*>(sm + Y.ring + ((a.qtot + (wid >> 2)) % R) * kATile) +
                        q4 * 64 * 32;                            // [64 rows n][32 features] bf16
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int c0 = 64 * hf + 32 * c;
          if (c0 >= ncol) break;
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k)
            stg[(32 * c + k) * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[k]) * a.uscale));
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int ch = lane + 32 * i, row = ch >> 2, part = ch & 3;
          const int n = 64 * hf + row;
          if (n < ncol && n / h < nb)
            *reinterpret_cast<uint4*>(a.Ubf + (t0 * h + n) * static_cast<int64_t>(d) + 32 * q4 + 8 * part) =
                *reinterpret_cast<const uint4*>(stg + row * 32 + 8 * part);
        }
      } else if (kind == kUG) {
        for (int p = 0; p < G.mb / 2; ++p) {
          uint32_t u[8], g[8];
          tmem_ld8(tmem + lane_base + (2 * p) * kTgt + t8, u);
          tmem_ld8(tmem + lane_base + (2 * p + 1) * kTgt + t8, g);
          tmem_ld_wait();
          float hv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float gg = __uint_as_float(g[j]);
            hv[j] = __uint_as_float(u[j]) * __fdividef(gg, 1.0f + __expf(-gg));
          }
          put_b8(bufs[kD], 128 * p + 32 * q4 + lane, t8, hv, lane);
        }
      } else {
        // at most two blocks: the loops over m are unrolled so that vals stays in registers
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          if (m < G.mb) {
            uint32_t r[8];
            tmem_ld8(tmem + lane_base + m * kTgt + t8, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) vals[m][j] = __uint_as_float(r[j]);
          }
        }
        if (kind == kD && L < 0) {
          // LayerNorm of Eq. (3) over the d features of each target column:
          // features are spread over lanes, lane quarters and blocks; the
          // scale and shift of this thread's features are loaded first, so
          // they are in flight during the reductions
          float lg[2], lb[2];
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const int f = 128 * m + 32 * q4 + lane;
            lg[m] = m < G.mb ? __ldg(a.q_ln_g + f) : 0.f;
            lb[m] = m < G.mb ? __ldg(a.q_ln_b + f) : 0.f;
          }
          const float inv_d = 1.0f / d;
          float s[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            s[j] = vals[0][j] + (G.mb > 1 ? vals[1][j] : 0.f);
            for (int o = 16; o > 0; o >>= 1) s[j] += __shfl_xor_sync(0xffffffffu, s[j], o);
          }
          if (lane == 0)
            for (int j = 0; j < 8; ++j) red[((0 * 2 + (wid >> 2)) * 4 + q4) * 8 + j] = s[j];
          workers_sync();
          float mean[8], s2[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float tot = 0.f;
            for (int qq = 0; qq < 4; ++qq) tot += red[((0 * 2 + (wid >> 2)) * 4 + qq) * 8 + j];
            mean[j] = tot * inv_d;
            float e0 = vals[0][j] - mean[j];
            s2[j] = e0 * e0;
            if (G.mb > 1) { const float e1 = vals[1][j] - mean[j]; s2[j] = fmaf(e1, e1, s2[j]); }
            for (int o = 16; o > 0; o >>= 1) s2[j] += __shfl_xor_sync(0xffffffffu, s2[j], o);
          }
          if (lane == 0)
            for (int j = 0; j < 8; ++j) red[((1 * 2 + (wid >> 2)) * 4 + q4) * 8 + j] = s2[j];
          workers_sync();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float tot = 0.f;
            for (int qq = 0; qq < 4; ++qq) tot += red[((1 * 2 + (wid >> 2)) * 4 + qq) * 8 + j];
            const float rstd = rsqrtf(tot * inv_d + 1e-5f);
#pragma unroll
            for (int m = 0; m < 2; ++m)
              if (m < G.mb) vals[m][j] = (vals[m][j] - mean[j]) * rstd * lg[m] + lb[m];
          }
        }
        for (int m = 0; m < G.mb; ++m) {
          const int f = 128 * m + 32 * q4 + lane;
          if (kind == kO) {
            for (int j = 0; j < 8; ++j)
              if (t8 + j < nb) a.Z[((t0 + t8 + j) * M + L) * d + f] = vals[m][j];
            if (L + 1 < M || a.zout) put_b8(bufs[kC], L * d + f, t8, vals[m], lane);
          } else if (kind == kC) {
            put_b8(bufs[kUG], f, t8, vals[m], lane);
          } else if (kind == kD) {
            put_b8(bufs[kQ], f, t8, vals[m], lane);
          } else if (kind == kZ) {   // the head's token z of Eq. (9)
            for (int j = 0; j < 8; ++j)
              if (t8 + j < nb) a.zout[(t0 + t8 + j) * d + f] = vals[m][j];
          } else if (a.wk_tc) {   // kQ: P = q W_Q into Pblk, row t h + f / d_h, column f
            uint8_t* blk = sm + Y.ring + ((a.qtot + (f >> 6)) % R) * kATile;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<__nv_bfloat16*>(blk + sw128_off((t8 + j) * h + f / dh, f & 63)) =
                  __float2bfloat16_rn(vals[m][j]);
          } else {   // kQ: P = q W_Q in fp32, as P^T[feature][target] for the W_K products
            float4* dst = reinterpret_cast<float4*>(scr + f * kTgt + t8);
            dst[0] = make_float4(vals[m][0], vals[m][1], vals[m][2], vals[m][3]);
            dst[1] = make_float4(vals[m][4], vals[m][5], vals[m][6], vals[m][7]);
          }
        }
      }
      tc_fence_before();
      if (gi + 1 < a.ng) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bready);
      }
    }
    // ---- u_j = P_j W_K^j^T (Eq. (13)), scaled, as bf16 rows for the attention.
    // A thread owns blocks of 16 targets x 4 outputs (head j, columns k..k+3):
    // per c < d_h, one 8-byte load of W_K^T and the 16 targets' P[j d_h + c].
    if (L + 1 < M && a.naive) {
      // naive form: q W_Q of head j as row (j % G) Tq + tt of tile (j / G) nslots + qs
      // of the packed layout (target qs Tq + tt of its request), non-zero only in
      // the head's own d_h of the tile's 64 columns, scaled like u
      workers_sync();
      const int G = a.nG, Tq = a.nTq, ng8 = h * 8;
      for (int e = tid; e < kTgt * ng8; e += 32 * kWorkers) {
        const int t = e / ng8, rest = e - t * ng8;
        const int j = rest >> 3, c8 = rest & 7;
        if (t >= nb) continue;
        const int64_t tg = t0 + t;
        const int r = a.plan.treq[tg];
        const int64_t tl = tg - a.plan.toff[r], Tr = a.plan.toff[r + 1] - a.plan.toff[r];
        const int64_t nslots = (Tr + Tq - 1) / Tq, qs = tl / Tq, tt = tl - qs * Tq;
        const int jg = j / G, sl = j - jg * G;
        const int64_t row = a.qbase[r] + (jg * nslots + qs) * 128 + static_cast<int64_t>(sl) * Tq + tt;
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = 8 * c8 + u;                // column of the 64-wide packed row
          v[u] = c / dh == sl ? scr[(jg * 64 + c) * kTgt + t] * a.uscale : 0.f;
        }
        *reinterpret_cast<uint4*>(a.upk + row * 64 + 8 * c8) =
            make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                       pack_bf16x2(v[6], v[7]));
      }
    } else if (L + 1 < M && !a.wk_tc) {
      workers_sync();
      const int hd = h * d;
      for (int b = tid; b < hd / 4; b += 32 * kWorkers) {
        const int jk = 4 * b, j = jk / d;
        float acc[kTgt][4];
#pragma unroll
        for (int t = 0; t < kTgt; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
        for (int c0 = 0; c0 < dh; c0 += 8) {        // d_h is even; 8 loads in flight
          uint2 wk[8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (c0 + u < dh) wk[u] = __ldg(reinterpret_cast<const uint2*>(a.WkT + (c0 + u) * hd + jk));
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) {
            const int c = c0 + u8;
            if (c >= dh) break;
            const uint2 w = wk[u8];
            const float w0 = __uint_as_float(w.x << 16), w1 = __uint_as_float(w.x & 0xFFFF0000u);
            const float w2 = __uint_as_float(w.y << 16), w3 = __uint_as_float(w.y & 0xFFFF0000u);
            const float4* pp = reinterpret_cast<const float4*>(scr + (j * dh + c) * kTgt);
#pragma unroll
            for (int t4 = 0; t4 < 4; ++t4) {
              const float4 pv = pp[t4];
              const float pt[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                float* ac = acc[4 * t4 + u];
                ac[0] = fmaf(pt[u], w0, ac[0]);
                ac[1] = fmaf(pt[u], w1, ac[1]);
                ac[2] = fmaf(pt[u], w2, ac[2]);
                ac[3] = fmaf(pt[u], w3, ac[3]);
              }
            }
          }
        }
#pragma unroll
        for (int t = 0; t < kTgt; ++t)
          if (t < nb) {
            uint2 o;
            o.x = pack_bf16x2(acc[t][0] * a.uscale, acc[t][1] * a.uscale);
            o.y = pack_bf16x2(acc[t][2] * a.uscale, acc[t][3] * a.uscale);
            *reinterpret_cast<uint2*>(a.Ubf + (t0 + t) * hd + jk) = o;
          }
      }
    }
  }
  // deferred: this grid completes only after its predecessor has, so the
  // launches after it see the predecessor's results as well
  if (a.defer_wait) pdl_wait();
  tc_fence_before();
  __syncthreads();
  pdl_trigger();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

__global__ void __launch_bounds__(kStepThreads, 1) step_tc_kernel(const StepTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  step_tc_body(a, smem_raw, static_cast<int>(blockIdx.x));
}

}  // namespace

// ------------------------------------------------------------------ launch
// layer < 0: q(1) and its u; 0 <= layer < M-1: output of layer `layer`, then
// q(layer+2) and its u; layer = M-1: output only.  Writes the bf16 query rows
// scaled by log2(e) / sqrt(d_h) (the tensor-core attention's units).
int step_tc_max_items() { return kMaxItems; }

namespace {
// the deepest weight ring that fits in shared memory
int ring_stages(const stca_handle* H, int M) {
  int nring = kMaxRing;
  while (nring > 2 && step_layout(H->d, H->rd, M, H->h, nring).total + 1024 > 227u * 1024) --nring;
  return nring;
}
}  // namespace
int step_tc_max_items_proj() { return kQslots; }

// The prediction head of Eq. (9) alone, for T targets whose Z (T x M x d) is
// given: one launch of the step kernel with the head's three products.
int launch_step_tc_head(const stca_handle* H, const void* targets, int64_t T, const float* Z, float* zout,
                        cudaStream_t s) {
  if (T <= 0) return STCA_OK;
  if (!H->step_tc_ready || !H->head_tc) return set_error(STCA_ESTATE, "tensor-core head weights are not set up");
  const int M = H->M;
  StepTcArgs a{};
  a.layer = M - 1;
  a.M = M; a.d = H->d; a.h = H->h; a.dh = H->dh; a.rd = H->rd;
  a.T = T;
  a.targets = static_cast<const uint16_t*>(targets);
  a.Z = const_cast<float*>(Z);     // read only: the head writes zout
  a.tiles = H->wstep_tc;
  a.q_ln_g = H->q_ln_g;
  a.q_ln_b = H->q_ln_b;
  a.status = H->status_d;
  a.zout = zout;
  a.head_only = 1;
  a.kind[0] = kC; a.g[0] = H->tcZC;
  a.kind[1] = kUG; a.g[1] = H->tcZUG;
  a.kind[2] = kZ; a.g[2] = H->tcZD;
  a.ng = 3;
  int nring = kMaxRing;
  while (nring > 2 && step_layout(H->d, H->rd, M, H->h, nring).total + 1024 > 227u * 1024) --nring;
  const StepLayout Y = step_layout(H->d, H->rd, M, H->h, nring);
  if (Y.total + 1024 > 227u * 1024) return set_error(STCA_EINVAL, "tensor-core head: shared memory");
  a.nring = nring;
  a.kch = 4;
  const size_t smem = Y.total + 1024;
  cudaError_t e = cudaFuncSetAttribute(step_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("step_tc smem: ") + cudaGetErrorString(e));
  const unsigned grid = static_cast<unsigned>((T + kTgt - 1) / kTgt);
  e = launch_pdl(step_tc_kernel, dim3(grid), dim3(kStepThreads), smem, s, a);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("step_tc launch: ") + cudaGetErrorString(e));
  return STCA_OK;
}

namespace {
// The step kernel's arguments, shared memory and grid for one launch (T > 0).
int make_step_args(const stca_handle* H, int layer, const void* targets, int64_t T,
                   const float* cmerged, const StepPlan* plan, const float* part, int64_t G,
                   float* Z, uint16_t* Ubf, const NaiveStep* naive, float* zout, int proj,
                   const QslotBufs* qs, StepTcArgs& a, size_t& smem, unsigned& grid) {
  if (!H->step_tc_ready) return set_error(STCA_ESTATE, "tensor-core step weights are not set up");
  const int M = H->M;
  a = StepTcArgs{};
  a.layer = layer;
  a.M = M; a.d = H->d; a.h = H->h; a.dh = H->dh; a.rd = H->rd;
  a.T = T;
  a.targets = static_cast<const uint16_t*>(targets);
  a.cmerged = cmerged;
  if (layer >= 0 && cmerged == nullptr && proj != 2) {
    if (!plan || !part || G >= (int64_t(1) << 31))
      return set_error(STCA_EINVAL, "tensor-core step: no split partials to merge");
    a.plan = *plan;
    a.pacc = part;
    a.pm = part + G * H->d;
    a.pl = a.pm + G;
  }
  if (plan) a.plan = *plan;
  if (proj < 0 || proj > 2 || (proj && (naive || (proj == 1) != (cmerged != nullptr))))
    return set_error(STCA_EINVAL, "tensor-core step: bad projected-input mode");
  a.proj = layer >= 0 ? proj : 0;
  if (a.proj == 2) {
    if (!qs) return set_error(STCA_EINVAL, "tensor-core step: merging projected partials needs their row slots");
    a.pacc = qs->pacc;
    a.qml = qs->qml;
    a.qn = qs->qn;
  }
  if (naive) {
    if (!plan || (layer >= 0 && !cmerged))
      return set_error(STCA_EINVAL, "tensor-core step: the naive form needs o_head and the plan");
    a.naive = 1;
    a.nG = naive->G;
    a.nTq = naive->Tq;
    a.qbase = naive->qbase;
    a.upk = naive->upk;
  }
  a.Z = Z;
  a.Ubf = Ubf;
  a.tiles = H->wstep_tc;
  a.Wv = layer >= 0 ? static_cast<const uint16_t*>(H->Lstep[layer].Wv) : nullptr;
  a.WkT = layer + 1 < M ? static_cast<const uint16_t*>(H->Lstep[layer + 1].WkT) : nullptr;
  a.q_ln_g = H->q_ln_g;
  a.q_ln_b = H->q_ln_b;
  a.uscale = 1.4426950408889634f / sqrtf(static_cast<float>(H->dh));
  a.status = H->status_d;
  auto add = [&](int kind, const TcGemm& g) {
    a.kind[a.ng] = kind;
    a.g[a.ng] = g;
    ++a.ng;
  };
  if (layer >= 0) add(kO, H->tcO[layer]);
  if (zout) {
    if (layer != M - 1 || !H->head_tc)
      return set_error(STCA_EINVAL, "tensor-core step: the head runs after the last layer, with head weights");
    a.zout = zout;
    add(kC, H->tcZC);
    add(kUG, H->tcZUG);
    add(kZ, H->tcZD);
  }
  if (layer + 1 < M) {
    const int n = layer + 1;
    if (layer >= 0) add(kC, H->tcC[n]);
    add(kUG, H->tcUG[n]);
    add(kD, H->tcD[n]);
    add(kQ, H->tcQ[n]);
    // the W_K products on the tensor cores: their operand Pblk takes the two
    // ring slots after the launch's last A tiles, so the ring needs 4 slots
    if (!naive && H->tcK.size() == static_cast<size_t>(M) && H->tcK[n].tile0 >= 0 &&
        ring_stages(H, M) >= 4) {
      add(kK, H->tcK[n]);
      a.wk_tc = 1;
    }
  }
  for (int gi = 0; gi < a.ng; ++gi) a.qtot += a.g[gi].mb * a.g[gi].kc;
  // the deepest ring that fits, and the widest W_V staging chunk that fits
  // in the buffers it borrows
  int nring = kMaxRing;
  while (nring > 2 && step_layout(H->d, H->rd, M, H->h, nring).total + 1024 > 227u * 1024) --nring;
  const StepLayout Y = step_layout(H->d, H->rd, M, H->h, nring);
  if (Y.total + 1024 > 227u * 1024) return set_error(STCA_EINVAL, "tensor-core step: shared memory");
  // the W_V staging loads at most 8 float4 of c_j and 4 x 16 bytes of W_V per
  // worker thread and chunk
  auto stage_ok = [&](int k) {
    return static_cast<uint32_t>(kTgt * H->h * k * 4 + k * H->d * 2) <= Y.red - Y.bU &&
           kTgt * H->h * (k / 4) <= 8 * 32 * kWorkers && k * H->d / 8 <= 4 * 32 * kWorkers;
  };
  int kch = 32;
  while (kch > 4 && !stage_ok(kch)) kch /= 2;
  if (!stage_ok(kch))
    return set_error(STCA_EINVAL, "tensor-core step: too many heads for the W_V staging");
  a.nring = nring;
  a.kch = kch;
  smem = Y.total + 1024;
  grid = static_cast<unsigned>((T + kTgt - 1) / kTgt);
  return STCA_OK;
}

// One launch of the two independent halves of a pipeline phase: CTAs
// 0 .. nstep - 1 run a per-target step (one half of the batch), the others the
// next attention layer (the other half; the split-softmax kernel with its
// query tile in TMEM and W_V in the epilogue, d = 128).
__global__ void __launch_bounds__(kAttnThreads, 1)
pipe_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, const AttnParams p, const StepTcArgs a, int nstep) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int b = static_cast<int>(blockIdx.x);
  if (b < nstep) step_tc_body(a, smem_raw, b);
  else attn_tc_body<128, 1, 5, 1, false, true, true>(tmQ, tmK, tmV, p, smem_raw, b - nstep);
}
using PipeAttnCfg = AttnCfg<128, 1, 5, 1, false, true, true>;
static_assert(kStepThreads <= kAttnThreads, "the pipeline kernel runs both bodies");
}  // namespace

int launch_step_tc(const stca_handle* H, int layer, const void* targets, int64_t T,
                   const float* cmerged, const StepPlan* plan, const float* part, int64_t G,
                   float* Z, uint16_t* Ubf, cudaStream_t s, const NaiveStep* naive, float* zout,
                   int proj, const QslotBufs* qs, bool defer_wait) {
  if (T <= 0) return STCA_OK;
  StepTcArgs a;
  size_t smem;
  unsigned grid;
  if (int rc = make_step_args(H, layer, targets, T, cmerged, plan, part, G, Z, Ubf, naive, zout, proj, qs, a,
                              smem, grid))
    return rc;
  // The query init reads only the targets and the weights and writes only U
  // rows, so right after this library's encoder launch (which triggers its
  // dependents once its own wait is over) it may start on the SMs the
  // encoder's last, shorter round of tiles leaves idle, and wait for the
  // encoder at its end instead.
  a.defer_wait = defer_wait && layer < 0 ? 1 : 0;
  cudaError_t e = cudaFuncSetAttribute(step_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("step_tc smem: ") + cudaGetErrorString(e));
  e = launch_pdl(step_tc_kernel, dim3(grid), dim3(kStepThreads), smem, s, a);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("step_tc launch: ") + cudaGetErrorString(e));
  return STCA_OK;
}

int launch_step_attn_pipe(const stca_handle* H, const PipeStep& st, const PipeAttn& at, cudaStream_t s) {
  if (!attn_tc_proj_supported(H)) return set_error(STCA_EINVAL, "pipelined step: needs the in-kernel projection");
  StepTcArgs a{};
  size_t smem_s = 0;
  unsigned nstep = 0;
  if (st.T > 0)
    if (int rc = make_step_args(H, st.layer, st.targets, st.T, nullptr, nullptr, nullptr, 0, st.Z, st.Ubf,
                                nullptr, nullptr, 2, &st.qs, a, smem_s, nstep))
      return rc;
  AttnParams p{};
  p.items = at.items;
  p.cta_item_begin = at.cta_begin;
  p.pacc = at.qs.pacc;
  p.pm = p.pl = nullptr;               // per-row slots only
  p.status = H->status_d;
  p.stop_tiles = H->opt_stop_tiles;
  p.h = H->h;
  p.dh = H->dh;
  p.qslot = 1;
  p.pair_item_begin = at.qs.pair_item_begin;
  p.qml = at.qs.qml;
  p.qn = at.qs.qn;
  const unsigned agrid = at.grid > 0 ? static_cast<unsigned>(at.grid) : 0u;
  if (nstep + agrid == 0) return STCA_OK;
  const size_t smem = std::max<size_t>(smem_s, PipeAttnCfg::kSmem);
  cudaError_t e = cudaFuncSetAttribute(pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("pipe smem: ") + cudaGetErrorString(e));
  const CUtensorMap& tmK = H->tmXt[at.grid > 0 ? at.layer : 0];
  const CUtensorMap& tmV = H->tmWvT[at.grid > 0 ? at.layer : 0];
  e = launch_pdl(pipe_kernel, dim3(nstep + agrid), dim3(kAttnThreads), smem, s, H->tmU, tmK, tmV, p, a,
                 static_cast<int>(nstep));
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("pipe launch: ") + cudaGetErrorString(e));
  return STCA_OK;
}

}  // namespace stca
