// Internal declarations shared by the STCA library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "stca.h"

namespace stca {

// ---------------------------------------------------------------- errors
int set_error(int code, const std::string& msg);

#define STCA_CUDA_TRY(expr)                                                              \
  do {                                                                                   \
    cudaError_t _e = (expr);                                                             \
    if (_e != cudaSuccess)                                                               \
      return ::stca::set_error(STCA_ECUDA, std::string(#expr) + ": " + cudaGetErrorString(_e)); \
  } while (0)

// Device status word bits written by kernels that give up a bounded wait.
enum : int { kStatusEncodeTimeout = 1, kStatusAttnTimeout = 2, kStatusStepTimeout = 4, kStatusKvTimeout = 8 };

// ---------------------------------------------------------------- work plan
// One attention work item: a contiguous key range of one request's history
// against one tile of its query rows (all T_r * h rows on the CUDA-core path,
// up to 128 rows on the tensor-core path).
struct AttnItem {
  int32_t req;        // request index
  int32_t nkeys;      // keys in this range (>= 1)
  int64_t key0;       // first history row (absolute row in X~)
  int64_t row_base;   // first partial row written by this item
  int64_t qrow0;      // first query row (row of U: target * h + head)
  int32_t mt;         // query tile index within the request
  int32_t rows;       // query rows of this tile that belong to the request
  int32_t kcol;       // naive form: first feature of the tile's head group in K and V
  int32_t pair;       // (request, query tile) pair of the item (tensor-core path)
};

// Query layout of the naive-form attention (Eq. (12) with K = X~ W_K and
// V = X~ W_V projected once per request): G = 64 / d_h heads share a tile, each
// with Tq = 128 / G query positions.  Request r has nslots = ceil(T_r / Tq)
// slots and (h / G) * nslots tiles of 128 rows, tile mt = jg * nslots + qs
// holding rows s * Tq + tt for head j = jg * G + s and target qs * Tq + tt.
struct NaiveLayout {
  int G = 0, Tq = 0;
};

// Per-layer pointers into the handle's fp32 weight slab (CUDA-core kernels and
// the per-target kernels).
struct LayerW32 {
  const float *Wu, *Wg, *Wd;        // history FFN: d x rd, d x rd, rd x d
  const float *qWu, *qWg, *qWd;     // query FFN (aliases the history FFN by default)
  const float *ln_g, *ln_b;         // d
  const float *Wq;                  // d x d
  const float *WkT;                 // h x d_h x d: WkT[j][c][k] = Wk[k][j*d_h + c]
  const float *Wv, *Wo;             // d x d
  const float *Wc;                  // (i+1)d x d, NULL for layer 0
};

// Per-layer weights of the per-target step, in the handle's element type
// (bf16 bits or fp32), laid out by step_weights_setup (target_step.cu).
struct LayerStep {
  const void *Wq;    // d x d
  const void *WkT;   // d_h x h d: WkT[c][j d + k] = W_K[k][j d_h + c]
  const void *Wv;    // d x d
  const void *Wo;    // d x d
  const void *Wc;    // (i+1) d x d, NULL for layer 0
  const void *Wug;   // d x 2rd: [query W_u | query W_g]
  const void *Wd;    // rd x d: query W_d
};

// Host fp32 weights of one layer handed to step_weights_setup.
struct StepHostW {
  const float *Wq, *Wk, *Wv, *Wo, *Wc, *qWu, *qWg, *qWd;
};

// One product of the tensor-core per-target step: MB blocks of 128 output
// features times KC chunks of 64 inputs, stored as A tiles tile0 ..
// tile0 + MB * KC - 1 (block-major) of the handle's step tile stream.
struct TcGemm {
  int mb = 0, kc = 0;
  int64_t tile0 = -1;
};

}  // namespace stca

struct stca_handle {
  int device = 0;
  int d = 0, h = 0, r = 0, M = 0, dtype = 0;
  int rd = 0, dh = 0;
  int elem = 4;                         // bytes per X / X~ element

  // weights
  float* w32 = nullptr;                 // fp32 slab
  void* wstep = nullptr;                // per-target step weights (dtype)
  std::vector<stca::LayerStep> Lstep;
  std::vector<stca::LayerW32> L32;
  const float* q_ln_g = nullptr;
  const float* q_ln_b = nullptr;
  uint16_t* wtc = nullptr;              // bf16 operands of the tensor-core encoder
  CUtensorMap tmW1, tmW2;               // their TMA descriptors
  CUtensorMap tmXt[16];                 // X~(i) of the last encode (tensor-core attention)
  CUtensorMap tmU;                      // bf16 query rows of the current forward
  CUtensorMap tmKn, tmVn;               // naive form: keys and values of the current layer
  int opt_attn_form = 0;                // 0 reordered (Eq. (13)), 1 naive (Eq. (12)), 2 auto
  bool last_naive = false;              // the last forward ran the naive form
  void* kv = nullptr;       size_t kv_cap = 0;     // naive form: N x 2d bf16, [K | V] per row
  void* wvt = nullptr;                  // per layer [W_V]^T (all heads), d x d bf16 (K-major), d = 128
  CUtensorMap tmWvT[16];                // their TMA descriptors (box 64 x 128)
  void* wkv = nullptr;                  // naive form: per layer [W_K | W_V]^T, 2d x d bf16 (K-major)
  CUtensorMap tmWkv[16];                // their TMA descriptors (box 64 inputs x 256 outputs)
  void* lt = nullptr;                   // cuBLASLt handle (naive-form projection)
  void* lt_ws = nullptr;    size_t lt_ws_cap = 0;  // its workspace
  void* bw_ws = nullptr;    size_t bw_ws_cap = 0;  // encoder backward workspace (fp32)
  void* bw_plan = nullptr;  size_t bw_plan_cap = 0;  // attention backward units and statistics
  bool tc_encode_ready = false;
  uint16_t* wstep_tc = nullptr;         // A-tile stream of the tensor-core per-target step
  std::vector<stca::TcGemm> tcO, tcC, tcUG, tcD, tcQ, tcK;   // per layer (tcK: d = 128, h <= 8)
  stca::TcGemm tcZC, tcZUG, tcZD;       // prediction head (Eq. (9)): W_Z, [zW_u | zW_g], zW_d
  bool head_tc = false;
  bool step_tc_ready = false;
  void* whead = nullptr;                // prediction-head weights (dtype): Wz, [zWu | zWg], zWd
  const void *hWz = nullptr, *hWug = nullptr, *hWd = nullptr;
  float* w32head = nullptr;             // the same in fp32, for the backward products:
  const float *hWz32 = nullptr, *hWu32 = nullptr, *hWg32 = nullptr, *hWd32 = nullptr;  // Wz, zWu, zWg, zWd
  int num_sms = 148;

  // options
  int opt_attn_path = 0, opt_encode_path = 0, opt_step_path = 0;
  int64_t opt_split_keys = 0;
  int opt_attn_kernel = 0;              // 0 auto (two-group kernel for d <= 128), 1 split-softmax kernel
  int opt_stop_tiles = 0;               // test hook: the attention loader stops after this many tiles
  int opt_bw_gemm = 0;                  // backward products of bf16 handles: 0 tensor cores (TF32), 1 cuBLASLt
  int opt_pipeline = 1;                 // 1: two-half pipeline where it applies (STCA_OPT_PIPELINE)
  int64_t launches = 0;
  bool timing = false;
  struct TimedRec { int cls; cudaEvent_t a, b; };
  std::vector<TimedRec> timed;          // events recorded around launches
  std::vector<cudaEvent_t> ev_pool;     // recycled events

  // encoded state
  bool encoded = false;
  int64_t R = 0, N = 0;
  std::vector<int64_t> offsets_h;
  void* xt = nullptr;                   // M x N x d, elem bytes each
  size_t xt_cap = 0;

  // forward workspace (device)
  float* q = nullptr;       size_t q_cap = 0;      // T x d
  float* U = nullptr;       size_t U_cap = 0;      // T x h x d (scaled)
  uint16_t* Ubf = nullptr;  size_t Ubf_cap = 0;    // bf16 copy for tensor cores
  float* part = nullptr;    size_t part_cap = 0;   // G x (d + 2)
  float* cbuf = nullptr;    size_t cbuf_cap = 0;   // T x h x d: merged alpha X~ rows
  int* attn_cnt = nullptr;  size_t attn_cnt_cap = 0;  // M x pairs x 8 arrival counters
  void* plan_d = nullptr;   size_t plan_cap = 0;   // uploaded plan arrays
  void* plan_h = nullptr;   size_t plan_h_cap = 0; // pinned staging
  cudaEvent_t plan_evt = nullptr;
  int* status_d = nullptr;

  // host-buffer entry point staging
  cudaStream_t copy_stream = nullptr;   // stca_run_host: the chunks' host-to-device copies
  std::vector<cudaEvent_t> chunk_evt;   // one per chunk: its copy has landed
  void* x_stage = nullptr;  size_t x_stage_cap = 0;
  void* t_stage = nullptr;  size_t t_stage_cap = 0;
  float* z_stage = nullptr; size_t z_stage_cap = 0;

  // last forward's plan (reused when the same targets layout repeats)
  std::vector<int64_t> last_toff;
  int last_path = 0;                    // 1 CUDA cores, 2 tensor cores
  int64_t last_G = 0, last_pairs = 0;
  int64_t last_npairs = 0;              // (request, query tile) pairs of the plan
  int last_max_items = 0;               // most items of one (request, query tile) pair
  int last_grid = 0;                    // CTAs of the tensor-core attention
  bool last_pipe = false;               // the plan is the two-half pipeline's
  bool last_pipe_asked = false;         // ... was asked for (part of the plan cache's key)
  int64_t pipe_RA = 0, pipe_TA = 0;     // its split: first request and first target of half B
  int pipe_gridA = 0, pipe_gridB = 0;   // its halves' attention CTAs (B's runs follow A's in cta_begin)
  size_t off_items = 0, off_pairs = 0, off_cta = 0, off_treq = 0, off_toff = 0, off_rpb = 0,
         off_pib = 0, off_qbase = 0;
  int64_t last_qrows = 0;               // naive form: rows of the packed query layout
};

namespace stca {

// ---------------------------------------------------------------- kernels
// CUDA-core kernels (simt_kernels.cu)
void launch_ffn_rows(const void* X, int x_is_bf16, int64_t nrows, const LayerW32& w,
                     bool history_ffn, const float* ln_g, const float* ln_b, void* Y,
                     int y_is_bf16, int d, int rd, cudaStream_t s);
void launch_attn_simt(const stca_handle* H, int layer, const void* xt_layer,
                      const AttnItem* items_d, const int32_t* pairs_d, int64_t npairs,
                      const int64_t* toff_d, cudaStream_t s);
struct StepPlan {
  const int32_t* treq;              // T: request of each target
  const int64_t* toff;              // R+1
  const int32_t* req_pair_begin;    // R+1: first (request, query tile) pair of r
  const int32_t* pair_item_begin;   // pairs+1: first item of each pair
  const AttnItem* items;
  int mtile_rows;                   // query rows per tile (1 << 30: one tile per request)
  int log2_partials;                // partial maxima are in log2 units
};
// Per-target step (target_step.cu)
void launch_combine(const stca_handle* H, const StepPlan& plan, const float* part, int64_t G,
                    int64_t T, float* out, cudaStream_t s);
// The same merge of d_h-wide partials already projected by W_V (the attention
// kernel's in-kernel projection): out = o_head, T x d.
void launch_combine_proj(const stca_handle* H, const StepPlan& plan, const float* part, int64_t G,
                         int64_t T, float* out, cudaStream_t s);
// Naive form: per-head outputs o_head (T x d fp32) from 64-wide partials.
void launch_combine_naive(const stca_handle* H, const StepPlan& plan, const float* part, int64_t G,
                          int64_t T, float* out, cudaStream_t s);
void launch_target_step(const stca_handle* H, int layer, const void* targets, int64_t T,
                        const StepPlan& plan, const float* cmerged, float* Z, cudaStream_t s);
size_t target_step_smem(const stca_handle* H);
int step_weights_setup(stca_handle* H, const std::vector<StepHostW>& layers);
// Prediction head of Eq. (9): host fp32 Wz ((M+1)d x d), zWu, zWg (d x rd), zWd (rd x d).
int head_weights_setup(stca_handle* H, const float* Wz, const float* zWu, const float* zWg,
                       const float* zWd);
void launch_head(const stca_handle* H, const void* targets, int64_t T, const float* Z, float* zout,
                 cudaStream_t s);
size_t attn_simt_smem(const stca_handle* H);
// Query rows per CTA of the CUDA-core attention for width d (its grid is
// (work item, first row) pairs, one per block of this many rows).
int attn_simt_rows_per_cta(int d);

// Tensor-core per-target step (step_tc.cu)
bool step_tc_supported(const stca_handle* H);
// head: fp32 host W_Z ((M+1)d x d), zW_u, zW_g (d x rd), zW_d (rd x d), or all NULL.
struct HeadHostW {
  const float *Wz = nullptr, *zWu = nullptr, *zWg = nullptr, *zWd = nullptr;
};
int step_tc_setup(stca_handle* H, const std::vector<StepHostW>& layers, const HeadHostW& head);
// cmerged: the merged rows c_j (T x h x d), or NULL to merge the split
// partials (part: G x d accumulators, then G maxima, G sums) inside the step;
// that needs at most step_tc_max_items() items per (request, query tile).
int step_tc_max_items();
int step_tc_max_items_proj();
// The prediction head of Eq. (9) alone on the tensor cores, from Z (T x M x d).
int launch_step_tc_head(const stca_handle* H, const void* targets, int64_t T, const float* Z, float* zout,
                        cudaStream_t s);
// Partials of the in-kernel projection kept per (query row, item of its pair)
// (at most kQslots items per pair): row q's item w at pacc[(q kQslots + w) d_h],
// its (m, l) at qml[(q kQslots + w) 2], the pair's item count at qn[q].  The
// per-target step then finds a row's partials without the work plan.
constexpr int kQslots = 8;
struct QslotBufs {
  const int32_t* pair_item_begin;
  float* pacc;
  float* qml;
  int* qn;
};
// Naive form of the step: `naive` not NULL; cmerged then holds o_head (T x d, the
// per-head outputs of Eq. (12)), and the query rows of the next layer are written
// into the packed layout (NaiveLayout) at naive->upk, request r from row qbase[r].
struct NaiveStep {
  int G, Tq;
  const int64_t* qbase;     // device, R + 1
  uint16_t* upk;            // device, [rows x 64] bf16
};
// proj: the attention already projected its rows by W_V (d_h-wide partials of
// o_j): 1 cmerged holds the merged o_head (T x d); 2 cmerged is NULL and the
// step merges the partials (part) itself, at most step_tc_max_items_proj()
// items per query row.  defer_wait (query init only, layer < 0): the launch
// directly follows this library's encoder launch on the stream, with nothing
// in between, so the kernel waits for it at its end rather than its start.
int launch_step_tc(const stca_handle* H, int layer, const void* targets, int64_t T,
                   const float* cmerged, const StepPlan* plan, const float* part, int64_t G,
                   float* Z, uint16_t* Ubf, cudaStream_t s, const NaiveStep* naive = nullptr,
                   float* zout = nullptr, int proj = 0, const QslotBufs* qs = nullptr,
                   bool defer_wait = false);

// One phase of the two-half pipeline (stca_forward at d = 128 with the
// in-kernel projection): one launch runs the per-target step of one half of
// the batch (layer, its targets, Z and U rows, the row slots of its query
// rows; T = 0: none) beside the attention of the other half (its plan's
// items and CTA runs; grid = 0: none).
struct PipeStep {
  int layer;
  const void* targets;
  int64_t T;
  float* Z;
  uint16_t* Ubf;
  QslotBufs qs;
};
struct PipeAttn {
  int layer;
  const AttnItem* items;
  const int32_t* cta_begin;
  int grid;
  QslotBufs qs;
};
int launch_step_attn_pipe(const stca_handle* H, const PipeStep& st, const PipeAttn& at, cudaStream_t s);

// Host-side attention work plan (stca_api.cu).
struct PlanHost {
  std::vector<AttnItem> items;
  std::vector<int32_t> pairs_simt;       // (item, first query row) pairs, CUDA-core grid
  std::vector<int32_t> cta_begin;        // tensor-core grid + 1
  std::vector<int32_t> req_pair_begin;   // R + 1
  std::vector<int32_t> pair_item_begin;  // pairs + 1
  std::vector<int64_t> qbase;            // naive form (path 3): first query row of each request
  int64_t qrows = 0;                     // naive form: query rows of the padded layout
  int64_t G = 0;                         // partial rows
  int grid = 0;                          // tensor-core CTAs
};
void build_plan_host(const int64_t* off, const int64_t* toff, int64_t R, int h, int path,
                     int num_ctas, int64_t split_keys, PlanHost& P, int dh = 0, int simt_rows = 1);
NaiveLayout naive_layout(int dh);
int check_plan(const PlanHost& P, const int64_t* off, const int64_t* toff, int64_t R, int h,
               int path);
void launch_target_step_ws(const stca_handle* H, int layer, const void* targets, int64_t T,
                           const float* cmerged, float* Z, uint16_t* Ubf, cudaStream_t s);
int launch_attn_tc_ws(int d, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                      const AttnItem* items_d, const int32_t* cta_begin_d, int grid, float* part,
                      int64_t G, int* status, cudaStream_t s);

// Two-group tensor-core attention with the split combine inside (attn_pp.cu):
// writes the merged rows c (T h x d fp32) to `cout`; part holds G x d partial
// rows then G x 4 (m, l) values; counters (pairs x 8 ints) must be zero.
// stats, when not NULL: T h x 2 floats, each row's softmax maximum (log2 units
// of the bf16 query rows' scores) and sum.
bool attn_pp_supported(int d);
int launch_attn_pp(int d, const CUtensorMap& tmQ, const CUtensorMap& tmK, const AttnItem* items_d,
                   const int32_t* cta_begin_d, const int32_t* pair_item_begin_d, int grid,
                   float* part, int64_t G, float* cout, int* counters, int* status, int stop_tiles,
                   cudaStream_t s, float* stats = nullptr);

// Naive form's K/V projection on the tensor cores (kv_proj.cu): out (N x 2d
// bf16) = X~ (tmX: N x d, box 64 x 128) times [W_K | W_V] (tmW: its transpose,
// 2d x d, box 64 x 256).
bool kv_proj_supported(int d);
int launch_kv_proj(int d, const CUtensorMap& tmX, const CUtensorMap& tmW, uint16_t* out, int64_t N,
                   int num_sms, int* status, cudaStream_t s);

// Attention backward on the tensor cores (attn_bw_tc.cu), d in {64, 128}.
bool attn_bw_tc_supported(int d);
void launch_bw_prep(const float* U, const float* dC, uint16_t* Ub, uint16_t* dCb, int64_t n, cudaStream_t s);
void launch_bw_delta(const float* dC, const float* c, float* delta, int64_t rows, int d, cudaStream_t s);
int launch_attn_bw_tc(int d, const CUtensorMap& tmQ, const CUtensorMap& tmC, const CUtensorMap& tmK,
                      const AttnItem* items, const int32_t* cta_begin, const int32_t* pair_item_begin,
                      const int32_t* req_pair_begin, int grid, const float* stats, const float* delta,
                      float* dU, float* dX, int* status, int stop_tiles, cudaStream_t s);

// Tensor-core attention (attn_tc.cu)
bool attn_tc_supported(int d);
// proj: the kernel also projects each item's rows by W_V (d = 128; [W_V]^T
// of the layer from H->tmWvT) and writes d_h-wide partials of o_j.
bool attn_tc_proj_supported(const stca_handle* H);
int launch_attn_tc(stca_handle* H, int layer, const AttnItem* items_d, const int32_t* cta_begin_d,
                   int grid, cudaStream_t s, bool proj = false, const QslotBufs* qs = nullptr);
int launch_attn_tc_naive(stca_handle* H, const AttnItem* items_d, const int32_t* cta_begin_d,
                         int grid, cudaStream_t s);

// Tensor-core encoder (encode_tc.cu)
bool encode_tc_supported(int d, int rd);
int encode_tc_setup(stca_handle* H, const std::vector<const float*>& Wu,
                    const std::vector<const float*>& Wg, const std::vector<const float*>& Wd);
// Encodes the N rows at X into rows row0 .. row0 + N - 1 of every layer's X~
// (H->N rows per layer).
int launch_encode_tc(stca_handle* H, const void* X, int64_t N, cudaStream_t s, int64_t row0 = 0);
int make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                      uint32_t box_inner, uint32_t box_outer);
// fp32 tensor map of three dimensions (innermost first; strides of the outer
// two in bytes, multiples of 16), 128-byte swizzle.
int make_tmap_f32_3d(CUtensorMap* m, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                     const uint32_t box[3]);
// Hand-written tensor-core GEMM with TF32 operands (gemm_tc.cu), row-major:
// C (m x n) = alpha op(A) op(B) + beta C, ta / tb: A / B stored transposed;
// `batch` products with operand strides sA, sB, sC (elements).  Returns
// STCA_EINVAL without launching when the operands' alignment does not allow
// TMA (addresses and row strides multiples of 16 bytes).
int tc_gemm_tf32(bool ta, bool tb, int64_t m, int64_t n, int64_t k, const float* A, int64_t lda,
                 const float* B, int64_t ldb, float* C, int64_t ldc, float beta, float alpha, int batch,
                 int64_t sA, int64_t sB, int64_t sC, int num_sms, int* status, cudaStream_t s);
// The same GEMM with bf16 operands (any layout), fp32 C; epi 0 stores C,
// epi 1 (SwiGLU forward: the weight's 128-row tiles interleave 64 up and 64
// gate rows) writes A16, G16 (row stride ld16) and H16 = A SiLU(G) (row
// stride ldh), all bf16, at hidden columns 64 tn; epi 2 (SwiGLU backward:
// acc = dH) reads A16 and G16 and overwrites them with dA and dG.
int tc_gemm_bf16(bool ta, bool tb, int64_t m, int64_t n, int64_t k, const uint16_t* A, int64_t lda,
                 const uint16_t* B, int64_t ldb, float* C, int64_t ldc, float beta, int epi, uint16_t* A16,
                 uint16_t* G16, uint16_t* H16, int64_t ld16, int64_t ldh, int num_sms, int* status,
                 cudaStream_t s);
// The same with rows `row_bytes` apart (a multiple of 16).
int make_tmap_bf16_2d_strided(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

}  // namespace stca
