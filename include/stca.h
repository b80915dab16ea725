/*
 * stca.h -- C ABI of the STCA library (libstca.so, sm_100a).
 *
 * Stacked Target Cross Attention over jagged user histories with
 * request-level batching.  Sources:
 *   [digest] "Make It Long, Keep It Fast: End-to-End 10k-Sequence Modeling at
 *            Billion Scale on Douyin" (paper digest), §2.1 Eqs. (1)-(9), (12),
 *            (13); §2.2 (request-level batching); §2.3 (ragged target
 *            attention; the sparse-training batch builder, Eqs. (15)-(17)).
 *   [blog]   "字节跳动-STCA：抖音 10k 长序列端到端建模的架构、系统与外推三件套"
 *            (STCA blog), §2.2-§2.6.
 *
 * Beyond the forward below: the Eq. (9) prediction-head token (stca_head,
 * stca_forward_head), the naive Eq. (12) form as an option (STCA_OPT_ATTN_FORM),
 * the sparse-training batch builder (stca_sl_*), and the backward of every
 * piece of the step under a given output gradient (stca_*_backward).
 *
 * What the calls compute.  For request r with history X_r (L_r x d, the rows
 * offsets[r] .. offsets[r+1]-1 of X) and targets x_t (rows target_offsets[r]
 * .. target_offsets[r+1]-1 of `targets`), for every layer i = 1..M:
 *   X~(i)   = LN_i(SwiGLUFFN_i(X_r))                        [digest] Eq. (2)
 *   q(1)    = LN_q(SwiGLUFFN_q1(x_t))                        Eq. (3)
 *   u_j     = (q(i) W_Q^(i,j)) W_K^(i,j)^T,  head j          Eq. (13)
 *   alpha_j = softmax(u_j X~(i)^T / sqrt(d_h)) over the L_r history rows
 *   o(i)    = [ (alpha_1 X~(i)) W_V^(i,1) || ... || (alpha_h X~(i)) W_V^(i,h) ] W_O^(i)
 *                                                            Eqs. (6), (13)
 *   q(i+1)  = SwiGLUFFN_q(i+1)([o(1) || ... || o(i) || x_t] W_C^(i+1))   Eq. (7)
 * and writes Z[t, i, :] = o(i) for every target t (Eq. (8)).
 *   SwiGLUFFN(x) = ((x W_u) * SiLU(x W_g)) W_d, no biases (Eq. (1) read with the
 *   blog's shapes: W_u, W_g d x rd, W_d rd x d).  LN: eps 1e-5, biased variance,
 *   affine (gamma, beta).  Head j owns columns [j d_h, (j+1) d_h) of W_Q, W_K, W_V.
 *   The history encodings X~(i) read the raw X for every i; they are not chained.
 *
 * Conventions.  Row-major everywhere, x * W (row vector times matrix).
 * Element type of X, targets and all weights: the handle's dtype (STCA_F32:
 * IEEE fp32; STCA_BF16: bfloat16 bit patterns, uint16).  Z is always fp32.
 * Return value: STCA_OK (0) or a negative STCA_E* code; stca_last_error()
 * gives a message (thread-local).  No call aborts the process.
 *
 * Threading and streams.  A handle is used by one host thread at a time and
 * orders its work on the stream passed to each call (NULL = the legacy
 * default stream).  Separate handles are independent.
 */
#ifndef STCA_H_
#define STCA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct stca_handle stca_handle;

typedef enum { STCA_F32 = 0, STCA_BF16 = 1 } stca_dtype;

enum {
  STCA_OK = 0,
  STCA_EINVAL = -1,      /* bad argument: shape, dtype, pointer, offsets       */
  STCA_ESTATE = -2,      /* call out of order, e.g. forward before encode      */
  STCA_ENOMEM = -3,      /* device or pinned host allocation failed            */
  STCA_ECUDA = -4,       /* a CUDA runtime or driver call failed               */
  STCA_EDEVICE = -5      /* a kernel reported a failure (bounded wait ran out) */
};

/*
 * Weights of all M layers.  Each field is a host array of M pointers, entry i
 * belonging to layer i+1.  Pointers are host pointers unless stca_init's
 * weights_on_device is nonzero; each points to dtype elements, row-major.
 *   Wu[i], Wg[i]  d x rd       SwiGLU up and gate projections   Eq. (1)-(2)
 *   Wd[i]         rd x d       SwiGLU down projection
 *   ln_gamma[i], ln_beta[i]  d LayerNorm affine of layer i's history encoding;
 *                 the field itself may be NULL: gamma = 1, beta = 0
 *   Wq[i], Wk[i], Wv[i], Wo[i]  d x d   attention projections   Eqs. (4)-(6)
 *   Wc[i]         (i+1)d x d   query fusion of layer i+1 (Eq. (7)); Wc[0] is
 *                 ignored and may be NULL; the field may be NULL when M == 1
 *   qWu, qWg, qWd optional query-side SwiGLU of each layer (Eqs. (3), (7));
 *                 NULL field: the query uses the history FFN of that layer
 *   q_ln_gamma, q_ln_beta  optional single pointers (d elements): the LN of
 *                 Eq. (3); NULL: layer 1's ln_gamma / ln_beta
 *   Wz, zWu, zWg, zWd  optional single pointers: the prediction-head token of
 *                 Eq. (9) ("Make It Long, Keep It Fast" digest, §2.1, Eq. (9)),
 *                 z = SwiGLUFFN([o(1) || ... || o(M) || x_t] W_Z), with
 *                 Wz (M+1)d x d, zWu and zWg d x rd, zWd rd x d.  The head's
 *                 SwiGLU has weights of its own and no LayerNorm (the pages
 *                 name no norm there).  All four NULL: stca_head is rejected;
 *                 some NULL: stca_init fails with STCA_EINVAL.
 * stca_init copies everything; the caller may free its buffers afterwards.
 */
typedef struct {
  const void* const* Wu;
  const void* const* Wg;
  const void* const* Wd;
  const void* const* ln_gamma;
  const void* const* ln_beta;
  const void* const* Wq;
  const void* const* Wk;
  const void* const* Wv;
  const void* const* Wo;
  const void* const* Wc;
  const void* const* qWu;
  const void* const* qWg;
  const void* const* qWd;
  const void* q_ln_gamma;
  const void* q_ln_beta;
  const void* Wz;
  const void* zWu;
  const void* zWg;
  const void* zWd;
} stca_weights;

/*
 * Create a handle on the current CUDA device and copy the weights into it.
 * d: model width; h: heads (d % h == 0); r: SwiGLU expansion (hidden rd = r*d);
 * M: stacked layers (1..16); dtype: STCA_F32 or STCA_BF16.
 * Supported sizes: d in [8, 1024] with d % 8 == 0, rd <= 4096.  The bf16
 * tensor-core kernels additionally need d in {64, 128, 256} and rd % 64 == 0;
 * other bf16 sizes run on the CUDA-core kernels.
 * On success *out owns device memory until stca_destroy.
 * Errors: STCA_EINVAL (sizes, NULL required field), STCA_ENOMEM, STCA_ECUDA.
 */
int stca_init(const stca_weights* w, int d, int h, int r, int M, int dtype,
              int weights_on_device, stca_handle** out);

/* Release everything the handle owns.  NULL is accepted. */
void stca_destroy(stca_handle* handle);

/*
 * Encode a jagged batch of histories: computes X~(i) for i = 1..M (Eq. (2))
 * into buffers the handle owns; they stay valid until the next stca_encode
 * or stca_destroy, so any number of stca_forward calls can reuse them
 * (request-level batching: one history, many targets).
 *   X        device pointer, N x d dtype elements, requests concatenated
 *   offsets  HOST pointer, R+1 int64: offsets[0] == 0, offsets[R] == N,
 *            offsets[r+1] - offsets[r] = L_r >= 1 (an empty history has no
 *            softmax and is rejected)
 *   R >= 1 requests, N rows in total.  stream: a cudaStream_t or NULL.
 * Asynchronous with respect to the host, except that a first call or a larger
 * batch than before allocates device memory.
 * Errors: STCA_EINVAL (offsets not monotone, L_r == 0, sizes), STCA_ENOMEM,
 * STCA_ECUDA.
 */
int stca_encode(stca_handle* handle, const void* X, const int64_t* offsets,
                int64_t R, int64_t N, void* stream);

/*
 * Run the stacked target attention for the targets of the encoded requests.
 *   targets         device pointer, T x d dtype elements, grouped by request
 *   target_offsets  HOST pointer, R+1 int64 with the R of the last encode:
 *                   targets of request r are rows target_offsets[r] ..
 *                   target_offsets[r+1]-1; T_r = 0 is allowed
 *   T               total targets (target_offsets[R]); T == 0 is a no-op
 *   Z               device pointer, caller-owned, T x M x d fp32; row t holds
 *                   [o(1); ...; o(M)] of target t (Eq. (8))
 * The attention's work plan depends on the key layout (the offsets of the last
 * encode), the target offsets and the options.  When one of them changed
 * since the last forward, the call builds the plan on the host and uploads it
 * on the stream (through a pinned buffer; the host first waits until the
 * previous upload has left it); otherwise the plan already on the device
 * serves, even across encodes of a batch with the same offsets.
 * Errors: STCA_ESTATE (no encode yet), STCA_EINVAL, STCA_ENOMEM, STCA_ECUDA.
 */
int stca_forward(stca_handle* handle, const void* targets, const int64_t* target_offsets,
                 int64_t T, float* Z, void* stream);

/*
 * stca_encode followed by stca_forward on the same stream, in one call: the
 * serving step of request-level batching ("Make It Long, Keep It Fast"
 * digest, §2.2: encode each request's history once, then attend to it for all
 * of its targets; Eqs. (2)-(8)).  Arguments, results and errors are those of
 * the two calls: X, offsets, R, N as for stca_encode; targets,
 * target_offsets, T, Z as for stca_forward (T == 0 encodes only).  The
 * encoded histories stay valid for later stca_forward calls.
 * Because nothing can be enqueued between the two parts, the first per-target
 * launch of the two-half pipeline (the query initialisation of the first
 * half, which reads only the targets and the weights) may start on the SMs
 * that the encoder's last round of tiles leaves idle, before the encoder has
 * finished.  The targets must therefore be complete before the call's work
 * starts on the stream, as for stca_encode's X.  Same Z as the two calls.
 */
int stca_encode_forward(stca_handle* handle, const void* X, const int64_t* offsets, int64_t R,
                        int64_t N, const void* targets, const int64_t* target_offsets, int64_t T,
                        float* Z, void* stream);

/*
 * Prediction-head token of Eq. (9) ("Make It Long, Keep It Fast" digest,
 * §2.1, Eq. (9)) for T targets:
 *   zout[t] = SwiGLUFFN_z([Z[t, 0, :] || ... || Z[t, M-1, :] || x_t] W_Z)
 * where SwiGLUFFN_z(v) = ((v zWu) * SiLU(v zWg)) zWd with the head weights
 * given to stca_init.
 *   targets  device pointer, T x d dtype elements (x_t, the rows given to
 *            stca_forward)
 *   Z        device pointer, T x M x d fp32: the output of stca_forward
 *   zout     device pointer, caller-owned, T x d fp32
 *   T >= 0 (0 is a no-op).  Needs no stca_encode; asynchronous on `stream`.
 * Errors: STCA_EINVAL (NULL pointer, T < 0, no head weights in the handle),
 * STCA_ECUDA.
 */
int stca_head(stca_handle* handle, const void* targets, int64_t T, const float* Z,
              float* zout, void* stream);

/*
 * stca_forward followed by the prediction-head token of Eq. (9): writes Z as
 * stca_forward does and zout (T x d fp32, caller-owned, 16-byte aligned) as
 * stca_head would.  On the tensor-core step path the head runs inside the last
 * layer's step launch (its [o(1) .. o(M) | x_t] operand is already on chip);
 * elsewhere the head kernel runs after the forward.  Same errors as
 * stca_forward, plus STCA_EINVAL when the handle has no head weights.
 */
int stca_forward_head(stca_handle* handle, const void* targets, const int64_t* target_offsets,
                      int64_t T, float* Z, float* zout, void* stream);

/*
 * Copy the encoded history X~(layer+1) of the last stca_encode (N x d, dtype
 * elements, the rows in the order of X) into `dst`, a device buffer the caller
 * owns.  layer is 0-based.  Lets a caller keep or inspect the encoding of a
 * request batch.  Errors: STCA_ESTATE (no encode yet), STCA_EINVAL, STCA_ECUDA.
 */
int stca_get_encoded(stca_handle* handle, int layer, void* dst, void* stream);

/*
 * stca_forward without device allocation.  (An addition of this library: the
 * STCA pages have no counterpart; it changes where the workspace lives, not
 * what is computed.)  Same arguments, result and errors as stca_forward, for
 * bf16 handles with d in {64, 128, 256} (the tensor-core path); other handles
 * get STCA_EINVAL.  For callers that cannot call cudaMalloc after start-up --
 * their device memory belongs to another allocator's pool, their memory budget
 * is fixed, or they cannot afford the synchronisation cudaMalloc / cudaFree
 * may imply -- the query rows, split partials and work plan of the call live in
 * a 32 MiB file-scope device array built into the library: every GPU that
 * loads the library holds it until the process exits.  A batch whose
 * workspace does not fit returns STCA_EINVAL with the size it needs.  All
 * calls on a device share the array: calls whose work overlaps on the GPU
 * (other streams, other handles) race, so keep them on one stream.  The first
 * call on a device looks up the array's address (cudaGetSymbolAddress).  A
 * call uploads its work plan from host memory every time, so it cannot be
 * captured into a CUDA graph: under an active capture it returns STCA_EINVAL.
 * Nothing a call reads is left over from an earlier call.  It always runs the
 * reordered form of Eq. (13): STCA_OPT_ATTN_FORM 1 (the naive form) is
 * rejected with STCA_EINVAL, and 2 runs the reordered form.  The per-target
 * step follows STCA_OPT_STEP_PATH as in stca_forward (tensor cores where the
 * handle has them).  stca_init and stca_encode still allocate as documented.
 */
int stca_forward_static(stca_handle* handle, const void* targets,
                        const int64_t* target_offsets, int64_t T, float* Z, void* stream);

/*
 * End-to-end call on HOST buffers: copies X and targets from host memory to
 * device staging buffers the handle owns, encodes, runs the forward, copies
 * Z (T x M x d fp32) back to host memory and waits for the stream.  With the
 * tensor-core encoder and at least 65536 history rows, X is copied in 8 chunks
 * of whole 128-row tiles on a second stream the handle owns, and each chunk is
 * encoded as soon as its copy has landed, so encoding overlaps the copy of the
 * later chunks.  Host buffers should be page-locked for the copies to overlap;
 * pageable memory works but is slower.  Same argument rules as stca_encode and
 * stca_forward.
 */
int stca_run_host(stca_handle* handle, const void* X_host, const int64_t* offsets,
                  int64_t R, int64_t N, const void* targets_host,
                  const int64_t* target_offsets, int64_t T, float* Z_host, void* stream);

/*
 * Check offsets on the host without touching a device: offsets[0] == 0,
 * non-decreasing, offsets[R] == total; with require_nonempty, every segment
 * has at least one row.  Returns STCA_OK or STCA_EINVAL.
 */
int stca_validate_offsets(const int64_t* offsets, int64_t R, int64_t total,
                          int require_nonempty);

/*
 * Host only, no device needed: the attention work split the library uses for a
 * batch (the same planner stca_forward runs).  path 1: CUDA-core kernel, items
 * are key ranges of at most split_keys keys over all T_r * h query rows (by
 * default 1024, or down to 128 when a batch has fewer than 2 num_ctas
 * (range, target) pairs of 1024 keys).  path 2: tensor-core kernel, (request, 128-row query tile) pairs
 * cut into num_ctas runs of equal numbers of 128-key tiles (capped at
 * split_keys / 128 tiles when split_keys > 0), one run per CTA; each maximal
 * run inside a pair is an item.  Outputs: *n_items, *grid (CTAs, path 2),
 * *partial_rows; when `items` is not NULL, 7 int64 per item (request, query
 * tile, first key row, keys, first query row, query rows, first partial row);
 * when `cta_begin` is not NULL (path 2), grid + 1 item indices.  The plan is
 * checked against the invariants the kernels rely on; a violation returns
 * STCA_EINVAL.  Offsets follow stca_encode / stca_forward.
 */
int stca_plan_attention(const int64_t* offsets, const int64_t* target_offsets, int64_t R,
                        int h, int path, int num_ctas, int64_t split_keys, int64_t* n_items,
                        int64_t* grid, int64_t* partial_rows, int64_t* items, int64_t items_cap,
                        int32_t* cta_begin, int64_t cta_cap);

/*
 * Wait for the handle's work on `stream` and read its device status word.
 * STCA_OK, or STCA_EDEVICE if a kernel gave up a bounded wait (the message
 * names the kernel), or STCA_ECUDA.  The status is cleared by the read.
 */
int stca_device_status(stca_handle* handle, void* stream);

/* ------------------------------------------------------------------------
 * Sparse-training batch builder ("Make It Long, Keep It Fast" digest, §2.3
 * "Extrapolation: Train Sparsely, Infer Densely"; STCA blog, §2.6): per-user
 * training lengths from the stochastic length curriculum, the temporal-suffix
 * selection, and the two-step batch-level load balance, producing the packed,
 * padding-free history stream and offsets that stca_encode takes.  Random
 * numbers are the caller's: it draws s_b ~ Beta(alpha, beta).
 * ------------------------------------------------------------------------ */

/*
 * Eq. (17): *beta = alpha (L_max - L_avg) / (L_avg - L_min), the Beta shape
 * that makes the mean of Eq. (16)'s L_raw equal L_avg; Eq. (15): *ss (may be
 * NULL) = L_avg / L_max, the sequence sparsity.  Host only.
 * Errors: STCA_EINVAL unless alpha > 0 and 0 <= L_min < L_avg < L_max.
 */
int stca_sl_beta(double alpha, int64_t L_min, int64_t L_max, int64_t L_avg, double* beta,
                 double* ss);

/*
 * Host only: the packed layout of one training batch of B users.
 *   hist_offsets  B+1 int64: user b's full history is rows hist_offsets[b] ..
 *                 hist_offsets[b+1]-1 of X, oldest first; every user has >= 1 row
 *   s             B doubles in [0, 1]: the user's Beta draw
 *   L_min, L_max, L_avg   0 <= L_min < L_avg < L_max; L_infer >= 1
 * For each user: L_raw = L_min + s (L_max - L_min) (Eq. (16), in double, in
 * that order), aligned down to a multiple of 8 (at least 8), capped by the
 * usable history min(H_b, L_infer).  Then the batch is brought to exactly
 * B * L_avg rows: a surplus is removed by keeping one row per user and sharing
 * the other B * L_avg - B rows in proportion to (length - 1), a shortfall is
 * filled in proportion to each user's unused usable history, both by the
 * largest-remainder method (ties to the lower user index); when the usable
 * histories hold fewer rows than the budget, every user takes all of its own.
 * Outputs (caller-owned host arrays): train[B] (the aligned Eq. (16) lengths,
 * may be NULL), lengths[B] (final, each >= 1), packed_offsets[B+1] (prefix
 * sums of lengths) and src_start[B] = hist_offsets[b+1] - lengths[b] (the
 * first row of the user's temporal suffix).  Deterministic: the same inputs
 * give the same integers on every machine.
 * Errors: STCA_EINVAL (bad offsets, empty history, s outside [0, 1] or not
 * finite, bad lengths, B < 1, NULL output).
 */
int stca_sl_plan(const int64_t* hist_offsets, int64_t B, const double* s, int64_t L_min,
                 int64_t L_max, int64_t L_avg, int64_t L_infer, int64_t* train, int64_t* lengths,
                 int64_t* packed_offsets, int64_t* src_start);

/*
 * Device gather of the packed stream: for user b and 0 <= k < packed_offsets[b+1]
 * - packed_offsets[b], row packed_offsets[b] + k of X_packed is row
 * src_start[b] + k of X, copied bit for bit, and seg[packed_offsets[b] + k] = b
 * (the index tensor of the ragged attention; seg may be NULL).
 *   X          device, N rows of row_bytes bytes (row_bytes a multiple of 16,
 *              X and X_packed 16-byte aligned)
 *   src_start, packed_offsets   DEVICE int64 arrays of B and B+1 entries, as
 *              stca_sl_plan writes them (caller-owned; the library does not check
 *              them on the device: every source row must lie in [0, N))
 *   P          packed rows, packed_offsets[B]
 *   X_packed   device, P rows of row_bytes (caller-owned); seg: device int32 P
 * Asynchronous on `stream`.  Errors: STCA_EINVAL (sizes, alignment, NULL),
 * STCA_ECUDA.
 */
int stca_sl_gather(const void* X, int64_t N, int64_t row_bytes, const int64_t* src_start,
                   const int64_t* packed_offsets, int64_t B, int64_t P, void* X_packed,
                   int32_t* seg, void* stream);

/* ------------------------------------------------------------------------
 * Backward pass of two pieces of the forward, under a loss whose gradient is
 * given ("Make It Long, Keep It Fast" digest §2.1, Eqs. (1)-(2) and (13);
 * request-level batching sums a history's gradient over all its targets).
 * All gradients are fp32 device buffers the caller owns; they are overwritten.
 * ------------------------------------------------------------------------ */

/*
 * History encoding of layer `layer` (0-based): X~ = LN(((X W_u) * SiLU(X W_g)) W_d).
 * Given dXt (N x d fp32, the gradient of X~), writes dX (N x d; may be NULL),
 * dWu, dWg (d x rd), dWd (rd x d), dgamma, dbeta (d), for the handle's weights
 * of that layer.  X: device, N x d in the handle's dtype (the rows given to
 * stca_encode, or any others).  The products run on cuBLASLt in fp32 (TF32
 * tensor cores for bf16 handles); the workspace (about N (2d + 3 rd) floats)
 * is the handle's.  Errors: STCA_EINVAL, STCA_ENOMEM, STCA_ECUDA.
 */
int stca_encode_backward(stca_handle* handle, int layer, const void* X, int64_t N,
                         const float* dXt, float* dX, float* dWu, float* dWg, float* dWd,
                         float* dgamma, float* dbeta, void* stream);

/*
 * Single-query attention of layer `layer` on merged rows (Eq. (13)): for each
 * request r and each of its T_r h query rows u (row t h + j of U: target t,
 * head j, scale included, u = (q W_Q^j) W_K^j^T / sqrt(d_h)),
 * c = softmax(u X~_r^T) X~_r with X~ the last stca_encode's encoding of that
 * layer.  Given dC (T h x d fp32, the gradient of c), writes dU (T h x d) and
 * dXt (N x d: every history row; rows of requests without targets get 0).
 * target_offsets: HOST, R+1 int64 as for stca_forward.  Needs d in {64, 128,
 * 256}.  Synchronises `stream` once to upload its work list.
 * Errors: STCA_ESTATE (no encode yet), STCA_EINVAL, STCA_ENOMEM, STCA_ECUDA.
 */
int stca_attention_backward(stca_handle* handle, int layer, const float* U,
                            const int64_t* target_offsets, int64_t T, const float* dC,
                            float* dU, float* dXt, void* stream);

/*
 * Output side of attention layer `layer` (digest Eqs. (6) and (13)): with the
 * merged rows C (T h x d fp32: row t h + j holds c_j = alpha_j X~ of target t,
 * head j), the layer output is o = [c_1 W_V^1 || ... || c_h W_V^h] W_O, head j
 * on columns [j d_h, (j+1) d_h) of W_V.  Given dZ (T x d fp32, the gradient of
 * o), writes dC (T h x d: the dC that stca_attention_backward takes), dWv and
 * dWo (d x d, row-major like the weights).  All pointers are DEVICE memory the
 * caller owns; W_V and W_O are the handle's.  T = 0 writes zero weight
 * gradients.  Errors: STCA_EINVAL, STCA_ENOMEM, STCA_ECUDA.
 */
int stca_output_backward(stca_handle* handle, int layer, const float* C, int64_t T,
                         const float* dZ, float* dC, float* dWv, float* dWo, void* stream);

/*
 * Query side of attention layer `layer` (digest Eq. (13)): the merged rows are
 * u_j = (q W_Q^j) W_K^j^T / sqrt(d_h) for each target's query vector q.
 * Given Q (T x d fp32, the layer's q as the forward formed it) and dU
 * (T h x d fp32, row t h + j; the dU stca_attention_backward returns), writes
 * dQ (T x d), dWq and dWk (d x d).  DEVICE pointers the caller owns; W_Q and
 * W_K are the handle's.  T = 0 writes zero weight gradients.
 * Errors: STCA_EINVAL, STCA_ENOMEM, STCA_ECUDA.
 */
int stca_query_backward(stca_handle* handle, int layer, const float* Q, int64_t T,
                        const float* dU, float* dQ, float* dWq, float* dWk, void* stream);

/*
 * Query init (digest Eq. (3)): q^(1) = LN(SwiGLUFFN(x_t)) with the query FFN and
 * query LayerNorm weights (layer 1's unless given separately).  Given the
 * targets x_t (DEVICE, T x d, handle dtype) and dq (T x d fp32, the gradient of
 * q^(1)), writes dxt (T x d fp32; may be NULL), dWu, dWg (d x rd), dWd (rd x d),
 * dgamma, dbeta (d), all DEVICE, caller-owned.  Recomputes the forward in fp32.
 * Errors: STCA_EINVAL, STCA_ENOMEM, STCA_ECUDA.
 */
int stca_query_init_backward(stca_handle* handle, const void* targets, int64_t T, const float* dq,
                             float* dxt, float* dWu, float* dWg, float* dWd, float* dgamma,
                             float* dbeta, void* stream);

/*
 * A fusion block: y = SwiGLUFFN([o^(1) || ... || o^(b) || x_t] W), x_t last.
 *   block b in [1, M-1]: Eq. (7), the next query q^(b+1), with W = W_C of layer
 *     b+1 ((b+1) d x d) and that layer's query FFN;
 *   block b = M: Eq. (9), the prediction-head token z, with W = W_Z
 *     ((M+1) d x d) and the head's FFN (needs the head weights at stca_init).
 * Z: (T, M, d) fp32 as stca_forward writes it; only o^(1..b), the first b d
 * columns of each row, are read.  targets: T x d, handle dtype.  dy: T x d
 * fp32, the gradient of y.  Writes dZ's first b d columns of each row (row
 * stride M d; the other columns are not touched) and dxt (T x d), overwriting
 * them, or adding to them when `accumulate` is nonzero (o^(1) and x_t feed
 * several blocks).  Writes dW ((b+1) d x d), dWu, dWg (d x rd), dWd (rd x d).
 * All DEVICE pointers, caller-owned.  T = 0 writes zero weight gradients.
 * Errors: STCA_EINVAL (bad block, no head weights for block M), STCA_ENOMEM,
 * STCA_ECUDA.
 */
int stca_fusion_backward(stca_handle* handle, int block, const float* Z, const void* targets,
                         int64_t T, const float* dy, int accumulate, float* dZ, float* dxt,
                         float* dW, float* dWu, float* dWg, float* dWd, void* stream);

/* Tunables and introspection (STCA_OPT_*).  Values are validated. */
enum {
  STCA_OPT_ATTN_PATH = 1,     /* 0 auto, 1 CUDA cores, 2 tensor cores (bf16 only) */
  STCA_OPT_ENCODE_PATH = 2,   /* 0 auto, 1 CUDA cores, 2 tensor cores (bf16 only) */
  STCA_OPT_SPLIT_KEYS = 3,    /* keys per attention work item, 0 = auto; multiple of 128 */
  STCA_OPT_TIMING = 4,        /* 1: record CUDA events around every kernel launch */
  STCA_OPT_STEP_PATH = 5,     /* per-target step: 0 auto, 1 CUDA cores, 2 tensor cores (bf16,
                                 d in {128, 256}, r d <= 512, with the tensor-core attention) */
  STCA_OPT_ATTN_FORM = 6,     /* 0: the reordered single-query form of Eq. (13) (default);
                                 1: the naive form of Eq. (12) -- K = X~ W_K and V = X~ W_V
                                 projected once per layer for all targets, then attention per
                                 head over d_h features (the pages' K/V-cache serving idea);
                                 2: whichever of the two has fewer FLOPs for the batch.
                                 The naive form needs the tensor-core step (see above) and
                                 d_h in {16, 32, 64}; form 1 without them is rejected, form 2
                                 falls back to the reordered form */
  STCA_OPT_ATTN_KERNEL = 7,   /* tensor-core attention of the reordered form: 0 auto (the
                                 split-softmax kernel, with its query tile in TMEM for
                                 d <= 128); 1 the split-softmax kernel; both are followed by
                                 the split combine (in the next per-target step, or its own
                                 launch); 2 the two-group kernel (d <= 128), which merges the
                                 split partials itself */
  STCA_OPT_TEST_STOP_TILES = 8, /* test hook, 0 = off: the tensor-core attention's loader stops
                                 after this many key tiles per CTA and the kernel takes the exit
                                 of a bounded wait that ran out (copies and MMAs in flight are
                                 let finish, TMEM is freed); the next stca_device_status then
                                 reports STCA_EDEVICE.  The forward's output is not valid then */
  STCA_OPT_BW_GEMM = 9,       /* products of the backward pieces for bf16 handles: 0 the library's
                                 tensor-core GEMM with TF32 operands (default); 1 cuBLASLt TF32
                                 (kept for comparison); fp32 handles always use exact fp32 */
  STCA_OPT_PIPELINE = 10,     /* 1 (default): when the forward runs the tensor-core attention
                                 with its in-kernel W_V projection (d = 128), stca_forward (not
                                 stca_forward_head) splits the requests into two halves of
                                 about equal attention work and runs one half's per-target step
                                 beside the other half's attention, in one launch per phase,
                                 when the batch has at least 24 (128-key tile x 128-row query
                                 tile) pairs of attention work per SM; 0: one batch, attention
                                 and step in turn.  Results are the same up to the split
                                 partials' rounding order. */
  STCA_OPT_LAUNCHES = 100,    /* read-only: kernels launched since the last encode */
  STCA_OPT_LAST_FORM = 101    /* read-only: 1 if the last forward ran the naive form, else 0 */
};
int stca_set_option(stca_handle* handle, int option, int64_t value);
int stca_get_option(stca_handle* handle, int option, int64_t* value);

/* Kernel classes reported by stca_kernel_times. */
enum { STCA_K_ENCODE = 0, STCA_K_ATTN = 1, STCA_K_STEP = 2, STCA_K_HEAD = 3,
       STCA_K_PIPE = 4,   /* a pipeline launch: one half's step beside the other half's attention */
       STCA_K_CLASSES = 5 };

/*
 * Device time of each kernel class since the previous call, from the CUDA
 * events recorded (on the launch stream) around every launch while
 * STCA_OPT_TIMING is 1.  Writes ms[c] (milliseconds, summed) and launches[c]
 * for c < min(n, STCA_K_CLASSES); either array may be NULL.  Waits for the
 * recorded events, then forgets them.
 */
int stca_kernel_times(stca_handle* handle, double* ms, int64_t* launches, int n);

/*
 * Device self-test of the attention softmax's exponential 2^x (an addition of
 * this library, for its own tests; the pages have no counterpart).  For n
 * fp32 inputs x (DEVICE), writes y (DEVICE) with method 0: the MUFU
 * ex2.approx; 1: the FMA-pipe form (range reduction to [-1/2, 1/2] and a
 * degree-3 minimax polynomial; relative error below 1.5e-4 for x in
 * [-126, 8], 2^-126 below -126); 2: the same two at a time with the packed
 * fp32 instructions, as the attention evaluates it.  Asynchronous on `stream`.
 * Errors: STCA_EINVAL, STCA_ECUDA.
 */
int stca_selftest_ex2(const float* x, float* y, int64_t n, int method, void* stream);

/* Message of the last error on this host thread ("" if none). */
const char* stca_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* STCA_H_ */
