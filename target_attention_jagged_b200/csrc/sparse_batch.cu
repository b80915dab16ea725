// Sparse-training batch builder ("Make It Long, Keep It Fast" digest, §2.3
// "Extrapolation: Train Sparsely, Infer Densely"; STCA blog, §2.6):
//   * the stochastic length curriculum: beta from the mean constraint (Eq. (17)),
//     the sequence sparsity (Eq. (15)), and per user L_raw = L_min + s (L_max -
//     L_min) (Eq. (16)) aligned down to a multiple of 8;
//   * the temporal-suffix selection: a user keeps its most recent rows, out of
//     at most L_infer;
//   * the batch-level load balance: (a) the batch is brought to exactly
//     B * L_avg rows by proportional shares (largest-remainder method),
//     (b) the suffixes are packed back to back into one padding-free stream with
//     a per-row user index, the ragged layout stca_encode reads.
// The plan is integer host work; the packing is one HBM-bound device gather.
#include <algorithm>
#include <cmath>
#include <string>
#include <vector>

#include "stca_internal.h"

namespace stca {
namespace {

// Rows of `total` shared in proportion to the non-negative weights w: the floor
// of each exact quota w_b total / W, then one more row to the `total - sum`
// users whose quotas have the largest remainders (ties to the lower index).
// All remainders share the denominator W, so they compare as integers.
void share_rows(const std::vector<int64_t>& w, int64_t total, std::vector<int64_t>& out) {
  const size_t n = w.size();
  out.assign(n, 0);
  if (total == 0) return;
  __int128 W = 0;
  for (int64_t x : w) W += x;
  std::vector<int64_t> rem(n);
  int64_t given = 0;
  for (size_t b = 0; b < n; ++b) {
    const __int128 num = static_cast<__int128>(w[b]) * total;
    out[b] = static_cast<int64_t>(num / W);
    rem[b] = static_cast<int64_t>(num % W);
    given += out[b];
  }
  const int64_t left = total - given;     // < number of users with a nonzero remainder
  std::vector<int64_t> order(n);
  for (size_t b = 0; b < n; ++b) order[b] = static_cast<int64_t>(b);
  std::partial_sort(order.begin(), order.begin() + left, order.end(), [&](int64_t a, int64_t c) {
    return rem[a] != rem[c] ? rem[a] > rem[c] : a < c;
  });
  for (int64_t i = 0; i < left; ++i) out[order[i]] += 1;
}

// Packed row p -> its user, then the row copy.  A warp owns a contiguous run
// of packed rows; it finds the user of its first row by binary search over the
// packed offsets and walks forward.  Rows move as 16-byte vectors with
// streaming (evict-first) loads and stores; eight rows are in flight per warp
// when a row is at most 32 vectors long.  A source row outside [0, N) is not
// read: its packed row is left as it was and its seg entry is -1.
constexpr int kGatherThreads = 256;
// u[lane] without dynamic register indexing
template <int N>
__device__ __forceinline__ int32_t user_sel(const int32_t (&u)[N], int lane) {
  int32_t r = -1;
#pragma unroll
  for (int i = 0; i < N; ++i) r = lane == i ? u[i] : r;
  return r;
}

__device__ __forceinline__ int64_t user_of(const int64_t* poff, int64_t B, int64_t p) {
  int64_t lo = 0, hi = B;                 // poff[lo] <= p < poff[hi] when offsets are valid
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) >> 1;
    if (__ldg(poff + mid) <= p) lo = mid;
    else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kGatherThreads) sl_gather_kernel(
    const uint4* __restrict__ X, int64_t N, int row16, const int64_t* __restrict__ src_start,
    const int64_t* __restrict__ poff, int64_t B, int64_t P, uint4* __restrict__ Y,
    int32_t* __restrict__ seg) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kGatherThreads / 32);
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (kGatherThreads / 32) + (threadIdx.x >> 5);
  const int64_t per = (P + warps - 1) / warps;
  const int64_t p0 = w * per, p1 = min(P, p0 + per);
  if (p0 >= p1) return;
  int64_t b = user_of(poff, B, p0);
  int64_t next = b + 1 < B ? __ldg(poff + b + 1) : P;   // first row of the next user
  int64_t base = __ldg(poff + b), src = __ldg(src_start + b);
  constexpr int kRows = 8;
  for (int64_t p = p0; p < p1; p += kRows) {
    int64_t srow[kRows];
    int32_t user[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int64_t q = p + r;
      srow[r] = -1;
      user[r] = -1;
      if (q < p1) {
        while (q >= next && b + 1 < B) {
          ++b;
          base = next;
          src = __ldg(src_start + b);
          next = b + 1 < B ? __ldg(poff + b + 1) : P;
        }
        const int64_t s = src + (q - base);
        if (s >= 0 && s < N) {
          srow[r] = s;
          user[r] = static_cast<int32_t>(b);
        }
      }
    }
    if (seg && lane < kRows && p + lane < p1)
      seg[p + lane] = user_sel(user, lane);
    for (int c = lane; c < row16; c += 32) {
      uint4 v[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r)
        if (srow[r] >= 0) v[r] = __ldcs(X + srow[r] * row16 + c);
#pragma unroll
      for (int r = 0; r < kRows; ++r)
        if (srow[r] >= 0) __stcs(Y + (p + r) * row16 + c, v[r]);
    }
  }
}

}  // namespace
}  // namespace stca

using namespace stca;

extern "C" int stca_sl_beta(double alpha, int64_t L_min, int64_t L_max, int64_t L_avg,
                            double* beta, double* ss) {
  if (!beta) return set_error(STCA_EINVAL, "beta is NULL");
  if (!(alpha > 0) || !std::isfinite(alpha))
    return set_error(STCA_EINVAL, "alpha must be a positive finite number");
  if (!(L_min >= 0 && L_min < L_avg && L_avg < L_max))
    return set_error(STCA_EINVAL, "need 0 <= L_min < L_avg < L_max");
  *beta = alpha * static_cast<double>(L_max - L_avg) / static_cast<double>(L_avg - L_min);
  if (ss) *ss = static_cast<double>(L_avg) / static_cast<double>(L_max);
  set_error(STCA_OK, "");
  return STCA_OK;
}

extern "C" int stca_sl_plan(const int64_t* hist_offsets, int64_t B, const double* s,
                            int64_t L_min, int64_t L_max, int64_t L_avg, int64_t L_infer,
                            int64_t* train, int64_t* lengths, int64_t* packed_offsets,
                            int64_t* src_start) {
  if (B < 1) return set_error(STCA_EINVAL, "B must be >= 1");
  if (!hist_offsets || !s || !lengths || !packed_offsets || !src_start)
    return set_error(STCA_EINVAL, "stca_sl_plan: NULL argument");
  if (!(L_min >= 0 && L_min < L_avg && L_avg < L_max) || L_infer < 1)
    return set_error(STCA_EINVAL, "need 0 <= L_min < L_avg < L_max and L_infer >= 1");
  if (B > (int64_t(1) << 40) / std::max<int64_t>(L_avg, 1))
    return set_error(STCA_EINVAL, "stca_sl_plan: B * L_avg too large");
  if (hist_offsets[0] != 0) return set_error(STCA_EINVAL, "hist_offsets[0] != 0");
  std::vector<int64_t> usable(B), capped(B), out;
  int64_t S = 0, U = 0;
  for (int64_t b = 0; b < B; ++b) {
    const int64_t H = hist_offsets[b + 1] - hist_offsets[b];
    if (H < 1)
      return set_error(STCA_EINVAL, "user " + std::to_string(b) +
                                        " has an empty history (or offsets decrease)");
    const double sb = s[b];
    if (!(sb >= 0.0 && sb <= 1.0)) return set_error(STCA_EINVAL, "s must lie in [0, 1]");
    // Eq. (16) in double, product then sum, then aligned down to 8 (at least 8)
    const double prod = sb * static_cast<double>(L_max - L_min);
    const double raw = static_cast<double>(L_min) + prod;
    int64_t Lt = (static_cast<int64_t>(std::floor(raw)) / 8) * 8;
    if (Lt < 8) Lt = 8;
    if (train) train[b] = Lt;
    usable[b] = std::min(H, L_infer);
    capped[b] = std::min(Lt, usable[b]);
    S += capped[b];
    U += usable[b];
  }
  const int64_t budget = B * L_avg;
  std::vector<int64_t> len(capped);
  if (S > budget) {
    std::vector<int64_t> w(B);
    for (int64_t b = 0; b < B; ++b) w[b] = capped[b] - 1;
    share_rows(w, budget - B, out);
    for (int64_t b = 0; b < B; ++b) len[b] = 1 + out[b];
  } else if (S < budget) {
    if (U - S <= budget - S) {
      len = usable;
    } else {
      std::vector<int64_t> w(B);
      for (int64_t b = 0; b < B; ++b) w[b] = usable[b] - capped[b];
      share_rows(w, budget - S, out);
      for (int64_t b = 0; b < B; ++b) len[b] = capped[b] + out[b];
    }
  }
  packed_offsets[0] = 0;
  for (int64_t b = 0; b < B; ++b) {
    lengths[b] = len[b];
    packed_offsets[b + 1] = packed_offsets[b] + len[b];
    src_start[b] = hist_offsets[b + 1] - len[b];
  }
  set_error(STCA_OK, "");
  return STCA_OK;
}

extern "C" int stca_sl_gather(const void* X, int64_t N, int64_t row_bytes,
                              const int64_t* src_start, const int64_t* packed_offsets, int64_t B,
                              int64_t P, void* X_packed, int32_t* seg, void* stream) {
  if (B < 1 || N < 0 || P < 0) return set_error(STCA_EINVAL, "stca_sl_gather: bad sizes");
  if (P == 0) {
    set_error(STCA_OK, "");
    return STCA_OK;
  }
  if (!X || !src_start || !packed_offsets || !X_packed)
    return set_error(STCA_EINVAL, "stca_sl_gather: NULL argument");
  if (row_bytes <= 0 || row_bytes % 16 || row_bytes / 16 > (int64_t(1) << 20))
    return set_error(STCA_EINVAL, "row_bytes must be a positive multiple of 16");
  if (reinterpret_cast<uintptr_t>(X) % 16 || reinterpret_cast<uintptr_t>(X_packed) % 16)
    return set_error(STCA_EINVAL, "X and X_packed must be 16-byte aligned");
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  // four 256-thread CTAs per SM, fewer when the batch is small
  const int64_t want = (P + 4 * (kGatherThreads / 32) - 1) / (4 * (kGatherThreads / 32));
  const unsigned grid = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(4 * sms, want)));
  sl_gather_kernel<<<grid, kGatherThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(X), N, static_cast<int>(row_bytes / 16), src_start, packed_offsets,
      B, P, static_cast<uint4*>(X_packed), seg);
  STCA_CUDA_TRY(cudaGetLastError());
  set_error(STCA_OK, "");
  return STCA_OK;
}
