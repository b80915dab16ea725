// Tensor-core split-L single-query attention: its kernel and host launchers
// (the device code, and what the kernel computes, are in attn_tc_dev.cuh).
#include <cuda.h>

#include <algorithm>
#include <string>
#include <vector>

#include "attn_tc_dev.cuh"

namespace stca {
namespace {

// tmV: the value tiles (SEPV) or the [W_V]^T tile (PROJ); otherwise unused.
template <int D, int QB, int KS, int PB, bool SEPV, bool QT, bool PROJ>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  attn_tc_body<D, QB, KS, PB, SEPV, QT, PROJ>(tmQ, tmK, tmV, p, smem_raw, static_cast<int>(blockIdx.x));
}

template <int D, int QB, int KS, int PB, bool SEPV = false, bool QT = false, bool PROJ = false>
int launch_cfg(stca_handle* H, const CUtensorMap& tmQ, const CUtensorMap& tmK, const AttnParams& p,
               int grid, cudaStream_t s, const CUtensorMap* tmV = nullptr) {
  using C = AttnCfg<D, QB, KS, PB, SEPV, QT, PROJ>;
  auto k = attn_tc_kernel<D, QB, KS, PB, SEPV, QT, PROJ>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("attn_tc smem: ") + cudaGetErrorString(e));
  e = launch_pdl(k, dim3(grid), dim3(kAttnThreads), C::kSmem, s, tmQ, tmK, tmV ? *tmV : tmK, p);
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("attn_tc launch: ") + cudaGetErrorString(e));
  return STCA_OK;
}

}  // namespace

bool attn_tc_supported(int d) { return d == 64 || d == 128 || d == 256; }

bool attn_tc_proj_supported(const stca_handle* H) {
  return H->d == 128 && H->wvt != nullptr && H->dh % 4 == 0;
}

int launch_attn_tc(stca_handle* H, int layer, const AttnItem* items_d, const int32_t* cta_begin_d,
                   int grid, cudaStream_t s, bool proj, const QslotBufs* qs) {
  AttnParams p{};
  p.items = items_d;
  p.cta_item_begin = cta_begin_d;
  const int64_t G = H->last_G;
  p.pacc = H->part;
  p.pm = H->part + G * H->d;
  p.pl = p.pm + G;
  p.status = H->status_d;
  p.stop_tiles = H->opt_stop_tiles;
  p.h = H->h;
  p.dh = H->dh;
  if (qs) {
    if (!proj) return set_error(STCA_EINVAL, "per-row partial slots need the in-kernel projection");
    p.qslot = 1;
    p.pair_item_begin = qs->pair_item_begin;
    p.pacc = qs->pacc;
    p.qml = qs->qml;
    p.qn = qs->qn;
  }
  const CUtensorMap& tmK = H->tmXt[layer];
  if (proj) {
    if (!attn_tc_proj_supported(H)) return set_error(STCA_EINVAL, "in-kernel W_V projection needs d = 128");
    return launch_cfg<128, 1, 5, 1, false, true, true>(H, H->tmU, tmK, p, grid, s, &H->tmWvT[layer]);
  }
  switch (H->d) {
    case 64: return launch_cfg<64, 2, 10, 2, false, true>(H, H->tmU, tmK, p, grid, s);
    case 128: return launch_cfg<128, 2, 5, 1, false, true>(H, H->tmU, tmK, p, grid, s);
    case 256: return launch_cfg<256, 1, 2, 1>(H, H->tmU, tmK, p, grid, s);
    default: return set_error(STCA_EINVAL, "tensor-core attention needs d in {64, 128, 256}");
  }
}

// Naive form: packed query rows (H->tmU over the [rows x 64] layout), keys and
// values of the projection (H->tmKn, H->tmVn); partial rows are 64 wide.
int launch_attn_tc_naive(stca_handle* H, const AttnItem* items_d, const int32_t* cta_begin_d,
                         int grid, cudaStream_t s) {
  AttnParams p{};
  p.items = items_d;
  p.cta_item_begin = cta_begin_d;
  const int64_t G = H->last_G;
  p.pacc = H->part;
  p.pm = H->part + G * 64;
  p.pl = p.pm + G;
  p.status = H->status_d;
  p.stop_tiles = H->opt_stop_tiles;
  return launch_cfg<64, 2, 5, 2, true>(H, H->tmU, H->tmKn, p, grid, s, &H->tmVn);
}

// The same kernel with every buffer given explicitly (no handle state).
int launch_attn_tc_ws(int d, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                      const AttnItem* items_d, const int32_t* cta_begin_d, int grid, float* part,
                      int64_t G, int* status, cudaStream_t s) {
  AttnParams p{};
  p.items = items_d;
  p.cta_item_begin = cta_begin_d;
  p.pacc = part;
  p.pm = part + G * d;
  p.pl = p.pm + G;
  p.status = status;
  switch (d) {
    case 64: return launch_cfg<64, 2, 10, 2, false, true>(nullptr, tmQ, tmK, p, grid, s);
    case 128: return launch_cfg<128, 2, 5, 1, false, true>(nullptr, tmQ, tmK, p, grid, s);
    case 256: return launch_cfg<256, 1, 2, 1>(nullptr, tmQ, tmK, p, grid, s);
    default: return set_error(STCA_EINVAL, "tensor-core attention needs d in {64, 128, 256}");
  }
}

}  // namespace stca
