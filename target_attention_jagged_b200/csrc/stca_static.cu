// stca_forward_static: stca_forward without any device allocation.
//
// Who needs it: a caller that must not call cudaMalloc once it is serving --
// a process whose device memory is already handed out to another allocator's
// pool (so a late cudaMalloc fails or steals from it), a deployment with a
// fixed per-process memory budget set at start-up, or a latency-critical loop
// that cannot afford the device-wide synchronisation cudaMalloc / cudaFree may
// imply.  stca_forward grows its workspace (query rows, split partials, work
// plan) on demand; this variant keeps all of it in one fixed array compiled
// into the library instead, so after stca_init and stca_encode nothing more is
// allocated on the device.  The call uses no CUDA or library allocation
// routine; its host-side work plan lives in ordinary heap memory.
//
// Set-up: the first call on each device looks up the array's device address
// with cudaGetSymbolAddress (with that device current), which also loads the
// module that holds the array.  No call can be captured into a CUDA graph: the
// work plan is uploaded from host memory each time, so a call under an active
// capture is refused.  The attention runs in the reordered form of Eq. (13);
// the per-target step runs where stca_forward would run it.
//
// The array is file-scope device memory of kStaticScratchBytes (32 MiB).
// Every GPU that loads the library holds it until the process exits, and
// every call on a device shares it: two calls whose work overlaps on the GPU
// (different streams, or different handles on one device) race on it, so
// order such calls on one stream or serialise them.  A call reads nothing that
// an earlier call left there: the plan, the query rows and every partial row
// it reads are written by the same call first.  Workspace per call: the plan,
// T*h*d bf16 query rows, T*h*d fp32 merged rows and the split partials.
#include <cuda_runtime.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "stca_internal.h"

namespace stca {
namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on each device, looked up once with that
// device current (in host code the symbol itself is only a host-side handle).
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

int scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return set_error(STCA_EINVAL, "device index out of range");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return set_error(STCA_ECUDA, std::string("cudaGetSymbolAddress(static scratch): ") +
                                       cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return STCA_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch layout of one call.
struct StaticLayout {
  size_t items, cta, treq, toff, rpb, pib, plan_end, ubf, cbuf, part, total;
};

StaticLayout layout_for(const PlanHost& P, int64_t R, int64_t T, int h, int d) {
  StaticLayout L{};
  L.items = 0;
  L.cta = up256(L.items + P.items.size() * sizeof(AttnItem));
  L.treq = up256(L.cta + P.cta_begin.size() * sizeof(int32_t));
  L.toff = up256(L.treq + static_cast<size_t>(T) * sizeof(int32_t));
  L.rpb = up256(L.toff + static_cast<size_t>(R + 1) * sizeof(int64_t));
  L.pib = up256(L.rpb + static_cast<size_t>(R + 1) * sizeof(int32_t));
  L.plan_end = up256(L.pib + P.pair_item_begin.size() * sizeof(int32_t));
  L.ubf = L.plan_end;
  L.cbuf = up256(L.ubf + static_cast<size_t>(T) * h * d * 2);
  L.part = up256(L.cbuf + static_cast<size_t>(T) * h * d * sizeof(float));
  L.total = up256(L.part + static_cast<size_t>(std::max<int64_t>(P.G, 1)) * (d + 2) * sizeof(float));
  return L;
}

}  // namespace
}  // namespace stca

using namespace stca;

extern "C" int stca_forward_static(stca_handle* H, const void* targets,
                                   const int64_t* target_offsets, int64_t T, float* Z,
                                   void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (!H->encoded) return set_error(STCA_ESTATE, "stca_forward_static before a successful stca_encode");
  if (T < 0) return set_error(STCA_EINVAL, "T must be >= 0");
  if (stca_validate_offsets(target_offsets, H->R, T, 0) != STCA_OK) return STCA_EINVAL;
  if (T == 0) return STCA_OK;
  if (!targets || !Z) return set_error(STCA_EINVAL, "targets or Z is NULL");
  if (reinterpret_cast<uintptr_t>(targets) % 16 || reinterpret_cast<uintptr_t>(Z) % 16)
    return set_error(STCA_EINVAL, "targets and Z must be 16-byte aligned");
  if (H->dtype != STCA_BF16 || !attn_tc_supported(H->d) || H->opt_attn_path == 1)
    return set_error(STCA_EINVAL,
                     "stca_forward_static runs the tensor-core path only: bf16 and d in {64, 128, 256}");
  if (H->opt_attn_form == 1)
    return set_error(STCA_EINVAL, "stca_forward_static runs the reordered form (Eq. (13)) only; "
                                  "STCA_OPT_ATTN_FORM 1 (the naive form) is not available here");
  if (H->opt_step_path == 2 && !H->step_tc_ready)
    return set_error(STCA_EINVAL, "tensor-core step needs bf16, d in {128, 256} and r d <= 512");
  {
    // the host-side plan is copied from this thread's staging memory on every
    // call, so a captured call would replay whatever that memory holds later
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cs) != cudaSuccess) {
      cudaGetLastError();
      return set_error(STCA_ECUDA, "stca_forward_static: cannot query the stream's capture state");
    }
    if (cs != cudaStreamCaptureStatusNone)
      return set_error(STCA_EINVAL, "stca_forward_static cannot be captured into a CUDA graph "
                                    "(its work plan is uploaded from host memory on every call)");
  }
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return set_error(STCA_ECUDA, "cudaGetDevice failed");
  if (prev != H->device && cudaSetDevice(H->device) != cudaSuccess)
    return set_error(STCA_ECUDA, "cannot select the handle's device");
  struct Restore {
    int dev;
    ~Restore() { if (dev >= 0) cudaSetDevice(dev); }
  } restore{prev != H->device ? prev : -1};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = H->d, h = H->h;
  const int64_t R = H->R;
  const int64_t* off = H->offsets_h.data();

  // Plan as stca_forward does; if the partials do not fit, use fewer, longer
  // runs (fewer CTAs) until they do.
  thread_local PlanHost P;
  thread_local std::vector<unsigned char> staging;
  // Runs per CTA are equal, so halving the CTAs roughly halves the items that
  // a pair's keys split into; stop once a halving no longer shrinks the
  // partials (e.g. when STCA_OPT_SPLIT_KEYS already caps the run length).
  int ctas = H->num_sms;
  StaticLayout L{};
  int64_t prev_G = -1;
  for (;;) {
    build_plan_host(off, target_offsets, R, h, 2, ctas, H->opt_split_keys, P);
    if (int rc = check_plan(P, off, target_offsets, R, h, 2)) return rc;
    L = layout_for(P, R, T, h, d);
    if (L.total <= kStaticScratchBytes || ctas == 1 || P.G == prev_G) break;
    prev_G = P.G;
    ctas = std::max(1, ctas / 2);
  }
  if (L.total > kStaticScratchBytes)
    return set_error(STCA_EINVAL, "batch needs " + std::to_string(L.total) +
                                      " bytes of scratch; the static scratch holds " +
                                      std::to_string(kStaticScratchBytes) +
                                      " (use stca_forward, or fewer targets per call)");
  void* base = nullptr;
  if (int rc = scratch_address(H->device, &base)) return rc;
  unsigned char* sc = static_cast<unsigned char*>(base);

  // plan -> scratch (the copy reads `staging` before returning)
  if (staging.size() < L.plan_end) staging.resize(L.plan_end);
  unsigned char* hp = staging.data();
  memcpy(hp + L.items, P.items.data(), P.items.size() * sizeof(AttnItem));
  memcpy(hp + L.cta, P.cta_begin.data(), P.cta_begin.size() * sizeof(int32_t));
  int32_t* treq = reinterpret_cast<int32_t*>(hp + L.treq);
  for (int64_t r = 0; r < R; ++r)
    for (int64_t t = target_offsets[r]; t < target_offsets[r + 1]; ++t) treq[t] = static_cast<int32_t>(r);
  memcpy(hp + L.toff, target_offsets, static_cast<size_t>(R + 1) * sizeof(int64_t));
  memcpy(hp + L.rpb, P.req_pair_begin.data(), static_cast<size_t>(R + 1) * sizeof(int32_t));
  memcpy(hp + L.pib, P.pair_item_begin.data(), P.pair_item_begin.size() * sizeof(int32_t));
  STCA_CUDA_TRY(cudaMemcpyAsync(sc, hp, L.plan_end, cudaMemcpyHostToDevice, s));

  const AttnItem* items_d = reinterpret_cast<const AttnItem*>(sc + L.items);
  const int32_t* cta_d = reinterpret_cast<const int32_t*>(sc + L.cta);
  uint16_t* Ubf = reinterpret_cast<uint16_t*>(sc + L.ubf);
  float* part = reinterpret_cast<float*>(sc + L.part);
  float* cbuf = reinterpret_cast<float*>(sc + L.cbuf);
  CUtensorMap tmU;
  if (int rc = make_tmap_bf16_2d(&tmU, Ubf, d, static_cast<uint64_t>(T) * h, 64, 128)) return rc;
  StepPlan plan;
  plan.treq = reinterpret_cast<const int32_t*>(sc + L.treq);
  plan.toff = reinterpret_cast<const int64_t*>(sc + L.toff);
  plan.req_pair_begin = reinterpret_cast<const int32_t*>(sc + L.rpb);
  plan.pair_item_begin = reinterpret_cast<const int32_t*>(sc + L.pib);
  plan.items = items_d;
  plan.mtile_rows = 128;
  plan.log2_partials = 1;

  // The per-target step runs where stca_forward runs it: on the tensor cores
  // when the handle has that step (merging the split partials itself when
  // every query tile has few enough items), else on the CUDA cores.
  const bool step_tc = H->step_tc_ready && H->opt_step_path != 1;
  int max_items = 0;
  for (size_t k = 0; k + 1 < P.pair_item_begin.size(); ++k)
    max_items = std::max(max_items, P.pair_item_begin[k + 1] - P.pair_item_begin[k]);
  const bool fused = step_tc && max_items <= step_tc_max_items();
  auto step = [&](int layer, const float* cm) -> int {
    if (step_tc)
      return launch_step_tc(H, layer, targets, T, fused ? nullptr : cm, &plan, part, P.G, Z, Ubf, s);
    launch_target_step_ws(H, layer, targets, T, cm, Z, Ubf, s);
    return STCA_OK;
  };
  if (int rc = step(-1, nullptr)) return rc;
  if (cudaError_t e = cudaGetLastError())
    return set_error(STCA_ECUDA, std::string("query init: ") + cudaGetErrorString(e));
  for (int i = 0; i < H->M; ++i) {
    if (int rc = launch_attn_tc_ws(d, tmU, H->tmXt[i], items_d, cta_d, P.grid, part, P.G,
                                   H->status_d, s))
      return rc;
    if (cudaError_t e = cudaGetLastError())
      return set_error(STCA_ECUDA, std::string("attention: ") + cudaGetErrorString(e));
    if (!fused) launch_combine(H, plan, part, P.G, T, cbuf, s);
    if (int rc = step(i, cbuf)) return rc;
    if (cudaError_t e = cudaGetLastError())
      return set_error(STCA_ECUDA, std::string("target step: ") + cudaGetErrorString(e));
  }
  return STCA_OK;
}
