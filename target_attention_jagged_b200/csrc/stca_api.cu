// C ABI of the STCA forward library: argument checks, weight staging, the
// attention work plan and the launch sequence.  See include/stca.h.
#include <cuda_runtime.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <new>
#include <string>
#include <vector>

#include <cublasLt.h>

#include "stca_internal.h"

namespace stca {

static thread_local std::string g_err;

int set_error(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

static int ok() {
  g_err.clear();
  return STCA_OK;
}

// Make the handle's device current for the duration of a call.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { prev = -1; ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

static int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(STCA_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return STCA_OK;
}

// Grow-only device buffer.
static int ensure_dev(void** p, size_t* cap, size_t need) {
  if (need <= *cap && *p) return STCA_OK;
  if (*p) { cudaFree(*p); *p = nullptr; *cap = 0; }
  size_t bytes = std::max<size_t>(need, 256);
  bytes = (bytes + (1u << 20) - 1) & ~static_cast<size_t>((1u << 20) - 1);
  if (cudaMalloc(p, bytes) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return set_error(STCA_ENOMEM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed");
  }
  *cap = bytes;
  return STCA_OK;
}

// Optional CUDA events around one launch (STCA_OPT_TIMING).
static cudaEvent_t pool_event(stca_handle* H) {
  if (!H->ev_pool.empty()) {
    cudaEvent_t e = H->ev_pool.back();
    H->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) { cudaGetLastError(); return nullptr; }
  return e;
}

struct TimedLaunch {
  stca_handle* H;
  int cls;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  TimedLaunch(stca_handle* h, int c, cudaStream_t st) : H(h), cls(c), s(st) {
    if (H->timing && (a = pool_event(H))) cudaEventRecord(a, s);
  }
  ~TimedLaunch() {
    if (!a) return;
    cudaEvent_t b = pool_event(H);
    if (!b) { H->ev_pool.push_back(a); return; }
    cudaEventRecord(b, s);
    H->timed.push_back({cls, a, b});
  }
};

static int validate_offsets(const int64_t* off, int64_t R, int64_t total, bool nonempty,
                            const char* name) {
  if (!off) return set_error(STCA_EINVAL, std::string(name) + " is NULL");
  if (R < 1) return set_error(STCA_EINVAL, "R must be >= 1");
  if (off[0] != 0) return set_error(STCA_EINVAL, std::string(name) + "[0] != 0");
  for (int64_t r = 0; r < R; ++r) {
    const int64_t len = off[r + 1] - off[r];
    if (len < 0)
      return set_error(STCA_EINVAL, std::string(name) + " decreases at index " +
                                        std::to_string(r + 1));
    if (nonempty && len == 0)
      return set_error(STCA_EINVAL, std::string(name) + ": segment " + std::to_string(r) +
                                        " is empty (an empty history has no softmax)");
    if (len > INT32_MAX)
      return set_error(STCA_EINVAL, std::string(name) + ": segment too long");
  }
  if (off[R] != total)
    return set_error(STCA_EINVAL, std::string(name) + "[R] = " + std::to_string(off[R]) +
                                      " != " + std::to_string(total));
  return STCA_OK;
}

// ------------------------------------------------------------------ weights
static float bf16_bits_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// Copy `n` dtype elements from a host or device pointer into fp32.
static int fetch(const void* src, size_t n, int dtype, bool on_device, std::vector<float>* out,
                 const char* name) {
  if (!src) return set_error(STCA_EINVAL, std::string("weight ") + name + " is NULL");
  const size_t esz = dtype == STCA_BF16 ? 2 : 4;
  std::vector<uint8_t> raw;
  const uint8_t* p = static_cast<const uint8_t*>(src);
  if (on_device) {
    raw.resize(n * esz);
    STCA_CUDA_TRY(cudaMemcpy(raw.data(), src, n * esz, cudaMemcpyDeviceToHost));
    p = raw.data();
  }
  out->resize(n);
  if (dtype == STCA_BF16) {
    for (size_t i = 0; i < n; ++i) {
      uint16_t b;
      memcpy(&b, p + 2 * i, 2);
      (*out)[i] = bf16_bits_to_float(b);
    }
  } else {
    memcpy(out->data(), p, n * 4);
  }
  return STCA_OK;
}

static const void* layer_ptr(const void* const* field, int i) { return field ? field[i] : nullptr; }

}  // namespace stca

using namespace stca;

// ====================================================================== ABI
extern "C" const char* stca_last_error(void) { return g_err.c_str(); }

extern "C" int stca_validate_offsets(const int64_t* offsets, int64_t R, int64_t total,
                                     int require_nonempty) {
  int rc = validate_offsets(offsets, R, total, require_nonempty != 0, "offsets");
  return rc == STCA_OK ? ok() : rc;
}

extern "C" void stca_destroy(stca_handle* H) {
  if (!H) return;
  DeviceGuard g(H->device);
  cudaDeviceSynchronize();
  cudaFree(H->w32);
  cudaFree(H->wstep);
  cudaFree(H->wstep_tc);
  cudaFree(H->whead);
  cudaFree(H->w32head);
  cudaFree(H->wkv);
  cudaFree(H->wvt);
  cudaFree(H->kv);
  cudaFree(H->lt_ws);
  cudaFree(H->bw_ws);
  cudaFree(H->bw_plan);
  if (H->lt) cublasLtDestroy(static_cast<cublasLtHandle_t>(H->lt));
  cudaFree(H->wtc);
  cudaFree(H->xt);
  cudaFree(H->q);
  cudaFree(H->U);
  cudaFree(H->Ubf);
  cudaFree(H->part);
  cudaFree(H->cbuf);
  cudaFree(H->attn_cnt);
  cudaFree(H->plan_d);
  cudaFree(H->status_d);
  cudaFree(H->x_stage);
  cudaFree(H->t_stage);
  cudaFree(H->z_stage);
  if (H->plan_h) cudaFreeHost(H->plan_h);
  for (auto e : H->chunk_evt) cudaEventDestroy(e);
  if (H->copy_stream) cudaStreamDestroy(H->copy_stream);
  if (H->plan_evt) cudaEventDestroy(H->plan_evt);
  for (auto& t : H->timed) { cudaEventDestroy(t.a); cudaEventDestroy(t.b); }
  for (auto e : H->ev_pool) cudaEventDestroy(e);
  delete H;
}

extern "C" int stca_init(const stca_weights* w, int d, int h, int r, int M, int dtype,
                         int weights_on_device, stca_handle** out) {
  if (!out) return set_error(STCA_EINVAL, "out is NULL");
  *out = nullptr;
  if (!w) return set_error(STCA_EINVAL, "weights is NULL");
  if (d < 8 || d > 1024 || d % 8) return set_error(STCA_EINVAL, "d must be in [8, 1024], d % 8 == 0");
  if (h < 1 || d % h) return set_error(STCA_EINVAL, "h must divide d");
  if ((d / h) % 2) return set_error(STCA_EINVAL, "h must divide d with an even d / h");
  if (r < 1 || static_cast<int64_t>(r) * d > 4096) return set_error(STCA_EINVAL, "need 1 <= r, r*d <= 4096");
  if (M < 1 || M > 16) return set_error(STCA_EINVAL, "M must be in [1, 16]");
  if (dtype != STCA_F32 && dtype != STCA_BF16) return set_error(STCA_EINVAL, "dtype must be STCA_F32 or STCA_BF16");
  if (!w->Wu || !w->Wg || !w->Wd || !w->Wq || !w->Wk || !w->Wv || !w->Wo)
    return set_error(STCA_EINVAL, "a required weight field is NULL");
  if (M > 1 && !w->Wc) return set_error(STCA_EINVAL, "Wc is NULL but M > 1");
  const bool qffn = w->qWu || w->qWg || w->qWd;
  if (qffn && !(w->qWu && w->qWg && w->qWd))
    return set_error(STCA_EINVAL, "qWu, qWg and qWd must be given together");
  if ((w->q_ln_gamma == nullptr) != (w->q_ln_beta == nullptr))
    return set_error(STCA_EINVAL, "q_ln_gamma and q_ln_beta must be given together");
  if ((w->ln_gamma == nullptr) != (w->ln_beta == nullptr))
    return set_error(STCA_EINVAL, "ln_gamma and ln_beta must be given together");
  const int nhead = (w->Wz != nullptr) + (w->zWu != nullptr) + (w->zWg != nullptr) + (w->zWd != nullptr);
  if (nhead != 0 && nhead != 4)
    return set_error(STCA_EINVAL, "Wz, zWu, zWg and zWd must be given together");

  stca_handle* H = new (std::nothrow) stca_handle();
  if (!H) return set_error(STCA_ENOMEM, "host allocation failed");
  if (cudaGetDevice(&H->device) != cudaSuccess) {
    delete H;
    cudaGetLastError();
    return set_error(STCA_ECUDA, "no CUDA device");
  }
  H->d = d; H->h = h; H->r = r; H->M = M; H->dtype = dtype;
  H->rd = r * d; H->dh = d / h;
  H->elem = dtype == STCA_BF16 ? 2 : 4;
  const int rd = H->rd, dh = H->dh;
  const bool dev = weights_on_device != 0;
  if (target_step_smem(H) > 227 * 1024) {
    delete H;
    return set_error(STCA_EINVAL, "per-target step needs more than 227 KB shared memory for these sizes");
  }

  // ---- fp32 slab: per layer Wu Wg Wd [qWu qWg qWd] ln_g ln_b Wq WkT Wv Wo [Wc]; then q_ln
  std::vector<size_t> lay_off(M + 1, 0);
  auto layer_floats = [&](int i) {
    size_t n = 3 * static_cast<size_t>(d) * rd + 2 * static_cast<size_t>(d) + 4 * static_cast<size_t>(d) * d;
    if (qffn) n += 3 * static_cast<size_t>(d) * rd;
    if (i > 0) n += static_cast<size_t>(i + 1) * d * d;
    return n;
  };
  for (int i = 0; i < M; ++i) lay_off[i + 1] = lay_off[i] + layer_floats(i);
  const size_t total = lay_off[M] + 2 * static_cast<size_t>(d);
  std::vector<float> slab(total, 0.f), tmp;
  int rc = STCA_OK;
  auto put = [&](size_t at, const void* src, size_t n, const char* name) -> int {
    int e = fetch(src, n, dtype, dev, &tmp, name);
    if (e) return e;
    std::copy(tmp.begin(), tmp.end(), slab.begin() + at);
    return STCA_OK;
  };
  struct Offs { size_t Wu, Wg, Wd, qWu, qWg, qWd, lg, lb, Wq, WkT, Wv, Wo, Wc; };
  std::vector<Offs> offs(M);
  for (int i = 0; i < M && rc == STCA_OK; ++i) {
    size_t at = lay_off[i];
    Offs& o = offs[i];
    o.Wu = at; at += static_cast<size_t>(d) * rd;
    o.Wg = at; at += static_cast<size_t>(d) * rd;
    o.Wd = at; at += static_cast<size_t>(rd) * d;
    if (qffn) {
      o.qWu = at; at += static_cast<size_t>(d) * rd;
      o.qWg = at; at += static_cast<size_t>(d) * rd;
      o.qWd = at; at += static_cast<size_t>(rd) * d;
    } else {
      o.qWu = o.Wu; o.qWg = o.Wg; o.qWd = o.Wd;
    }
    o.lg = at; at += d;
    o.lb = at; at += d;
    o.Wq = at; at += static_cast<size_t>(d) * d;
    o.WkT = at; at += static_cast<size_t>(d) * d;
    o.Wv = at; at += static_cast<size_t>(d) * d;
    o.Wo = at; at += static_cast<size_t>(d) * d;
    o.Wc = 0;
    if (i > 0) { o.Wc = at; at += static_cast<size_t>(i + 1) * d * d; }
    if ((rc = put(o.Wu, w->Wu[i], static_cast<size_t>(d) * rd, "Wu"))) break;
    if ((rc = put(o.Wg, w->Wg[i], static_cast<size_t>(d) * rd, "Wg"))) break;
    if ((rc = put(o.Wd, w->Wd[i], static_cast<size_t>(rd) * d, "Wd"))) break;
    if (qffn) {
      if ((rc = put(o.qWu, w->qWu[i], static_cast<size_t>(d) * rd, "qWu"))) break;
      if ((rc = put(o.qWg, w->qWg[i], static_cast<size_t>(d) * rd, "qWg"))) break;
      if ((rc = put(o.qWd, w->qWd[i], static_cast<size_t>(rd) * d, "qWd"))) break;
    }
    if (w->ln_gamma) {
      if ((rc = put(o.lg, layer_ptr(w->ln_gamma, i), d, "ln_gamma"))) break;
      if ((rc = put(o.lb, layer_ptr(w->ln_beta, i), d, "ln_beta"))) break;
    } else {
      std::fill(slab.begin() + o.lg, slab.begin() + o.lg + d, 1.f);
    }
    if ((rc = put(o.Wq, w->Wq[i], static_cast<size_t>(d) * d, "Wq"))) break;
    if ((rc = fetch(w->Wk[i], static_cast<size_t>(d) * d, dtype, dev, &tmp, "Wk"))) break;
    for (int j = 0; j < h; ++j)          // WkT[j][c][k] = Wk[k][j*dh + c]
      for (int c = 0; c < dh; ++c)
        for (int k = 0; k < d; ++k)
          slab[o.WkT + (static_cast<size_t>(j) * dh + c) * d + k] = tmp[static_cast<size_t>(k) * d + j * dh + c];
    if ((rc = put(o.Wv, w->Wv[i], static_cast<size_t>(d) * d, "Wv"))) break;
    if ((rc = put(o.Wo, w->Wo[i], static_cast<size_t>(d) * d, "Wo"))) break;
    if (i > 0 && (rc = put(o.Wc, w->Wc[i], static_cast<size_t>(i + 1) * d * d, "Wc"))) break;
  }
  const size_t qlg = lay_off[M], qlb = qlg + d;
  if (rc == STCA_OK) {
    if (w->q_ln_gamma) {
      if (!(rc = put(qlg, w->q_ln_gamma, d, "q_ln_gamma"))) rc = put(qlb, w->q_ln_beta, d, "q_ln_beta");
    } else {
      std::copy(slab.begin() + offs[0].lg, slab.begin() + offs[0].lg + d, slab.begin() + qlg);
      std::copy(slab.begin() + offs[0].lb, slab.begin() + offs[0].lb + d, slab.begin() + qlb);
    }
  }
  if (rc != STCA_OK) { delete H; return rc; }
  if (cudaMalloc(&H->w32, total * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&H->status_d, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    stca_destroy(H);
    return set_error(STCA_ENOMEM, "weight allocation failed");
  }
  if (cudaMemcpy(H->w32, slab.data(), total * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemset(H->status_d, 0, sizeof(int)) != cudaSuccess ||
      cudaEventCreateWithFlags(&H->plan_evt, cudaEventDisableTiming) != cudaSuccess) {
    std::string m = cudaGetErrorString(cudaGetLastError());
    stca_destroy(H);
    return set_error(STCA_ECUDA, "weight upload failed: " + m);
  }
  H->L32.resize(M);
  for (int i = 0; i < M; ++i) {
    const Offs& o = offs[i];
    LayerW32& L = H->L32[i];
    L.Wu = H->w32 + o.Wu; L.Wg = H->w32 + o.Wg; L.Wd = H->w32 + o.Wd;
    L.qWu = H->w32 + o.qWu; L.qWg = H->w32 + o.qWg; L.qWd = H->w32 + o.qWd;
    L.ln_g = H->w32 + o.lg; L.ln_b = H->w32 + o.lb;
    L.Wq = H->w32 + o.Wq; L.WkT = H->w32 + o.WkT;
    L.Wv = H->w32 + o.Wv; L.Wo = H->w32 + o.Wo;
    L.Wc = i > 0 ? H->w32 + o.Wc : nullptr;
  }
  H->q_ln_g = H->w32 + qlg;
  H->q_ln_b = H->w32 + qlb;
  if (cudaDeviceGetAttribute(&H->num_sms, cudaDevAttrMultiProcessorCount, H->device) != cudaSuccess) {
    cudaGetLastError();
    H->num_sms = 148;
  }
  // prediction-head weights of Eq. (9), when given (fp32 host copies)
  std::vector<float> wz, zu, zg, zd;
  HeadHostW hw;
  if (nhead == 4) {
    int rc2 = fetch(w->Wz, static_cast<size_t>(M + 1) * d * d, dtype, dev, &wz, "Wz");
    if (!rc2) rc2 = fetch(w->zWu, static_cast<size_t>(d) * rd, dtype, dev, &zu, "zWu");
    if (!rc2) rc2 = fetch(w->zWg, static_cast<size_t>(d) * rd, dtype, dev, &zg, "zWg");
    if (!rc2) rc2 = fetch(w->zWd, static_cast<size_t>(rd) * d, dtype, dev, &zd, "zWd");
    if (rc2) {
      stca_destroy(H);
      return rc2;
    }
    hw.Wz = wz.data();
    hw.zWu = zu.data();
    hw.zWg = zg.data();
    hw.zWd = zd.data();
  }
  {
    std::vector<StepHostW> sw(M);
    for (int i = 0; i < M; ++i) {
      sw[i].Wq = slab.data() + offs[i].Wq;
      sw[i].Wk = nullptr;
      sw[i].Wv = slab.data() + offs[i].Wv;
      sw[i].Wo = slab.data() + offs[i].Wo;
      sw[i].Wc = i > 0 ? slab.data() + offs[i].Wc : nullptr;
      sw[i].qWu = slab.data() + offs[i].qWu;
      sw[i].qWg = slab.data() + offs[i].qWg;
      sw[i].qWd = slab.data() + offs[i].qWd;
    }
    // W_K in its original [d x d] layout, recovered from the per-head transpose
    std::vector<std::vector<float>> wk(M, std::vector<float>(static_cast<size_t>(d) * d));
    for (int i = 0; i < M; ++i) {
      for (int j = 0; j < h; ++j)
        for (int c = 0; c < dh; ++c)
          for (int k = 0; k < d; ++k)
            wk[i][static_cast<size_t>(k) * d + j * dh + c] =
                slab[offs[i].WkT + (static_cast<size_t>(j) * dh + c) * d + k];
      sw[i].Wk = wk[i].data();
    }
    if (int rc2 = step_weights_setup(H, sw)) {
      stca_destroy(H);
      return rc2;
    }
    if (step_tc_supported(H)) {
      if (int rc2 = step_tc_setup(H, sw, hw)) {
        stca_destroy(H);
        return rc2;
      }
      if (d == 128) {
        // [W_V]^T of every layer (output n = j d_h + c of head j, input k):
        // the B operand of the attention kernel's in-kernel projection
        std::vector<uint16_t> vt(static_cast<size_t>(M) * d * d);
        for (int i = 0; i < M; ++i)
          for (int o = 0; o < d; ++o)
            for (int k = 0; k < d; ++k) {
              uint32_t u;
              memcpy(&u, &sw[i].Wv[static_cast<size_t>(k) * d + o], 4);
              vt[(static_cast<size_t>(i) * d + o) * d + k] = static_cast<uint16_t>(u >> 16);   // bf16-valued
            }
        if (cudaMalloc(&H->wvt, vt.size() * 2) != cudaSuccess ||
            cudaMemcpy(H->wvt, vt.data(), vt.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) {
          cudaGetLastError();
          stca_destroy(H);
          return set_error(STCA_ENOMEM, "W_V upload failed");
        }
        for (int i = 0; i < M; ++i)
          if (int rc2 = make_tmap_bf16_2d(&H->tmWvT[i],
                                          static_cast<const uint16_t*>(H->wvt) + static_cast<size_t>(i) * d * d,
                                          d, d, 64, 128)) {
            stca_destroy(H);
            return rc2;
          }
      }
      if (naive_layout(dh).G > 0 && kv_proj_supported(d)) {
        // naive form (Eq. (12)): [W_K | W_V] of every layer, stored transposed
        // (2d outputs x d inputs, K-major) as the B operand of the projection
        std::vector<uint16_t> kvw(static_cast<size_t>(M) * 2 * d * d);
        auto bf = [](float f) {
          uint32_t u;
          memcpy(&u, &f, 4);
          return static_cast<uint16_t>(u >> 16);     // bf16-valued already
        };
        for (int i = 0; i < M; ++i)
          for (int o = 0; o < 2 * d; ++o)
            for (int k = 0; k < d; ++k)
              kvw[(static_cast<size_t>(i) * 2 * d + o) * d + k] =
                  bf(o < d ? sw[i].Wk[static_cast<size_t>(k) * d + o] : sw[i].Wv[static_cast<size_t>(k) * d + o - d]);
        if (cudaMalloc(&H->wkv, kvw.size() * 2) != cudaSuccess ||
            cudaMemcpy(H->wkv, kvw.data(), kvw.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) {
          cudaGetLastError();
          stca_destroy(H);
          return set_error(STCA_ENOMEM, "naive-form weight upload failed");
        }
        for (int i = 0; i < M; ++i)
          if (int rc2 = make_tmap_bf16_2d(&H->tmWkv[i],
                                          static_cast<const uint16_t*>(H->wkv) + static_cast<size_t>(i) * 2 * d * d,
                                          d, 2 * d, 64, 256)) {
            stca_destroy(H);
            return rc2;
          }
      }
    }
  }
  if (nhead == 4) {
    if (int rc2 = head_weights_setup(H, wz.data(), zu.data(), zg.data(), zd.data())) {
      stca_destroy(H);
      return rc2;
    }
    // fp32 copies for the backward of Eq. (9): Wz, zWu, zWg, zWd back to back
    const size_t n[4] = {wz.size(), zu.size(), zg.size(), zd.size()};
    const float* src[4] = {wz.data(), zu.data(), zg.data(), zd.data()};
    if (cudaMalloc(&H->w32head, (n[0] + n[1] + n[2] + n[3]) * sizeof(float)) != cudaSuccess) {
      cudaGetLastError();
      stca_destroy(H);
      return set_error(STCA_ENOMEM, "prediction-head weight allocation failed");
    }
    const float* part[4];
    size_t at = 0;
    for (int k = 0; k < 4; ++k) {
      part[k] = H->w32head + at;
      if (cudaMemcpy(H->w32head + at, src[k], n[k] * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaGetLastError();
        stca_destroy(H);
        return set_error(STCA_ECUDA, "prediction-head weight upload failed");
      }
      at += n[k];
    }
    H->hWz32 = part[0];
    H->hWu32 = part[1];
    H->hWg32 = part[2];
    H->hWd32 = part[3];
  }
  if (dtype == STCA_BF16 && encode_tc_supported(d, rd)) {
    std::vector<const float*> Wu(M), Wg(M), Wd(M);
    for (int i = 0; i < M; ++i) {
      Wu[i] = slab.data() + offs[i].Wu;
      Wg[i] = slab.data() + offs[i].Wg;
      Wd[i] = slab.data() + offs[i].Wd;
    }
    if (int rc2 = encode_tc_setup(H, Wu, Wg, Wd)) {
      stca_destroy(H);
      return rc2;
    }
  }
  *out = H;
  return ok();
}

// ------------------------------------------------------------------ encode

// Checks, the handle's encoded-state bookkeeping and the X~ tensor maps of an
// encode of N rows (the launches follow).
static int encode_begin(stca_handle* H, const void* X, const int64_t* offsets, int64_t R, int64_t N) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (!X) return set_error(STCA_EINVAL, "X is NULL");
  if (reinterpret_cast<uintptr_t>(X) % 16) return set_error(STCA_EINVAL, "X must be 16-byte aligned");
  if (N < 1) return set_error(STCA_EINVAL, "N must be >= 1");
  if (int rc = validate_offsets(offsets, R, N, true, "offsets")) return rc;
  const size_t layer_bytes = static_cast<size_t>(N) * H->d * H->elem;
  if (int rc = ensure_dev(&H->xt, &H->xt_cap, layer_bytes * H->M)) return rc;
  H->encoded = false;
  H->R = R;
  H->N = N;
  // the attention plan depends on the key layout: a batch with other offsets
  // needs a new one, the same layout keeps the one on the device (no upload
  // between the encoder and the forward's first launch)
  if (H->offsets_h.size() != static_cast<size_t>(R + 1) ||
      !std::equal(H->offsets_h.begin(), H->offsets_h.end(), offsets))
    H->last_toff.clear();
  H->offsets_h.assign(offsets, offsets + R + 1);
  H->launches = 0;
  if (H->dtype == STCA_BF16 && attn_tc_supported(H->d)) {
    for (int i = 0; i < H->M; ++i)
      if (int rc = make_tmap_bf16_2d(&H->tmXt[i], static_cast<char*>(H->xt) + layer_bytes * i,
                                     H->d, N, 64, 128))
        return rc;
  }
  if (H->opt_encode_path == 2 && !H->tc_encode_ready)
    return set_error(STCA_EINVAL, "tensor-core encoder needs bf16 and d in {64,128,256}, rd % 64 == 0");
  return STCA_OK;
}

static bool encode_on_tensor_cores(const stca_handle* H) {
  return H->tc_encode_ready && H->opt_encode_path != 1;
}

extern "C" int stca_encode(stca_handle* H, const void* X, const int64_t* offsets, int64_t R,
                           int64_t N, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  DeviceGuard g(H->device);
  if (!g.ok) return set_error(STCA_ECUDA, "cannot select the handle's device");
  if (int rc = encode_begin(H, X, offsets, R, N)) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t layer_bytes = static_cast<size_t>(N) * H->d * H->elem;
  const bool bf = H->dtype == STCA_BF16;
  if (encode_on_tensor_cores(H)) {
    int rc;
    {
      TimedLaunch tl(H, STCA_K_ENCODE, s);
      rc = launch_encode_tc(H, X, N, s);
    }
    if (rc) return rc;
    H->launches++;
    if (int rc2 = check_launch("encode (tensor cores)")) return rc2;
  } else {
    for (int i = 0; i < H->M; ++i) {
      void* xti = static_cast<char*>(H->xt) + layer_bytes * i;
      {
        TimedLaunch tl(H, STCA_K_ENCODE, s);
        launch_ffn_rows(X, bf, N, H->L32[i], true, H->L32[i].ln_g, H->L32[i].ln_b, xti, bf,
                        H->d, H->rd, s);
      }
      H->launches++;
      if (int rc = check_launch("encode")) return rc;
    }
  }
  H->encoded = true;
  return ok();
}

// ------------------------------------------------------------------ forward
static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Attention path of a forward: 2 tensor cores, 1 CUDA cores.
static int attn_path(const stca_handle* H) {
  const bool tc = H->dtype == STCA_BF16 && attn_tc_supported(H->d);
  if (H->opt_attn_path == 1) return 1;
  if (H->opt_attn_path == 2) return tc ? 2 : -1;
  return tc ? 2 : 1;
}

// Cut the attention of one forward into work items.
//  CUDA cores (path 1): each request's keys cut into ranges of at most `split`
//    keys (by default 1024, or down to 128 for small batches so that the grid
//    has two entries per CTA); one item per range covers all T_r * h query
//    rows; the kernel grid is the list of (item, target) pairs.
//  Tensor cores (path 2): (request, 128-row query tile) pairs, each over all
//    its key tiles, laid end to end and cut into runs of equal numbers of key
//    tiles, one run per CTA (stream-K); every maximal run inside one pair is
//    an item.  `split`, when set, caps a run at split/128 key tiles.
NaiveLayout stca::naive_layout(int dh) {
  NaiveLayout L;
  if (dh == 16 || dh == 32 || dh == 64) {
    L.G = 64 / dh;
    L.Tq = 128 / L.G;
  }
  return L;
}

void stca::build_plan_host(const int64_t* off, const int64_t* toff, int64_t R, int h, int path,
                            int num_ctas, int64_t split_keys, PlanHost& P, int dh, int simt_rows) {
  P = PlanHost();
  P.req_pair_begin.assign(R + 1, 0);
  auto& items = P.items;
  int64_t& G = P.G;
  if (path == 1) {
    // default: 1024 keys, or shorter ranges (down to 128) when that leaves
    // fewer than two (item, target) grid entries per CTA
    int64_t split = split_keys;
    if (split <= 0) {
      int64_t work = 0;                 // key-target pairs
      for (int64_t r = 0; r < R; ++r) work += (toff[r + 1] - toff[r]) * (off[r + 1] - off[r]);
      const int64_t per = (work + 2 * num_ctas - 1) / (2 * std::max(num_ctas, 1));
      split = std::min<int64_t>(1024, std::max<int64_t>(128, (per + 127) / 128 * 128));
    }
    for (int64_t r = 0; r < R; ++r) {
      P.req_pair_begin[r] = static_cast<int32_t>(r);
      P.pair_item_begin.push_back(static_cast<int32_t>(items.size()));
      const int64_t Tr = toff[r + 1] - toff[r];
      for (int64_t k0 = off[r]; k0 < off[r + 1]; k0 += split) {
        AttnItem it{};
        it.req = static_cast<int32_t>(r);
        it.nkeys = static_cast<int32_t>(std::min<int64_t>(split, off[r + 1] - k0));
        it.key0 = k0;
        it.row_base = G;
        it.qrow0 = toff[r] * h;
        it.mt = 0;
        it.rows = static_cast<int32_t>(Tr * h);
        it.pair = static_cast<int32_t>(r);
        G += Tr * h;
        for (int64_t row0 = 0; row0 < Tr * h; row0 += std::max(simt_rows, 1)) {
          P.pairs_simt.push_back(static_cast<int32_t>(items.size()));
          P.pairs_simt.push_back(static_cast<int32_t>(row0));
        }
        items.push_back(it);
      }
    }
    P.req_pair_begin[R] = static_cast<int32_t>(R);
    P.pair_item_begin.push_back(static_cast<int32_t>(items.size()));
    return;
  }
  // path 2: a request's T_r h query rows in tiles of 128; path 3 (naive form):
  // (h / G) nslots tiles of 128 rows each (NaiveLayout)
  const NaiveLayout NL = naive_layout(dh);
  auto tiles_of = [&](int64_t r) -> int64_t {
    const int64_t Tr = toff[r + 1] - toff[r];
    if (path == 3) return Tr == 0 ? 0 : (h / NL.G) * ((Tr + NL.Tq - 1) / NL.Tq);
    return (Tr * h + 127) / 128;
  };
  struct Pair { int64_t r, mt, ntiles; };
  std::vector<Pair> pairs;
  int64_t W = 0;
  if (path == 3) P.qbase.assign(R + 1, 0);
  for (int64_t r = 0; r < R; ++r) {
    P.req_pair_begin[r] = static_cast<int32_t>(pairs.size());
    const int64_t nt = (off[r + 1] - off[r] + 127) / 128;
    const int64_t ntile = tiles_of(r);
    for (int64_t mt = 0; mt < ntile; ++mt) {
      pairs.push_back({r, mt, nt});
      W += nt;
    }
    if (path == 3) P.qbase[r + 1] = P.qbase[r] + 128 * ntile;
  }
  if (path == 3) P.qrows = P.qbase[R];
  P.req_pair_begin[R] = static_cast<int32_t>(pairs.size());
  int64_t cs = (W + num_ctas - 1) / std::max(num_ctas, 1);      // key tiles per CTA
  if (split_keys > 0) cs = std::min<int64_t>(cs, std::max<int64_t>(1, split_keys / 128));
  cs = std::max<int64_t>(cs, 1);
  P.grid = static_cast<int>((W + cs - 1) / cs);
  P.cta_begin.assign(P.grid + 1, 0);
  int64_t cursor = 0;     // global key-tile index of the pair's first tile
  int next_cta = 0;
  for (size_t pi = 0; pi < pairs.size(); ++pi) {
    const Pair& pr = pairs[pi];
    P.pair_item_begin.push_back(static_cast<int32_t>(items.size()));
    const int64_t L = off[pr.r + 1] - off[pr.r];
    const int64_t rows = path == 3 ? 128
                                   : std::min<int64_t>(128, (toff[pr.r + 1] - toff[pr.r]) * h - pr.mt * 128);
    int64_t a = 0;
    while (a < pr.ntiles) {
      const int64_t g0 = cursor + a;
      const int64_t b = std::min<int64_t>(pr.ntiles, (g0 / cs + 1) * cs - cursor);
      while (next_cta <= g0 / cs) P.cta_begin[next_cta++] = static_cast<int32_t>(items.size());
      AttnItem it{};
      it.req = static_cast<int32_t>(pr.r);
      it.key0 = off[pr.r] + a * 128;
      it.nkeys = static_cast<int32_t>(std::min<int64_t>(b * 128, L) - a * 128);
      it.row_base = G;
      it.mt = static_cast<int32_t>(pr.mt);
      it.rows = static_cast<int32_t>(rows);
      it.pair = static_cast<int32_t>(pi);
      if (path == 3) {
        const int64_t nslots = (toff[pr.r + 1] - toff[pr.r] + NL.Tq - 1) / NL.Tq;
        it.qrow0 = P.qbase[pr.r] + pr.mt * 128;
        it.kcol = static_cast<int32_t>((pr.mt / nslots) * 64);
      } else {
        it.qrow0 = toff[pr.r] * h + pr.mt * 128;
      }
      G += rows;
      items.push_back(it);
      a = b;
    }
    cursor += pr.ntiles;
  }
  while (next_cta <= P.grid) P.cta_begin[next_cta++] = static_cast<int32_t>(items.size());
  P.pair_item_begin.push_back(static_cast<int32_t>(items.size()));
}

// Invariants every kernel relies on for in-bounds access; a violation is a
// library bug and is reported instead of launched.
int stca::check_plan(const PlanHost& P, const int64_t* off, const int64_t* toff, int64_t R,
                      int h, int path) {
  const int64_t N = off[R], T = toff[R];
  auto bad = [](const std::string& m) { return set_error(STCA_EINVAL, "internal plan check: " + m); };
  if (path == 3 && static_cast<int64_t>(P.qbase.size()) != R + 1) return bad("naive query layout");
  int64_t rows_sum = 0;
  for (size_t w = 0; w < P.items.size(); ++w) {
    const AttnItem& it = P.items[w];
    if (it.req < 0 || it.req >= R) return bad("request index");
    if (it.nkeys < 1 || it.key0 < off[it.req] || it.key0 + it.nkeys > off[it.req + 1])
      return bad("key range outside its request");
    if (it.rows < 0 || it.row_base != rows_sum) return bad("partial rows not contiguous");
    rows_sum += it.rows;
    const int64_t req_rows = (toff[it.req + 1] - toff[it.req]) * h;
    if (path == 3) {
      const int64_t ntile = P.req_pair_begin[it.req + 1] - P.req_pair_begin[it.req];
      if (it.rows != 128 || it.mt < 0 || it.mt >= ntile ||
          it.qrow0 != P.qbase[it.req] + int64_t(it.mt) * 128 || it.qrow0 + 128 > P.qrows ||
          it.kcol < 0 || it.kcol % 64 != 0 || it.kcol + 64 > int64_t(h) * 64)
        return bad("naive query tile");
    } else if (path == 2) {
      if (it.rows < 1 || it.rows > 128 || int64_t(it.mt) * 128 + it.rows > req_rows ||
          it.qrow0 != toff[it.req] * h + int64_t(it.mt) * 128 || it.qrow0 + it.rows > T * h)
        return bad("query tile");
    } else if (it.rows != req_rows) {
      return bad("query rows");
    }
  }
  if (rows_sum != P.G) return bad("partial row count");
  if (static_cast<int64_t>(P.req_pair_begin.size()) != R + 1) return bad("request pairs");
  const int64_t npairs = static_cast<int64_t>(P.pair_item_begin.size()) - 1;
  if (P.req_pair_begin[R] != npairs) return bad("pair count");
  for (int64_t p = 0; p < npairs; ++p)
    if (P.pair_item_begin[p] > P.pair_item_begin[p + 1]) return bad("pair items");
  if (P.pair_item_begin[npairs] != static_cast<int32_t>(P.items.size())) return bad("pair end");
  if (path >= 2)
    for (int64_t p = 0; p < npairs; ++p)
      for (int32_t w = P.pair_item_begin[p]; w < P.pair_item_begin[p + 1]; ++w)
        if (P.items[w].pair != p) return bad("item's pair index");
  for (int64_t r = 0; r < R; ++r) {
    const int64_t rows = (toff[r + 1] - toff[r]) * h;
    const int64_t want = path == 2 ? (rows + 127) / 128 : path == 3 ? (P.qbase[r + 1] - P.qbase[r]) / 128 : 1;
    if (P.req_pair_begin[r + 1] - P.req_pair_begin[r] != want) return bad("pairs of a request");
    for (int32_t p = P.req_pair_begin[r]; p < P.req_pair_begin[r + 1]; ++p) {
      // the pair's items cover the request's keys exactly once, in order
      int64_t k = off[r];
      for (int32_t w = P.pair_item_begin[p]; w < P.pair_item_begin[p + 1]; ++w) {
        if (P.items[w].req != r || P.items[w].key0 != k) return bad("key coverage");
        k += P.items[w].nkeys;
      }
      if (rows > 0 && k != off[r + 1]) return bad("keys not covered");
    }
  }
  if (path >= 2) {
    if (static_cast<int>(P.cta_begin.size()) != P.grid + 1 || P.cta_begin[0] != 0 ||
        P.cta_begin[P.grid] != static_cast<int32_t>(P.items.size()))
      return bad("CTA ranges");
    for (int c = 0; c < P.grid; ++c)
      if (P.cta_begin[c] > P.cta_begin[c + 1]) return bad("CTA ranges order");
  } else {
    for (size_t q = 0; q < P.pairs_simt.size(); q += 2) {
      const int32_t w = P.pairs_simt[q], row0 = P.pairs_simt[q + 1];
      if (w < 0 || w >= static_cast<int32_t>(P.items.size()) || row0 < 0 || row0 >= P.items[w].rows)
        return bad("(item, query row block) pair");
    }
  }
  (void)N;
  return STCA_OK;
}

// The two-half pipeline's plan: requests [0, RA) and [RA, R) split at about
// half of the attention work (key tiles x query tiles), each half planned for
// the SMs its attention leaves to the other half's per-target step (16
// targets per CTA), both checked, then joined into one plan: half B's items,
// pairs and partial rows follow half A's, and its CTA runs follow A's
// grid + 1 entries of cta_begin.  False when it does not apply (a half would
// be empty, or a pair would have more items than the step merges) or does not
// pay: every pipelined launch holds a per-target step, whose latency (about
// 20 key tiles of attention per SM) the other half's attention must cover, so
// a batch with less than kPipeMinWork key tiles x query tiles per SM runs in
// one piece (measured: the pipeline slowed a 32-request batch of 200..2000 keys
// by half, and left the 64 x 10000-key serving batch, 34 per SM, even).
constexpr int64_t kPipeMinWork = 24;
static bool build_pipe_plan(stca_handle* H, const int64_t* off, const int64_t* toff, int64_t R,
                            PlanHost& P) {
  const int h = H->h;
  if (R < 2) return false;
  std::vector<int64_t> work(R + 1, 0);
  for (int64_t r = 0; r < R; ++r)
    work[r + 1] = work[r] + ((toff[r + 1] - toff[r]) * h + 127) / 128 * ((off[r + 1] - off[r] + 127) / 128);
  if (work[R] < kPipeMinWork * H->num_sms) return false;
  int64_t RA = 1;
  while (RA < R - 1 && 2 * work[RA] < work[R]) ++RA;
  const int64_t TA = toff[RA], T = toff[R];
  if (TA <= 0 || TA >= T) return false;
  const int nstepA = static_cast<int>((TA + 15) / 16), nstepB = static_cast<int>((T - TA + 15) / 16);
  const int ctasA = H->num_sms - nstepB, ctasB = H->num_sms - nstepA;
  if (ctasA < H->num_sms / 4 || ctasB < H->num_sms / 4) return false;
  PlanHost A, B;
  build_plan_host(off, toff, RA, h, 2, ctasA, H->opt_split_keys, A, H->dh, 0);
  build_plan_host(off + RA, toff + RA, R - RA, h, 2, ctasB, H->opt_split_keys, B, H->dh, 0);
  if (check_plan(A, off, toff, RA, h, 2) || check_plan(B, off + RA, toff + RA, R - RA, h, 2)) {
    set_error(STCA_OK, "");
    return false;
  }
  for (const PlanHost* X : {&A, &B})
    for (size_t k = 0; k + 1 < X->pair_item_begin.size(); ++k)
      if (X->pair_item_begin[k + 1] - X->pair_item_begin[k] > kQslots) return false;
  const int32_t nA = static_cast<int32_t>(A.items.size()), pA = static_cast<int32_t>(A.req_pair_begin[RA]);
  P = PlanHost();
  P.items = A.items;
  for (AttnItem it : B.items) {
    it.req += static_cast<int32_t>(RA);
    it.pair += pA;
    it.row_base += A.G;
    P.items.push_back(it);
  }
  P.cta_begin = A.cta_begin;
  for (int32_t c : B.cta_begin) P.cta_begin.push_back(c + nA);
  P.req_pair_begin.assign(A.req_pair_begin.begin(), A.req_pair_begin.end());
  for (int64_t r = 1; r <= R - RA; ++r) P.req_pair_begin.push_back(B.req_pair_begin[r] + pA);
  P.pair_item_begin = A.pair_item_begin;
  for (size_t k = 1; k < B.pair_item_begin.size(); ++k) P.pair_item_begin.push_back(B.pair_item_begin[k] + nA);
  P.G = A.G + B.G;
  P.grid = A.grid + B.grid;
  H->pipe_RA = RA;
  H->pipe_TA = TA;
  H->pipe_gridA = A.grid;
  H->pipe_gridB = B.grid;
  return true;
}

// Build (or reuse) the plan for the targets layout `toff` and upload it; with
// pipe, the two-half pipeline's plan where it applies (H->last_pipe says).
static int build_plan(stca_handle* H, const int64_t* toff, int64_t T, int path, cudaStream_t s,
                      bool pipe = false) {
  const int64_t R = H->R;
  if (path == H->last_path && pipe == H->last_pipe_asked && !H->last_toff.empty() &&
      static_cast<int64_t>(H->last_toff.size()) == R + 1 &&
      std::equal(H->last_toff.begin(), H->last_toff.end(), toff))
    return STCA_OK;   // same layout as the previous forward on this encode: plan is on device
  const int64_t* off = H->offsets_h.data();
  PlanHost P;
  H->last_pipe = pipe && path == 2 && build_pipe_plan(H, off, toff, R, P);
  if (!H->last_pipe) {
    build_plan_host(off, toff, R, H->h, path, H->num_sms, H->opt_split_keys, P, H->dh,
                    attn_simt_rows_per_cta(H->d));
    if (int rc = check_plan(P, off, toff, R, H->h, path)) return rc;
  }
  const auto& items = P.items;
  const auto& pairs_simt = P.pairs_simt;
  const auto& cta_begin = P.cta_begin;
  const auto& req_pair_begin = P.req_pair_begin;
  const auto& pair_item_begin = P.pair_item_begin;
  const int64_t G = P.G;
  const int grid = P.grid;
  const size_t n_items = items.size();
  H->off_items = 0;
  H->off_pairs = align256(H->off_items + n_items * sizeof(AttnItem));
  H->off_cta = align256(H->off_pairs + pairs_simt.size() * sizeof(int32_t));
  H->off_treq = align256(H->off_cta + cta_begin.size() * sizeof(int32_t));
  H->off_toff = align256(H->off_treq + static_cast<size_t>(T) * sizeof(int32_t));
  H->off_rpb = align256(H->off_toff + static_cast<size_t>(R + 1) * sizeof(int64_t));
  H->off_pib = align256(H->off_rpb + static_cast<size_t>(R + 1) * sizeof(int32_t));
  H->off_qbase = align256(H->off_pib + pair_item_begin.size() * sizeof(int32_t));
  const size_t bytes = align256(H->off_qbase + P.qbase.size() * sizeof(int64_t));
  // pinned staging: wait until the previous upload has left it
  if (H->plan_h && cudaEventSynchronize(H->plan_evt) != cudaSuccess)
    return set_error(STCA_ECUDA, "plan event wait failed");
  if (bytes > H->plan_h_cap) {
    if (H->plan_h) cudaFreeHost(H->plan_h);
    H->plan_h = nullptr;
    H->plan_h_cap = 0;
    if (cudaMallocHost(&H->plan_h, bytes) != cudaSuccess) {
      cudaGetLastError();
      H->plan_h = nullptr;
      return set_error(STCA_ENOMEM, "pinned plan buffer allocation failed");
    }
    H->plan_h_cap = bytes;
  }
  if (int rc = ensure_dev(&H->plan_d, &H->plan_cap, bytes)) return rc;
  char* p = static_cast<char*>(H->plan_h);
  memcpy(p + H->off_items, items.data(), n_items * sizeof(AttnItem));
  memcpy(p + H->off_pairs, pairs_simt.data(), pairs_simt.size() * sizeof(int32_t));
  memcpy(p + H->off_cta, cta_begin.data(), cta_begin.size() * sizeof(int32_t));
  int32_t* treq = reinterpret_cast<int32_t*>(p + H->off_treq);
  for (int64_t r = 0; r < R; ++r)
    for (int64_t t = toff[r]; t < toff[r + 1]; ++t) treq[t] = static_cast<int32_t>(r);
  memcpy(p + H->off_toff, toff, static_cast<size_t>(R + 1) * sizeof(int64_t));
  memcpy(p + H->off_rpb, req_pair_begin.data(), static_cast<size_t>(R + 1) * sizeof(int32_t));
  memcpy(p + H->off_pib, pair_item_begin.data(), pair_item_begin.size() * sizeof(int32_t));
  if (!P.qbase.empty()) memcpy(p + H->off_qbase, P.qbase.data(), P.qbase.size() * sizeof(int64_t));
  H->last_qrows = P.qrows;
  STCA_CUDA_TRY(cudaMemcpyAsync(H->plan_d, H->plan_h, bytes, cudaMemcpyHostToDevice, s));
  STCA_CUDA_TRY(cudaEventRecord(H->plan_evt, s));
  H->last_G = G;
  H->last_npairs = static_cast<int64_t>(pair_item_begin.size()) - 1;
  H->last_pairs = static_cast<int64_t>(pairs_simt.size() / 2);
  H->last_max_items = 0;
  for (size_t k = 0; k + 1 < pair_item_begin.size(); ++k)
    H->last_max_items = std::max(H->last_max_items, pair_item_begin[k + 1] - pair_item_begin[k]);
  H->last_grid = grid;
  H->last_path = path;
  H->last_pipe_asked = pipe;
  H->last_toff.assign(toff, toff + R + 1);
  return STCA_OK;
}

// Naive form, Eq. (12): K = X~(layer+1) W_K and V = X~(layer+1) W_V for every
// history row at once, into H->kv (row n: [K_n | V_n], bf16), by the
// tensor-core projection kernel (kv_proj.cu).
static int kv_project(stca_handle* H, int layer, cudaStream_t s) {
  return launch_kv_proj(H->d, H->tmXt[layer], H->tmWkv[layer], static_cast<uint16_t*>(H->kv), H->N,
                        H->num_sms, H->status_d, s);
}

// FLOPs of one layer's attention in either form: the reordered form contracts
// d features for each of the T_r h query rows; the naive form projects K and V
// (4 L d^2) and then contracts the tile's 64 head-group features for the
// padded query rows of its layout.
static bool naive_cheaper(const stca_handle* H, const int64_t* toff) {
  const NaiveLayout NL = naive_layout(H->dh);
  double re = 0, nv = 0;
  const double d = H->d, h = H->h;
  for (int64_t r = 0; r < H->R; ++r) {
    const double L = static_cast<double>(H->offsets_h[r + 1] - H->offsets_h[r]);
    const int64_t Tr = toff[r + 1] - toff[r];
    re += 4.0 * Tr * h * L * d;
    const double rows = Tr == 0 ? 0.0 : 128.0 * (h / NL.G) * ((Tr + NL.Tq - 1) / NL.Tq);
    nv += 4.0 * L * d * d + 4.0 * rows * L * 64.0;
  }
  return nv < re;
}

// The forward of stca_forward; with zout, also the prediction-head token of
// Eq. (9), inside the last per-target step when that runs on the tensor cores,
// else by the separate head kernel after it.
// after_encode: the call directly follows this library's encoder launch on
// the stream (stca_encode_forward, stca_run_host), so the two-half pipeline's
// query init may overlap the encoder's last round of tiles.
static int forward_impl(stca_handle* H, const void* targets, const int64_t* target_offsets,
                        int64_t T, float* Z, float* zout, void* stream, bool after_encode = false) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (!H->encoded) return set_error(STCA_ESTATE, "stca_forward before a successful stca_encode");
  if (T < 0) return set_error(STCA_EINVAL, "T must be >= 0");
  if (int rc = validate_offsets(target_offsets, H->R, T, false, "target_offsets")) return rc;
  if (T == 0) return ok();
  if (!targets || !Z) return set_error(STCA_EINVAL, "targets or Z is NULL");
  if (reinterpret_cast<uintptr_t>(targets) % 16 || reinterpret_cast<uintptr_t>(Z) % 16)
    return set_error(STCA_EINVAL, "targets and Z must be 16-byte aligned");
  DeviceGuard g(H->device);
  if (!g.ok) return set_error(STCA_ECUDA, "cannot select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int path = attn_path(H);
  if (path < 0)
    return set_error(STCA_EINVAL, "tensor-core attention needs bf16 and d in {64, 128, 256}");
  if (path == 1 && attn_simt_smem(H) > 227 * 1024)
    return set_error(STCA_EINVAL, "h * d too large for the CUDA-core attention kernel");
  // attention form: the reordered Eq. (13) unless the naive Eq. (12) is asked for
  const NaiveLayout NL = naive_layout(H->dh);
  const bool naive_ok = path == 2 && H->step_tc_ready && H->opt_step_path != 1 && NL.G > 0 &&
                        H->wkv != nullptr;
  if (H->opt_attn_form == 1 && !naive_ok)
    return set_error(STCA_EINVAL, "the naive attention form needs the tensor-core attention and step "
                                  "(bf16, d in {128, 256}, r d <= 512) and d_h in {16, 32, 64}");
  const bool naive = naive_ok && (H->opt_attn_form == 1 ||
                                  (H->opt_attn_form == 2 && naive_cheaper(H, target_offsets)));
  H->last_naive = naive;
  // the two-half pipeline (STCA_OPT_PIPELINE): the reordered form on the
  // tensor cores with the in-kernel W_V projection and the step's merge
  const bool want_pipe = !naive && path == 2 && H->opt_pipeline == 1 && zout == nullptr &&
                         H->step_tc_ready && H->opt_step_path != 1 && H->opt_attn_kernel == 0 &&
                         attn_tc_proj_supported(H);
  if (int rc = build_plan(H, target_offsets, T, naive ? 3 : path, s, want_pipe)) return rc;
  const int d = H->d, h = H->h;
  const size_t urows = static_cast<size_t>(T) * h;
  if (naive) {
    const size_t qrows = static_cast<size_t>(H->last_qrows);
    if (int rc = ensure_dev(reinterpret_cast<void**>(&H->Ubf), &H->Ubf_cap, std::max<size_t>(qrows, 1) * 128))
      return rc;
    if (int rc = make_tmap_bf16_2d(&H->tmU, H->Ubf, 64, qrows, 64, 128)) return rc;
    if (int rc = ensure_dev(&H->kv, &H->kv_cap, static_cast<size_t>(H->N) * 4 * d)) return rc;
    if (int rc = make_tmap_bf16_2d_strided(&H->tmKn, H->kv, d, H->N, 4 * d, 64, 128)) return rc;
    if (int rc = make_tmap_bf16_2d_strided(&H->tmVn, static_cast<char*>(H->kv) + 2 * d, d, H->N, 4 * d,
                                           64, 128))
      return rc;
    STCA_CUDA_TRY(cudaMemsetAsync(H->Ubf, 0, qrows * 128, s));   // padding rows stay zero
  } else if (path == 1) {
    if (int rc = ensure_dev(reinterpret_cast<void**>(&H->U), &H->U_cap, urows * d * sizeof(float)))
      return rc;
  } else {
    if (int rc = ensure_dev(reinterpret_cast<void**>(&H->Ubf), &H->Ubf_cap, urows * d * 2)) return rc;
    if (int rc = make_tmap_bf16_2d(&H->tmU, H->Ubf, d, urows, 64, 128)) return rc;
  }
  // the two-group kernel (d <= 128, reordered form) merges the split
  // partials itself, counting arrivals per pair and layer
  const bool pp = path == 2 && !naive && attn_pp_supported(d) && H->opt_attn_kernel == 2;
  // the split partials: G item rows of d (naive form: 64) floats plus (m, l);
  // or, with the in-kernel projection, kQslots slots of d_h + 2 floats per
  // query row plus its item count
  const size_t part_floats =
      std::max(static_cast<size_t>(std::max<int64_t>(H->last_G, 1)) * ((naive ? 64 : d) + 4),
               urows * (kQslots * (static_cast<size_t>(H->dh) + 2) + 1));
  if (int rc = ensure_dev(reinterpret_cast<void**>(&H->part), &H->part_cap, part_floats * sizeof(float)))
    return rc;
  const size_t cnt_per_layer = static_cast<size_t>(std::max<int64_t>(H->last_npairs, 1)) * 8;
  if (pp) {
    if (int rc = ensure_dev(reinterpret_cast<void**>(&H->attn_cnt), &H->attn_cnt_cap,
                            cnt_per_layer * H->M * sizeof(int)))
      return rc;
    STCA_CUDA_TRY(cudaMemsetAsync(H->attn_cnt, 0, cnt_per_layer * H->M * sizeof(int), s));
  }
  if (int rc = ensure_dev(reinterpret_cast<void**>(&H->cbuf), &H->cbuf_cap, urows * d * sizeof(float)))
    return rc;
  char* p = static_cast<char*>(H->plan_d);
  const AttnItem* items_d = reinterpret_cast<const AttnItem*>(p + H->off_items);
  const int32_t* pairs_d = reinterpret_cast<const int32_t*>(p + H->off_pairs);
  const int32_t* cta_d = reinterpret_cast<const int32_t*>(p + H->off_cta);
  StepPlan plan;
  plan.treq = reinterpret_cast<const int32_t*>(p + H->off_treq);
  plan.toff = reinterpret_cast<const int64_t*>(p + H->off_toff);
  plan.req_pair_begin = reinterpret_cast<const int32_t*>(p + H->off_rpb);
  plan.pair_item_begin = reinterpret_cast<const int32_t*>(p + H->off_pib);
  plan.items = items_d;
  plan.mtile_rows = path == 2 ? 128 : (1 << 30);
  plan.log2_partials = path == 2 ? 1 : 0;
  const size_t layer_bytes = static_cast<size_t>(H->N) * d * H->elem;
  // per-target step: tensor cores when the attention is (their query units)
  if (H->opt_step_path == 2 && !(path == 2 && H->step_tc_ready))
    return set_error(STCA_EINVAL, "tensor-core step needs the tensor-core attention, bf16, "
                                  "d in {128, 256} and r d <= 512");
  const bool step_tc = path == 2 && H->step_tc_ready && H->opt_step_path != 1;
  // proj: the attention kernel projects its rows by W_V itself (o_j = alpha_j
  // X~ W_V^j, Eqs. (6), (13)), so partials are d_h wide and the step starts
  // from o_head; STCA_OPT_ATTN_KERNEL = 1 keeps the unprojected rows c_j
  const bool proj = path == 2 && !naive && !pp && step_tc && H->opt_attn_kernel == 0 &&
                    attn_tc_proj_supported(H);
  // the tensor-core step merges the split partials itself when every query
  // tile has few enough items; otherwise combine_kernel merges them first
  const bool fused = !naive && !pp && step_tc &&
                     H->last_max_items <= (proj ? step_tc_max_items_proj() : step_tc_max_items()) &&
                     H->last_G < (int64_t(1) << 31);
  const int proj_mode = proj ? (fused ? 2 : 1) : 0;
  // proj with the step's merge: partials in per-row slots (fused implies at
  // most step_tc_max_items_proj() = kQslots items per pair)
  QslotBufs qs{};
  if (proj_mode == 2) {
    qs.pair_item_begin = plan.pair_item_begin;
    qs.pacc = H->part;
    qs.qml = H->part + urows * kQslots * H->dh;
    qs.qn = reinterpret_cast<int*>(qs.qml + urows * kQslots * 2);
  }
  NaiveStep ns{NL.G, NL.Tq, reinterpret_cast<const int64_t*>(p + H->off_qbase), H->Ubf};
  const bool head_in_step = zout && step_tc && H->head_tc;
  auto step = [&](int layer, const float* cm) {
    if (step_tc)
      return launch_step_tc(H, layer, targets, T, fused ? nullptr : cm, &plan, H->part, H->last_G,
                            Z, H->Ubf, s, naive ? &ns : nullptr,
                            head_in_step && layer == H->M - 1 ? zout : nullptr, layer >= 0 ? proj_mode : 0,
                            proj_mode == 2 ? &qs : nullptr);
    launch_target_step(H, layer, targets, T, plan, cm, Z, s);
    return static_cast<int>(STCA_OK);
  };
  if (H->last_pipe) {
    // Two halves, A = targets [0, TA), B = [TA, T): A's query init alone, then
    // per layer i one launch of A's attention beside B's step i - 1 (the query
    // init for i = 0) and one of B's attention beside A's step i, then B's
    // last step alone.  Each launch's two parts are independent; each part
    // depends only on the previous launch.
    if (proj_mode != 2) return set_error(STCA_EINVAL, "internal: pipeline plan without the projected merge");
    const int64_t TA = H->pipe_TA, TB = T - TA, M = H->M, dh = H->dh;
    const uint16_t* tg = static_cast<const uint16_t*>(targets);
    auto half_qs = [&](int64_t t0) {
      QslotBufs q = qs;
      q.pacc += t0 * h * kQslots * dh;
      q.qml += t0 * h * kQslots * 2;
      q.qn += t0 * h;
      return q;
    };
    PipeStep sA{0, tg, TA, Z, H->Ubf, half_qs(0)};
    PipeStep sB{0, tg + TA * d, TB, Z + TA * M * d, H->Ubf + TA * h * d, half_qs(TA)};
    PipeAttn aA{0, items_d, cta_d, H->pipe_gridA, qs};
    PipeAttn aB{0, items_d, cta_d + H->pipe_gridA + 1, H->pipe_gridB, qs};
    {
      TimedLaunch tl(H, STCA_K_STEP, s);
      if (int rc = launch_step_tc(H, -1, tg, TA, nullptr, &plan, H->part, H->last_G, Z, H->Ubf, s, nullptr,
                                  nullptr, 0, nullptr, after_encode && !H->timing))
        return rc;
    }
    if (int rc2 = check_launch("query init")) return rc2;
    for (int i = 0; i < M; ++i) {
      sB.layer = i - 1;
      aA.layer = i;
      {
        TimedLaunch tl(H, STCA_K_PIPE, s);
        if (int rc = launch_step_attn_pipe(H, sB, aA, s)) return rc;
      }
      if (int rc2 = check_launch("pipeline")) return rc2;
      sA.layer = i;
      aB.layer = i;
      {
        TimedLaunch tl(H, STCA_K_PIPE, s);
        if (int rc = launch_step_attn_pipe(H, sA, aB, s)) return rc;
      }
      if (int rc2 = check_launch("pipeline")) return rc2;
    }
    {
      TimedLaunch tl(H, STCA_K_STEP, s);
      QslotBufs qB = half_qs(TA);
      if (int rc = launch_step_tc(H, static_cast<int>(M - 1), sB.targets, TB, nullptr, nullptr, nullptr, 0,
                                  sB.Z, sB.Ubf, s, nullptr, nullptr, 2, &qB))
        return rc;
    }
    if (int rc2 = check_launch("target step")) return rc2;
    H->launches += 2 * M + 2;
    return ok();
  }
  {
    TimedLaunch tl(H, STCA_K_STEP, s);
    if (int rc = step(-1, nullptr)) return rc;
  }
  H->launches++;
  if (int rc = check_launch("query init")) return rc;
  for (int i = 0; i < H->M; ++i) {
    int rc = STCA_OK;
    {
      TimedLaunch tl(H, STCA_K_ATTN, s);
      if (naive) {
        rc = kv_project(H, i, s);
        if (!rc) rc = launch_attn_tc_naive(H, items_d, cta_d, H->last_grid, s);
        H->launches++;
      } else if (pp) {
        rc = launch_attn_pp(d, H->tmU, H->tmXt[i], items_d, cta_d, plan.pair_item_begin,
                            H->last_grid, H->part, H->last_G, H->cbuf,
                            H->attn_cnt + cnt_per_layer * i, H->status_d, H->opt_stop_tiles, s);
      } else if (path == 2) {
        rc = launch_attn_tc(H, i, items_d, cta_d, H->last_grid, s, proj, proj_mode == 2 ? &qs : nullptr);
      } else {
        const void* xti = static_cast<const char*>(H->xt) + layer_bytes * i;
        launch_attn_simt(H, i, xti, items_d, pairs_d, H->last_pairs, plan.toff, s);
      }
    }
    if (rc) return rc;
    H->launches++;
    if (int rc2 = check_launch("attention")) return rc2;
    {
      TimedLaunch tl(H, STCA_K_STEP, s);
      if (naive) {
        launch_combine_naive(H, plan, H->part, H->last_G, T, H->cbuf, s);
        H->launches++;
      } else if (!fused && !pp) {
        if (proj) launch_combine_proj(H, plan, H->part, H->last_G, T, H->cbuf, s);
        else launch_combine(H, plan, H->part, H->last_G, T, H->cbuf, s);
        H->launches++;
      }
      rc = step(i, H->cbuf);
    }
    if (rc) return rc;
    H->launches++;
    if (int rc2 = check_launch("target step")) return rc2;
  }
  if (zout && !head_in_step) {
    {
      TimedLaunch tl(H, STCA_K_HEAD, s);
      launch_head(H, targets, T, Z, zout, s);
    }
    H->launches++;
    if (int rc2 = check_launch("prediction head")) return rc2;
  }
  return ok();
}

extern "C" int stca_forward(stca_handle* H, const void* targets, const int64_t* target_offsets,
                            int64_t T, float* Z, void* stream) {
  return forward_impl(H, targets, target_offsets, T, Z, nullptr, stream);
}

extern "C" int stca_encode_forward(stca_handle* H, const void* X, const int64_t* offsets, int64_t R,
                                   int64_t N, const void* targets, const int64_t* target_offsets,
                                   int64_t T, float* Z, void* stream) {
  if (int rc = stca_encode(H, X, offsets, R, N, stream)) return rc;
  return forward_impl(H, targets, target_offsets, T, Z, nullptr, stream, true);
}

extern "C" int stca_forward_head(stca_handle* H, const void* targets, const int64_t* target_offsets,
                                 int64_t T, float* Z, float* zout, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (!H->whead) return set_error(STCA_EINVAL, "stca_forward_head: the handle has no head weights (Wz, zWu, zWg, zWd)");
  if (T > 0 && !zout) return set_error(STCA_EINVAL, "stca_forward_head: zout is NULL");
  if (reinterpret_cast<uintptr_t>(zout) % 16) return set_error(STCA_EINVAL, "zout must be 16-byte aligned");
  return forward_impl(H, targets, target_offsets, T, Z, zout, stream);
}

extern "C" int stca_head(stca_handle* H, const void* targets, int64_t T, const float* Z,
                         float* zout, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (!H->whead) return set_error(STCA_EINVAL, "stca_head: the handle has no head weights (Wz, zWu, zWg, zWd)");
  if (T < 0) return set_error(STCA_EINVAL, "T must be >= 0");
  if (T == 0) return ok();
  if (!targets || !Z || !zout) return set_error(STCA_EINVAL, "stca_head: targets, Z and zout must not be NULL");
  if (T > (int64_t(1) << 40)) return set_error(STCA_EINVAL, "stca_head: T too large");
  DeviceGuard g(H->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  {
    TimedLaunch tl(H, STCA_K_HEAD, s);
    // bf16 handles with the tensor-core step: its head products, as in the
    // forward's last step; otherwise the CUDA-core head kernel
    if (H->step_tc_ready && H->head_tc && H->opt_step_path != 1 &&
        reinterpret_cast<uintptr_t>(targets) % 16 == 0 && reinterpret_cast<uintptr_t>(Z) % 16 == 0) {
      if (int rc = launch_step_tc_head(H, targets, T, Z, zout, s)) return rc;
    } else {
      launch_head(H, targets, T, Z, zout, s);
    }
  }
  H->launches++;
  STCA_CUDA_TRY(cudaGetLastError());
  return ok();
}

extern "C" int stca_get_encoded(stca_handle* H, int layer, void* dst, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (!H->encoded) return set_error(STCA_ESTATE, "no encoded history");
  if (layer < 0 || layer >= H->M) return set_error(STCA_EINVAL, "layer out of range");
  if (!dst) return set_error(STCA_EINVAL, "dst is NULL");
  DeviceGuard g(H->device);
  const size_t bytes = static_cast<size_t>(H->N) * H->d * H->elem;
  STCA_CUDA_TRY(cudaMemcpyAsync(dst, static_cast<const char*>(H->xt) + bytes * layer, bytes,
                                cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
  return ok();
}

extern "C" int stca_plan_attention(const int64_t* offsets, const int64_t* target_offsets,
                                   int64_t R, int h, int path, int num_ctas, int64_t split_keys,
                                   int64_t* n_items, int64_t* grid, int64_t* partial_rows,
                                   int64_t* items, int64_t items_cap, int32_t* cta_begin,
                                   int64_t cta_cap) {
  if (!n_items || !grid || !partial_rows) return set_error(STCA_EINVAL, "NULL output count");
  if (path != 1 && path != 2) return set_error(STCA_EINVAL, "path must be 1 or 2");
  if (h < 1 || num_ctas < 1 || split_keys < 0) return set_error(STCA_EINVAL, "bad h, num_ctas or split_keys");
  if (int rc = validate_offsets(offsets, R, offsets ? offsets[R] : 0, true, "offsets")) return rc;
  if (int rc = validate_offsets(target_offsets, R, target_offsets ? target_offsets[R] : 0, false,
                                "target_offsets"))
    return rc;
  PlanHost P;
  build_plan_host(offsets, target_offsets, R, h, path, num_ctas, split_keys, P);
  if (int rc = check_plan(P, offsets, target_offsets, R, h, path)) return rc;
  *n_items = static_cast<int64_t>(P.items.size());
  *grid = P.grid;
  *partial_rows = P.G;
  if (items) {
    if (items_cap < *n_items) return set_error(STCA_EINVAL, "items_cap too small");
    for (size_t w = 0; w < P.items.size(); ++w) {
      const AttnItem& it = P.items[w];
      int64_t* o = items + 7 * w;
      o[0] = it.req; o[1] = it.mt; o[2] = it.key0; o[3] = it.nkeys;
      o[4] = it.qrow0; o[5] = it.rows; o[6] = it.row_base;
    }
  }
  if (cta_begin && path == 2) {
    if (cta_cap < P.grid + 1) return set_error(STCA_EINVAL, "cta_cap too small");
    std::copy(P.cta_begin.begin(), P.cta_begin.end(), cta_begin);
  }
  return ok();
}

// ------------------------------------------------------------------ host entry
// End to end from host buffers.  With the tensor-core encoder and a large
// batch, X crosses to the device in chunks of whole 128-row tiles on a second
// stream, and each chunk is encoded as soon as its copy lands (an event per
// chunk), so the encoder works while the next chunks are still in flight; the
// forward follows the last chunk.  One cudaMemcpyAsync per chunk.
extern "C" int stca_run_host(stca_handle* H, const void* X_host, const int64_t* offsets,
                             int64_t R, int64_t N, const void* targets_host,
                             const int64_t* target_offsets, int64_t T, float* Z_host,
                             void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (!X_host || (T > 0 && (!targets_host || !Z_host)))
    return set_error(STCA_EINVAL, "a host buffer is NULL");
  if (N < 1) return set_error(STCA_EINVAL, "N must be >= 1");
  if (int rc = validate_offsets(offsets, R, N, true, "offsets")) return rc;
  if (T < 0) return set_error(STCA_EINVAL, "T must be >= 0");
  if (int rc = validate_offsets(target_offsets, R, T, false, "target_offsets")) return rc;
  DeviceGuard g(H->device);
  if (!g.ok) return set_error(STCA_ECUDA, "cannot select the handle's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = static_cast<size_t>(H->d) * H->elem;
  const size_t xb = static_cast<size_t>(N) * row_bytes;
  const size_t tb = static_cast<size_t>(T) * H->d * H->elem;
  const size_t zb = static_cast<size_t>(T) * H->M * H->d * sizeof(float);
  if (int rc = ensure_dev(&H->x_stage, &H->x_stage_cap, xb)) return rc;
  if (T > 0) {
    if (int rc = ensure_dev(&H->t_stage, &H->t_stage_cap, tb)) return rc;
    if (int rc = ensure_dev(reinterpret_cast<void**>(&H->z_stage), &H->z_stage_cap, zb)) return rc;
  }
  constexpr int kChunks = 8;
  constexpr int64_t kMinChunkRows = 8192;
  const bool chunked = encode_on_tensor_cores(H) && N >= kChunks * kMinChunkRows;
  if (T > 0) STCA_CUDA_TRY(cudaMemcpyAsync(H->t_stage, targets_host, tb, cudaMemcpyHostToDevice, s));
  if (!chunked) {
    STCA_CUDA_TRY(cudaMemcpyAsync(H->x_stage, X_host, xb, cudaMemcpyHostToDevice, s));
    if (int rc = stca_encode(H, H->x_stage, offsets, R, N, stream)) return rc;
  } else {
    if (!H->copy_stream &&
        cudaStreamCreateWithFlags(&H->copy_stream, cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      H->copy_stream = nullptr;
      return set_error(STCA_ECUDA, "cannot create the copy stream");
    }
    while (H->chunk_evt.size() < kChunks + 1) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        return set_error(STCA_ECUDA, "cannot create the chunk events");
      }
      H->chunk_evt.push_back(e);
    }
    if (int rc = encode_begin(H, H->x_stage, offsets, R, N)) return rc;
    // the copies overwrite the staging buffer: after everything on `stream` so far
    STCA_CUDA_TRY(cudaEventRecord(H->chunk_evt[kChunks], s));
    STCA_CUDA_TRY(cudaStreamWaitEvent(H->copy_stream, H->chunk_evt[kChunks], 0));
    const int64_t tiles = (N + 127) / 128;
    const int64_t per = (tiles + kChunks - 1) / kChunks * 128;
    for (int c = 0; c < kChunks; ++c) {
      const int64_t r0 = c * per, rows = std::min<int64_t>(per, N - r0);
      if (rows <= 0) break;
      STCA_CUDA_TRY(cudaMemcpyAsync(static_cast<char*>(H->x_stage) + r0 * row_bytes,
                                    static_cast<const char*>(X_host) + r0 * row_bytes, rows * row_bytes,
                                    cudaMemcpyHostToDevice, H->copy_stream));
      STCA_CUDA_TRY(cudaEventRecord(H->chunk_evt[c], H->copy_stream));
    }
    for (int c = 0; c < kChunks; ++c) {
      const int64_t r0 = c * per, rows = std::min<int64_t>(per, N - r0);
      if (rows <= 0) break;
      STCA_CUDA_TRY(cudaStreamWaitEvent(s, H->chunk_evt[c], 0));
      int rc;
      {
        TimedLaunch tl(H, STCA_K_ENCODE, s);
        rc = launch_encode_tc(H, static_cast<const char*>(H->x_stage) + r0 * row_bytes, rows, s, r0);
      }
      if (rc) return rc;
      H->launches++;
      if (int rc2 = check_launch("encode (tensor cores, chunk)")) return rc2;
    }
    H->encoded = true;
  }
  if (T > 0) {
    if (int rc = forward_impl(H, H->t_stage, target_offsets, T, H->z_stage, nullptr, stream, true)) return rc;
    STCA_CUDA_TRY(cudaMemcpyAsync(Z_host, H->z_stage, zb, cudaMemcpyDeviceToHost, s));
  }
  STCA_CUDA_TRY(cudaStreamSynchronize(s));
  return ok();
}

// ------------------------------------------------------------------ misc
extern "C" int stca_device_status(stca_handle* H, void* stream) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  DeviceGuard g(H->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  STCA_CUDA_TRY(cudaStreamSynchronize(s));
  int st = 0;
  STCA_CUDA_TRY(cudaMemcpy(&st, H->status_d, sizeof(int), cudaMemcpyDeviceToHost));
  STCA_CUDA_TRY(cudaMemset(H->status_d, 0, sizeof(int)));
  if (st) {
    std::string m = "device status 0x" + std::to_string(st) + ":";
    if (st & kStatusEncodeTimeout) m += " encoder gave up a bounded wait;";
    if (st & kStatusAttnTimeout) m += " attention gave up a bounded wait;";
    if (st & kStatusStepTimeout) m += " per-target step gave up a bounded wait;";
    if (st & kStatusKvTimeout) m += " K/V projection gave up a bounded wait;";
    return set_error(STCA_EDEVICE, m);
  }
  return ok();
}

extern "C" int stca_set_option(stca_handle* H, int option, int64_t value) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  switch (option) {
    case STCA_OPT_ATTN_PATH:
      if (value < 0 || value > 2) return set_error(STCA_EINVAL, "attention path must be 0, 1 or 2");
      H->opt_attn_path = static_cast<int>(value);
      return ok();
    case STCA_OPT_ENCODE_PATH:
      if (value < 0 || value > 2) return set_error(STCA_EINVAL, "encode path must be 0, 1 or 2");
      H->opt_encode_path = static_cast<int>(value);
      return ok();
    case STCA_OPT_STEP_PATH:
      if (value < 0 || value > 2) return set_error(STCA_EINVAL, "step path must be 0, 1 or 2");
      H->opt_step_path = static_cast<int>(value);
      return ok();
    case STCA_OPT_TIMING:
      if (value != 0 && value != 1) return set_error(STCA_EINVAL, "timing must be 0 or 1");
      H->timing = value != 0;
      return ok();
    case STCA_OPT_ATTN_FORM:
      if (value < 0 || value > 2) return set_error(STCA_EINVAL, "attention form must be 0, 1 or 2");
      H->opt_attn_form = static_cast<int>(value);
      return ok();
    case STCA_OPT_ATTN_KERNEL:
      if (value < 0 || value > 2) return set_error(STCA_EINVAL, "attention kernel must be 0, 1 or 2");
      H->opt_attn_kernel = static_cast<int>(value);
      return ok();
    case STCA_OPT_TEST_STOP_TILES:
      if (value < 0 || value > (int64_t(1) << 30)) return set_error(STCA_EINVAL, "stop tiles must be >= 0");
      H->opt_stop_tiles = static_cast<int>(value);
      return ok();
    case STCA_OPT_BW_GEMM:
      if (value < 0 || value > 1) return set_error(STCA_EINVAL, "backward GEMM must be 0 or 1");
      H->opt_bw_gemm = static_cast<int>(value);
      return ok();
    case STCA_OPT_PIPELINE:
      if (value < 0 || value > 1) return set_error(STCA_EINVAL, "pipeline must be 0 or 1");
      H->opt_pipeline = static_cast<int>(value);
      return ok();
    case STCA_OPT_SPLIT_KEYS:
      if (value < 0 || value % 128 || value > (int64_t(1) << 30))
        return set_error(STCA_EINVAL, "split must be 0 or a positive multiple of 128");
      if (value != H->opt_split_keys) H->last_toff.clear();   // the plan cuts the keys by it
      H->opt_split_keys = value;
      return ok();
    default:
      return set_error(STCA_EINVAL, "unknown or read-only option " + std::to_string(option));
  }
}

extern "C" int stca_get_option(stca_handle* H, int option, int64_t* value) {
  if (!H || !value) return set_error(STCA_EINVAL, "handle or value is NULL");
  switch (option) {
    case STCA_OPT_ATTN_PATH: *value = H->opt_attn_path; return ok();
    case STCA_OPT_ENCODE_PATH: *value = H->opt_encode_path; return ok();
    case STCA_OPT_STEP_PATH: *value = H->opt_step_path; return ok();
    case STCA_OPT_SPLIT_KEYS: *value = H->opt_split_keys; return ok();
    case STCA_OPT_TIMING: *value = H->timing ? 1 : 0; return ok();
    case STCA_OPT_LAUNCHES: *value = H->launches; return ok();
    case STCA_OPT_ATTN_FORM: *value = H->opt_attn_form; return ok();
    case STCA_OPT_ATTN_KERNEL: *value = H->opt_attn_kernel; return ok();
    case STCA_OPT_TEST_STOP_TILES: *value = H->opt_stop_tiles; return ok();
    case STCA_OPT_BW_GEMM: *value = H->opt_bw_gemm; return ok();
    case STCA_OPT_PIPELINE: *value = H->opt_pipeline; return ok();
    case STCA_OPT_LAST_FORM: *value = H->last_naive ? 1 : 0; return ok();
    default: return set_error(STCA_EINVAL, "unknown option " + std::to_string(option));
  }
}

extern "C" int stca_kernel_times(stca_handle* H, double* ms, int64_t* launches, int n) {
  if (!H) return set_error(STCA_EINVAL, "handle is NULL");
  if (n < 0) return set_error(STCA_EINVAL, "n must be >= 0");
  DeviceGuard g(H->device);
  double acc[STCA_K_CLASSES] = {};
  int64_t cnt[STCA_K_CLASSES] = {};
  int rc = STCA_OK;
  for (auto& t : H->timed) {
    float v = 0.f;
    if (rc == STCA_OK) {
      cudaError_t e = cudaEventSynchronize(t.b);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&v, t.a, t.b);
      if (e != cudaSuccess) rc = set_error(STCA_ECUDA, std::string("event timing: ") + cudaGetErrorString(e));
    }
    acc[t.cls] += v;
    cnt[t.cls] += 1;
    H->ev_pool.push_back(t.a);
    H->ev_pool.push_back(t.b);
  }
  H->timed.clear();
  if (rc != STCA_OK) return rc;
  for (int c = 0; c < n && c < STCA_K_CLASSES; ++c) {
    if (ms) ms[c] = acc[c];
    if (launches) launches[c] = cnt[c];
  }
  return ok();
}
