// pkm_api.cu -- the extern "C" entry points declared in include/pkm.h: argument
// validation, workspace layout and the launch sequence of each pass.
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "../../include/pkm.h"
#include "pkm_common.cuh"
#include "pkm_kernels.h"
#include "pkm_tc.h"

namespace {

using pkm::LayerArgs;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Which implementation of the query network and per-half search runs.
enum class Path { kTensor, kSimt };

Path choose_path(const pkm_shape* s) {
  const char* env = getenv("PKM_PATH");
  if (env && strcmp(env, "simt") == 0) return Path::kSimt;
  return pkm::tc_supported(s->dtype, s->d_model, s->H, s->dq, s->n, s->k) ? Path::kTensor
                                                                          : Path::kSimt;
}

// Fields both passes use: B, H, n, k, v, dtype.
int validate_common(const pkm_shape* s) {
  if (!s) return PKM_ERR_INVALID_ARG;
  if (s->B < 0 || s->H < 1 || s->n < 1 || s->k < 1 || s->k > s->n || s->v < 1)
    return PKM_ERR_INVALID_ARG;
  if (s->dtype != PKM_F32 && s->dtype != PKM_BF16) return PKM_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s->n) * s->n > 0x7fffffffLL) return PKM_ERR_INVALID_ARG;
  if (s->B * s->H * static_cast<int64_t>(s->k) > 0x7fffffffLL) return PKM_ERR_UNSUPPORTED;
  if (s->k > pkm::kMaxK) return PKM_ERR_UNSUPPORTED;
  const int esz = s->dtype == PKM_F32 ? 4 : 2;
  if ((static_cast<int64_t>(s->v) * esz) % 16) return PKM_ERR_UNSUPPORTED;
  if (!pkm::select_gather_supported(s->H, s->k, s->v, s->dtype)) return PKM_ERR_UNSUPPORTED;
  return PKM_OK;
}

// The forward also needs d_model, dq and bn_eps.
int validate_shape(const pkm_shape* s) {
  const int rc = validate_common(s);
  if (rc != PKM_OK) return rc;
  if (s->d_model < 1 || s->dq < 2 || (s->dq & 1)) return PKM_ERR_INVALID_ARG;
  if (!(s->bn_eps >= 0.f) || s->bn_eps > 1e30f) return PKM_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s->H) * s->dq > (1 << 24)) return PKM_ERR_INVALID_ARG;
  if (pkm::subkey_topk_simt_smem(s->dq) > 200 * 1024) return PKM_ERR_UNSUPPORTED;
  return PKM_OK;
}

struct ForwardWs {
  int* status;
  float* q;         // SIMT path: fp32 q [B][H*dq]
  void* planes;     // tensor path: bf16 q planes [3][B][H*dq]
  float* list_s;    // [B][H][2][32] best 32 per half (any order)
  int* list_i;      // [B][H][2][32]
};

size_t forward_ws(const pkm_shape* s, ForwardWs* w, char* base) {
  const int64_t F = static_cast<int64_t>(s->H) * s->dq;
  const int64_t L = s->B * s->H * 2 * static_cast<int64_t>(pkm::kMaxK);
  size_t off = pkm::kStatusBytes;
  const size_t o_q = off;  off += align256(static_cast<size_t>(s->B) * F * 6);  // fp32 q or 3 bf16 planes
  const size_t o_ls = off; off += align256(sizeof(float) * L);
  const size_t o_li = off; off += align256(sizeof(int) * L);
  if (w && base) {
    w->status = reinterpret_cast<int*>(base);
    w->q = reinterpret_cast<float*>(base + o_q);
    w->planes = base + o_q;
    w->list_s = reinterpret_cast<float*>(base + o_ls);
    w->list_i = reinterpret_cast<int*>(base + o_li);
  }
  return off;
}

size_t backward_ws(const pkm_shape* s, pkm::BackwardWs* w, char* base) {
  return pkm::backward_ws_bytes(s->B, s->H, s->k, static_cast<int64_t>(s->n) * s->n, w, base);
}

// ---------------------------------------------------------------------------
// Stage tracing: when enabled, every call records a CUDA event on its stream at
// each stage boundary; pkm_trace_read() waits for them and sums the durations.
// ---------------------------------------------------------------------------
constexpr int kMaxStages = 4;
constexpr int kPasses = 2;

struct TraceSet {
  int pass;
  int nstages;
  cudaEvent_t ev[kMaxStages + 1];
};

std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<TraceSet> g_trace_pending;
std::vector<cudaEvent_t> g_event_pool;
int64_t g_launches = 0;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Records stage boundaries for one call (no-op when tracing is off).
struct Tracer {
  bool on = false;
  TraceSet set{};
  int next = 0;
  cudaStream_t st;
  Tracer(int pass, int nstages, cudaStream_t s) : st(s) {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    on = g_trace_on;
    if (!on) return;
    set.pass = pass;
    set.nstages = nstages;
    for (int i = 0; i <= nstages; ++i) {
      set.ev[i] = take_event();
      if (!set.ev[i]) on = false;
    }
  }
  void mark() {
    if (on && next <= set.nstages) cudaEventRecord(set.ev[next++], st);
  }
  void finish(bool ok, int launches) {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (ok) g_launches += launches;
    if (!on) return;
    if (ok && next == set.nstages + 1) {
      g_trace_pending.push_back(set);
    } else {
      for (int i = 0; i <= set.nstages; ++i)
        if (set.ev[i]) g_event_pool.push_back(set.ev[i]);
    }
  }
};

}  // namespace

extern "C" {

int pkm_trace_enable(int on) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  g_trace_on = on != 0;
  return PKM_OK;
}

int pkm_trace_read(int pass, double* stage_ms, int max_stages, int64_t* calls,
                   int64_t* launches) {
  if (pass < 0 || pass >= kPasses || max_stages < 0 || (max_stages && !stage_ms))
    return PKM_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  for (int i = 0; i < max_stages; ++i) stage_ms[i] = 0.0;
  int64_t n = 0;
  std::vector<TraceSet> keep;
  int rc = PKM_OK;
  for (const TraceSet& t : g_trace_pending) {
    if (t.pass != pass) {
      keep.push_back(t);
      continue;
    }
    if (cudaEventSynchronize(t.ev[t.nstages]) != cudaSuccess) rc = PKM_ERR_CUDA;
    for (int i = 0; i < t.nstages && i < max_stages; ++i) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, t.ev[i], t.ev[i + 1]) != cudaSuccess) rc = PKM_ERR_CUDA;
      stage_ms[i] += ms;
    }
    for (int i = 0; i <= t.nstages; ++i) g_event_pool.push_back(t.ev[i]);
    ++n;
  }
  g_trace_pending.swap(keep);
  if (calls) *calls = n;
  if (launches) {
    *launches = g_launches;
    g_launches = 0;
  }
  return rc;
}

size_t pkm_workspace_size(const pkm_shape* s, int for_backward) {
  if ((for_backward ? validate_common(s) : validate_shape(s)) != PKM_OK) return 0;
  return for_backward ? backward_ws(s, nullptr, nullptr) : forward_ws(s, nullptr, nullptr);
}

int pkm_forward(const pkm_shape* s, const void* x, const void* W_q, const float* bn_mean,
                const float* bn_var, const float* bn_gamma, const float* bn_beta,
                const void* subkeys, const void* values, float* out, int32_t* indices,
                float* weights, float* scores, void* workspace, size_t workspace_bytes,
                void* stream) {
  int rc = validate_shape(s);
  if (rc != PKM_OK) return rc;
  // Per-token tensors may be NULL when there are no tokens.
  const bool tok = s->B > 0;
  if (!W_q || !bn_mean || !bn_var || !bn_gamma || !bn_beta || !subkeys || !values ||
      (tok && (!x || !out || !indices || !weights)))
    return PKM_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W_q, bn_mean, bn_var, bn_gamma, bn_beta, subkeys, values, out,
                        indices, weights, scores};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return PKM_ERR_UNSUPPORTED;
  const size_t need = forward_ws(s, nullptr, nullptr);
  if (!workspace || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PKM_ERR_WORKSPACE;
  if (s->B == 0) return PKM_OK;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ForwardWs w;
  forward_ws(s, &w, static_cast<char*>(workspace));
  LayerArgs a{s->B, s->d_model, s->H, s->dq, s->n, s->k, s->v, s->dtype, s->bn_eps,
              x, W_q, bn_mean, bn_var, bn_gamma, bn_beta, subkeys, values, w.status};
  if (cudaMemsetAsync(w.status, 0, sizeof(int), st) != cudaSuccess) return PKM_ERR_CUDA;
  // Stages: 0 query network, 1 per-half scores + top-k, 2 candidate top-k + softmax + gather.
  Tracer tr(0, 3, st);
  cudaError_t e;
  tr.mark();
  if (choose_path(s) == Path::kTensor) {
    e = pkm::launch_query_tc(a, w.planes, st);
    tr.mark();
    if (e == cudaSuccess) e = pkm::launch_score_topk_tc(a, w.planes, w.list_s, w.list_i, st);
  } else {
    e = pkm::launch_query_bn_simt(a, w.q, st);
    tr.mark();
    if (e == cudaSuccess) e = pkm::launch_subkey_topk_simt(a, w.q, w.list_s, w.list_i, st);
  }
  tr.mark();
  if (e == cudaSuccess)
    e = pkm::launch_select_gather(a, w.list_s, w.list_i, out, indices, weights, scores, st);
  tr.mark();
  tr.finish(e == cudaSuccess, 3);
  return e == cudaSuccess ? PKM_OK : PKM_ERR_CUDA;
}

int pkm_backward_values(const pkm_shape* s, const void* values, const int32_t* indices,
                        const float* weights, const void* grad_out, float* grad_values,
                        float* grad_scores, void* workspace, size_t workspace_bytes,
                        void* stream) {
  int rc = validate_common(s);
  if (rc != PKM_OK) return rc;
  if (!values || !grad_values || (s->B > 0 && (!indices || !weights || !grad_out)))
    return PKM_ERR_INVALID_ARG;
  const void* ptrs[] = {values, indices, weights, grad_out, grad_values, grad_scores};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return PKM_ERR_UNSUPPORTED;
  const size_t need = backward_ws(s, nullptr, nullptr);
  if (!workspace || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PKM_ERR_WORKSPACE;
  if (s->B == 0) return PKM_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  pkm::BackwardWs w;
  backward_ws(s, &w, static_cast<char*>(workspace));
  int* status = static_cast<int*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return PKM_ERR_CUDA;
  // Stages: 0 grad wrt kept scores, 1 slot grouping + row sums into grad_values.
  Tracer tr(1, 2, st);
  tr.mark();
  cudaError_t e = pkm::launch_backward_values(
      s->B, s->H, s->k, s->v, s->dtype, static_cast<int64_t>(s->n) * s->n, values, indices,
      weights, grad_out, grad_values, grad_scores, w, status, st, [&] { tr.mark(); });
  tr.mark();
  tr.finish(e == cudaSuccess, grad_scores ? 7 : 6);
  return e == cudaSuccess ? PKM_OK : PKM_ERR_CUDA;
}

int pkm_device_status(void* workspace, void* stream) {
  if (!workspace) return PKM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PKM_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return PKM_ERR_CUDA;
  if (cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return PKM_ERR_CUDA;
  return h == 0 ? PKM_OK : PKM_ERR_DEVICE;
}

const char* pkm_status_string(int status) {
  switch (status) {
    case PKM_OK: return "ok";
    case PKM_ERR_INVALID_ARG: return "invalid argument";
    case PKM_ERR_UNSUPPORTED: return "unsupported shape, dtype or alignment";
    case PKM_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case PKM_ERR_CUDA: return "CUDA error";
    case PKM_ERR_DEVICE: return "device-side error recorded by a kernel";
  }
  return "unknown status";
}

}  // extern "C"
