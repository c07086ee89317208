// pkm_api.cu -- the extern "C" entry points declared in include/pkm.h: argument
// validation, workspace layout and the launch sequence of each pass.
#include <stdlib.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include <atomic>
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

// Which implementation of the forward runs: the small-batch kernels for a few
// tokens, else the tensor-core kernels where the shape fits their tiles, else the
// CUDA-core kernels. The option PKM_OPT_PATH pins one of the large-batch paths
// (tests compare the paths on the same inputs).
enum class Path { kTensor, kSimt, kSmall };

// Process-wide implementation switches (pkm_set_option). The environment variables
// PKM_PATH (auto | tc | simt | small_fused | small_split) and PKM_SUBBATCHES (1..4) give their initial values and
// are read once, at the first call that needs them.
std::atomic<int> g_opt_path{PKM_PATH_AUTO};
std::atomic<int> g_opt_subbatches{1};

void init_options() {
  static std::once_flag once;
  std::call_once(once, [] {
    const char* p = getenv("PKM_PATH");
    if (p && strcmp(p, "simt") == 0) g_opt_path = PKM_PATH_SIMT;
    if (p && strcmp(p, "tc") == 0) g_opt_path = PKM_PATH_TC;
    if (p && strcmp(p, "small_fused") == 0) g_opt_path = PKM_PATH_SMALL_FUSED;
    if (p && strcmp(p, "small_split") == 0) g_opt_path = PKM_PATH_SMALL_SPLIT;
    const char* sb = getenv("PKM_SUBBATCHES");
    if (sb) {
      const int v = atoi(sb);
      g_opt_subbatches = v < 1 ? 1 : (v > 4 ? 4 : v);
    }
  });
}

// The options one call works with, read once when it starts: a concurrent
// pkm_set_option cannot give a call the workspace layout of one path and the launches
// of another.
struct Opts {
  int path;
  int subbatches;
};

Opts current_options() {
  init_options();
  return {g_opt_path.load(std::memory_order_relaxed),
          g_opt_subbatches.load(std::memory_order_relaxed)};
}

Path choose_path(const pkm_shape* s, const Opts& o) {
  const int pin = o.path;
  if (pin == PKM_PATH_SIMT) return Path::kSimt;
  // A pinned small-batch form takes every batch the small-batch kernels support; the
  // automatic choice only those up to the measured crossover for the head count.
  const bool pinned_small = pin == PKM_PATH_SMALL_FUSED || pin == PKM_PATH_SMALL_SPLIT;
  if (pin != PKM_PATH_TC &&
      pkm::small_supported(s->B, s->d_model, s->H, s->dq, s->n, s->k, s->v, s->dtype) &&
      (pinned_small || s->B <= pkm::small_auto_max_b(s->H, s->d_model, s->dq, s->dtype)))
    return Path::kSmall;
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

// The slot-usage count reads B, H, n and k.
int validate_usage(const pkm_shape* s) {
  if (!s) return PKM_ERR_INVALID_ARG;
  if (s->B < 0 || s->H < 1 || s->n < 1 || s->k < 1 || s->k > s->n) return PKM_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s->n) * s->n > 0x7fffffffLL) return PKM_ERR_INVALID_ARG;
  if (s->B * s->H * static_cast<int64_t>(s->k) > 0x7fffffffLL) return PKM_ERR_UNSUPPORTED;
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
  void* planes;     // tensor path: bf16 q planes [kScorePlanes][sub][H*dq] of a sub-batch
  float* list_s;    // [B][H][2][32] best 32 per half (any order)
  int* list_i;      // [B][H][2][32]
  float* part;      // small-batch path: [B][H][v] each head's output row, then [B]
                    // per-token counts (single-kernel form)
};

// Tokens per pipelined sub-batch of the tensor-core path: PKM_OPT_SUBBATCHES (1..4,
// default 1) sub-batches of at least 2048 tokens, a multiple of the 128-token tile.
int64_t sub_batch_tokens(int64_t B, const Opts& o) {
  const int64_t want = o.subbatches;
  int64_t S = B / 2048;
  if (S > want) S = want;
  if (S < 1) S = 1;
  int64_t sub = (B + S - 1) / S;
  sub = (sub + 127) / 128 * 128;
  return sub < B ? sub : B;
}

size_t forward_ws(const pkm_shape* s, const Opts& o, ForwardWs* w, char* base) {
  const int64_t F = static_cast<int64_t>(s->H) * s->dq;
  const Path path = choose_path(s, o);
  const size_t qbytes = path == Path::kTensor
                            ? static_cast<size_t>(sub_batch_tokens(s->B, o)) * F * 2 *
                                  pkm::kScorePlanes
                            : static_cast<size_t>(s->B) * F * 4;
  // The small-batch path keeps each chunk's best 32 before merging them.
  const int64_t L = path == Path::kSmall
                        ? static_cast<int64_t>(pkm::small_chunk_entries(s->B, s->H, s->n))
                        : s->B * s->H * 2 * static_cast<int64_t>(pkm::kMaxK);
  size_t off = pkm::kStatusBytes;
  const size_t o_q = off;  off += align256(qbytes);
  const size_t o_ls = off; off += align256(sizeof(float) * L);
  const size_t o_li = off; off += align256(sizeof(int) * L);
  const size_t o_pt = off;
  off += align256(path == Path::kSmall
                      ? sizeof(float) * s->B * s->H * s->v + sizeof(unsigned) * s->B
                      : 0);
  if (w && base) {
    w->status = reinterpret_cast<int*>(base);
    w->q = reinterpret_cast<float*>(base + o_q);
    w->planes = base + o_q;
    w->list_s = reinterpret_cast<float*>(base + o_ls);
    w->list_i = reinterpret_cast<int*>(base + o_li);
    w->part = reinterpret_cast<float*>(base + o_pt);
  }
  return off;
}

// BatchNorm training mode: acc of the whole batch (three bf16 planes on the tensor
// path, fp32 otherwise) and the per-chunk statistics, after the forward's workspace.
struct TrainWs {
  void* acc;
  double* part;
};

size_t forward_train_ws(const pkm_shape* s, const Opts& o, ForwardWs* fw, TrainWs* tw,
                        char* base) {
  const int64_t F = static_cast<int64_t>(s->H) * s->dq;
  const size_t accb =
      static_cast<size_t>(s->B) * F * (choose_path(s, o) == Path::kTensor ? 6 : 4);
  const int64_t chunks = (s->B + pkm::kStatChunk - 1) / pkm::kStatChunk;
  size_t off = forward_ws(s, o, fw, base);
  const size_t o_acc = off;  off += align256(accb);
  const size_t o_part = off; off += align256(sizeof(double) * 2 * F * (chunks > 0 ? chunks : 1));
  if (tw && base) {
    tw->acc = base + o_acc;
    tw->part = reinterpret_cast<double*>(base + o_part);
  }
  return off;
}

size_t backward_ws(const pkm_shape* s, pkm::BackwardWs* w, char* base) {
  return pkm::backward_ws_bytes(s->B, s->H, s->k, static_cast<int64_t>(s->n) * s->n, s->v, w,
                               base);
}

// ---------------------------------------------------------------------------
// Stage tracing: when enabled, every kernel a call launches is bracketed by two CUDA
// events on the stream it runs on; pkm_trace_read() waits for them and sums the
// durations per stage.
// ---------------------------------------------------------------------------
constexpr int kPasses = 2;

struct TraceSpan {
  int stage;
  int start, stop;  // indices into TraceCall::events
};
struct TraceCall {
  int pass;
  std::vector<cudaEvent_t> events;  // each recorded once; spans may share them
  std::vector<TraceSpan> spans;
};

std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<TraceCall> g_trace_pending;
std::vector<cudaEvent_t> g_event_pool;  // timing events, reused
int64_t g_launches = 0;

cudaEvent_t take_timing_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// NVTX range names of the traced stages (pass 0 forward, pass 1 backward).
const char* stage_name(int pass, int stage) {
  static const char* const kNames[kPasses][4] = {
      {"pkm.forward.query", "pkm.forward.scores", "pkm.forward.gather", "pkm.forward"},
      {"pkm.backward.scores", "pkm.backward.values", "pkm.backward.stage2", "pkm.backward"}};
  return kNames[pass][stage & 3];
}

class Tracer {
 public:
  Tracer(int pass) {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    on_ = g_trace_on;
    call_.pass = pass;
  }
  ~Tracer() {
    while (nvtx_open_ > 0) {
      nvtxRangePop();
      --nvtx_open_;
    }
  }
  // Spans nest: end() closes the most recently begun span that is still open. Every
  // span is also an NVTX range (host side; profilers attach the launches inside it).
  void begin(int stage, cudaStream_t st) { open_span(stage, record(st)); }
  void end(cudaStream_t st) { close_span(record(st)); }
  // The same at the point of the stream where the previous begin / end / next recorded
  // its event (one event for both): only where nothing has been issued to `st` since.
  // Each timing event recorded between two kernels delays the second one, so a call
  // records one event per stage boundary.
  void begin_here(int stage, cudaStream_t st) { open_span(stage, reuse(st)); }
  void end_here(cudaStream_t st) { close_span(reuse(st)); }
  // End the innermost open span and begin `stage` at one event (nothing in between).
  void next(int stage, cudaStream_t st) {
    const int ev = record(st);
    close_span(ev);
    open_span(stage, ev);
  }
  void finish(bool ok, int launches) {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (ok) g_launches += launches;
    if (!on_) return;
    if (ok && open_.empty()) {
      g_trace_pending.push_back(call_);
    } else {
      for (cudaEvent_t e : call_.events) g_event_pool.push_back(e);
    }
  }

 private:
  // Index of a newly recorded event (-1 when tracing is off or out of events).
  int record(cudaStream_t st) {
    if (!on_) return -1;
    cudaEvent_t e;
    {
      std::lock_guard<std::mutex> lk(g_trace_mu);
      e = take_timing_event();
    }
    if (!e) {
      on_ = false;
      return -1;
    }
    cudaEventRecord(e, st);
    call_.events.push_back(e);
    last_ = static_cast<int>(call_.events.size()) - 1;
    last_st_ = st;
    return last_;
  }
  int reuse(cudaStream_t st) { return (on_ && last_ >= 0 && last_st_ == st) ? last_ : record(st); }
  void open_span(int stage, int ev) {
    nvtxRangePushA(stage_name(call_.pass, stage));
    ++nvtx_open_;
    if (!on_ || ev < 0) return;
    open_.push_back(call_.spans.size());
    call_.spans.push_back(TraceSpan{stage, ev, -1});
  }
  void close_span(int ev) {
    if (nvtx_open_ > 0) {
      nvtxRangePop();
      --nvtx_open_;
    }
    if (!on_ || open_.empty() || ev < 0) return;
    call_.spans[open_.back()].stop = ev;
    open_.pop_back();
  }

  bool on_ = false;
  int nvtx_open_ = 0;
  TraceCall call_;
  std::vector<size_t> open_;
  int last_ = -1;
  cudaStream_t last_st_ = nullptr;
};

// ---------------------------------------------------------------------------
// Second stream per device (highest priority, so its blocks are scheduled ahead of the
// caller's when both have work queued) for the parts of a call that are independent
// of the rest: the value-gradient rows of the backward passes and the gathers of the
// pipelined forward. Plus ordering events.
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
std::mutex g_aux_mu;
cudaStream_t g_aux_stream[kMaxDevices] = {};
std::vector<cudaEvent_t> g_sync_events[kMaxDevices];
size_t g_sync_next[kMaxDevices] = {};

// The calling thread's device's helper stream and `n` ordering events (created on
// first use, then reused round robin).
int aux_resources(int n, cudaStream_t* aux, cudaEvent_t* evs) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_aux_mu);
  if (!g_aux_stream[dev]) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&g_aux_stream[dev], cudaStreamNonBlocking, greatest) !=
            cudaSuccess)
      return PKM_ERR_CUDA;
    for (int i = 0; i < 64; ++i) {
      cudaEvent_t e;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return PKM_ERR_CUDA;
      g_sync_events[dev].push_back(e);
    }
  }
  *aux = g_aux_stream[dev];
  std::vector<cudaEvent_t>& pool = g_sync_events[dev];
  for (int i = 0; i < n; ++i) evs[i] = pool[(g_sync_next[dev]++) % pool.size()];
  return PKM_OK;
}

// The helper stream with a fork and a join event, for a call that splits in two.
int side_stream(pkm::SideStream* side) {
  cudaEvent_t ev[2];
  const int rc = aux_resources(2, &side->st, ev);
  if (rc != PKM_OK) return rc;
  side->fork = ev[0];
  side->join = ev[1];
  return PKM_OK;
}

}  // namespace

extern "C" {

int pkm_set_option(int option, int value) {
  init_options();
  if (option == PKM_OPT_PATH) {
    if (value != PKM_PATH_AUTO && value != PKM_PATH_TC && value != PKM_PATH_SIMT &&
        value != PKM_PATH_SMALL_FUSED && value != PKM_PATH_SMALL_SPLIT)
      return PKM_ERR_INVALID_ARG;
    g_opt_path = value;
    return PKM_OK;
  }
  if (option == PKM_OPT_SUBBATCHES) {
    if (value < 1 || value > 4) return PKM_ERR_INVALID_ARG;
    g_opt_subbatches = value;
    return PKM_OK;
  }
  return PKM_ERR_INVALID_ARG;
}

int pkm_get_option(int option) {
  init_options();
  if (option == PKM_OPT_PATH) return g_opt_path.load();
  if (option == PKM_OPT_SUBBATCHES) return g_opt_subbatches.load();
  return PKM_ERR_INVALID_ARG;
}

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
  std::vector<TraceCall> keep;
  int rc = PKM_OK;
  for (const TraceCall& c : g_trace_pending) {
    if (c.pass != pass) {
      keep.push_back(c);
      continue;
    }
    for (const TraceSpan& sp : c.spans) {
      const cudaEvent_t a = c.events[sp.start], b = c.events[sp.stop];
      if (cudaEventSynchronize(b) != cudaSuccess) rc = PKM_ERR_CUDA;
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, a, b) != cudaSuccess) rc = PKM_ERR_CUDA;
      if (sp.stage < max_stages) stage_ms[sp.stage] += ms;
    }
    for (cudaEvent_t e : c.events) g_event_pool.push_back(e);
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
  const Opts o = current_options();
  if (for_backward == 4) {
    if (validate_shape(s) != PKM_OK || s->B < 2) return 0;
    return forward_train_ws(s, o, nullptr, nullptr, nullptr);
  }
  if (for_backward == 3) {
    if (validate_shape(s) != PKM_OK || 2 * s->B * s->H * static_cast<int64_t>(s->k) > 0x7fffffffLL)
      return 0;
    LayerArgs a{};
    a.B = s->B; a.H = s->H; a.dq = s->dq; a.n = s->n; a.k = s->k; a.v = s->v;
    return pkm::backward_full_ws_bytes(a, choose_path(s, o) == Path::kTensor, nullptr, nullptr);
  }
  if (for_backward == 2) {
    if (validate_usage(s) != PKM_OK) return 0;
    return pkm::kStatusBytes + align256(pkm::usage_bitmap_bytes(static_cast<int64_t>(s->n) * s->n));
  }
  if ((for_backward ? validate_common(s) : validate_shape(s)) != PKM_OK) return 0;
  return for_backward ? backward_ws(s, nullptr, nullptr) : forward_ws(s, o, nullptr, nullptr);
}

}  // extern "C"

namespace {

int backward_full_impl(const pkm_shape* s, bool bn_training, const void* x, const void* W_q,
                       const float* bn_mean, const float* bn_var, const float* bn_gamma,
                       const float* bn_beta, const void* subkeys, const void* values,
                       const int32_t* indices, const float* weights, const void* grad_out,
                       float* grad_x, float* grad_W_q, float* grad_bn_gamma, float* grad_bn_beta,
                       float* grad_subkeys, float* grad_values, float* grad_scores,
                       void* workspace, size_t workspace_bytes, void* stream) {
  int rc = validate_shape(s);
  if (rc != PKM_OK) return rc;
  if (bn_training && s->B == 1) return PKM_ERR_INVALID_ARG;
  // The sub-key grouping sorts two contributions per pick with 32-bit positions.
  if (2 * s->B * s->H * static_cast<int64_t>(s->k) > 0x7fffffffLL) return PKM_ERR_UNSUPPORTED;
  const bool tok = s->B > 0;
  if (!W_q || !bn_mean || !bn_var || !bn_gamma || !bn_beta || !subkeys || !values ||
      (tok && (!x || !indices || !weights || !grad_out)))
    return PKM_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W_q, bn_mean, bn_var, bn_gamma, bn_beta, subkeys, values, indices,
                        weights, grad_out, grad_x, grad_W_q, grad_bn_gamma, grad_bn_beta,
                        grad_subkeys, grad_values, grad_scores};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return PKM_ERR_UNSUPPORTED;
  const bool tensor = choose_path(s, current_options()) == Path::kTensor;
  LayerArgs a{s->B, s->d_model, s->H, s->dq, s->n, s->k, s->v, s->dtype, s->bn_eps,
              x, W_q, bn_mean, bn_var, bn_gamma, bn_beta, subkeys, values,
              static_cast<int*>(workspace), 0};
  const size_t need = pkm::backward_full_ws_bytes(a, tensor, nullptr, nullptr);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PKM_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!tok) {
    // Sums over no tokens: the requested parameter gradients are zero.
    const int64_t F = static_cast<int64_t>(s->H) * s->dq;
    const struct { float* p; int64_t count; } zero[] = {
        {grad_W_q, F * s->d_model}, {grad_bn_gamma, F}, {grad_bn_beta, F},
        {grad_subkeys, F * s->n}};
    for (const auto& z : zero)
      if (z.p && cudaMemsetAsync(z.p, 0, sizeof(float) * z.count, st) != cudaSuccess)
        return PKM_ERR_CUDA;
    return PKM_OK;
  }
  pkm::FullBackwardWs w;
  pkm::backward_full_ws_bytes(a, tensor, &w, static_cast<char*>(workspace));
  if (cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess) return PKM_ERR_CUDA;
  pkm::SideStream side;
  if (grad_values && side_stream(&side) != PKM_OK) return PKM_ERR_CUDA;
  Tracer tr(1);
  tr.begin(3, st);
  int launches = 0;
  const cudaError_t e = pkm::launch_backward_full(a, tensor, bn_training, indices, weights,
                                                  grad_out, grad_x, grad_W_q, grad_bn_gamma,
                                                  grad_bn_beta, grad_subkeys, grad_values,
                                                  grad_scores, w, side, st, &launches);
  tr.end(st);
  tr.finish(e == cudaSuccess, launches);
  return e == cudaSuccess ? PKM_OK : PKM_ERR_CUDA;
}

}  // namespace

extern "C" {

int pkm_backward(const pkm_shape* s, const void* x, const void* W_q, const float* bn_mean,
                 const float* bn_var, const float* bn_gamma, const float* bn_beta,
                 const void* subkeys, const void* values, const int32_t* indices,
                 const float* weights, const void* grad_out, float* grad_x, float* grad_W_q,
                 float* grad_bn_gamma, float* grad_bn_beta, float* grad_subkeys,
                 float* grad_values, float* grad_scores, void* workspace, size_t workspace_bytes,
                 void* stream) {
  return backward_full_impl(s, false, x, W_q, bn_mean, bn_var, bn_gamma, bn_beta, subkeys,
                            values, indices, weights, grad_out, grad_x, grad_W_q, grad_bn_gamma,
                            grad_bn_beta, grad_subkeys, grad_values, grad_scores, workspace,
                            workspace_bytes, stream);
}

int pkm_backward_train(const pkm_shape* s, const void* x, const void* W_q,
                       const float* batch_mean, const float* batch_var, const float* bn_gamma,
                       const float* bn_beta, const void* subkeys, const void* values,
                       const int32_t* indices, const float* weights, const void* grad_out,
                       float* grad_x, float* grad_W_q, float* grad_bn_gamma, float* grad_bn_beta,
                       float* grad_subkeys, float* grad_values, float* grad_scores,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return backward_full_impl(s, true, x, W_q, batch_mean, batch_var, bn_gamma, bn_beta, subkeys,
                            values, indices, weights, grad_out, grad_x, grad_W_q, grad_bn_gamma,
                            grad_bn_beta, grad_subkeys, grad_values, grad_scores, workspace,
                            workspace_bytes, stream);
}

int pkm_slot_usage(const pkm_shape* s, const int32_t* indices, unsigned long long* hits,
                   void* workspace, size_t workspace_bytes, void* stream) {
  const int rc = validate_usage(s);
  if (rc != PKM_OK) return rc;
  if (!hits || (s->B > 0 && !indices)) return PKM_ERR_INVALID_ARG;
  if ((indices && !aligned16(indices)) || (reinterpret_cast<uintptr_t>(hits) & 7u))
    return PKM_ERR_UNSUPPORTED;
  const int64_t slots = static_cast<int64_t>(s->n) * s->n;
  const size_t need = pkm::kStatusBytes + align256(pkm::usage_bitmap_bytes(slots));
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PKM_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(workspace);
  unsigned* bitmap = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + pkm::kStatusBytes);
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return PKM_ERR_CUDA;
  const cudaError_t e = pkm::launch_slot_usage(indices, s->B * s->H * static_cast<int64_t>(s->k),
                                               slots, bitmap, hits, status, st);
  {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (e == cudaSuccess) g_launches += s->B > 0 ? 2 : 1;
  }
  return e == cudaSuccess ? PKM_OK : PKM_ERR_CUDA;
}

}  // extern "C"

namespace {

// Checks shared by pkm_forward and pkm_forward_train (per-token tensors may be NULL
// when there are no tokens).
int validate_forward_args(const pkm_shape* s, const void* x, const void* W_q,
                          const float* bn_mean, const float* bn_var, const float* bn_gamma,
                          const float* bn_beta, const void* subkeys, const void* values,
                          const float* out, const int32_t* indices, const float* weights,
                          const float* scores) {
  int rc = validate_shape(s);
  if (rc != PKM_OK) return rc;
  const bool tok = s->B > 0;
  if (!W_q || !bn_mean || !bn_var || !bn_gamma || !bn_beta || !subkeys || !values ||
      (tok && (!x || !out || !indices || !weights)))
    return PKM_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W_q, bn_mean, bn_var, bn_gamma, bn_beta, subkeys, values, out,
                        indices, weights, scores};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return PKM_ERR_UNSUPPORTED;
  return PKM_OK;
}

// Small-batch path: the single cooperative kernel (only when pinned) rather than the
// three kernels.
bool small_fused_chosen(const pkm_shape* s, const Opts& o) {
  return o.path == PKM_PATH_SMALL_FUSED &&
         pkm::small_fused_supported(s->d_model, s->H, s->dq, s->n, s->v, s->dtype);
}

// The forward's launches for a validated call with B > 0. The status word is already
// cleared, or (clear_status) the small-batch three-kernel form clears it itself.
// Stages: 0 query network, 1 per-half scores + best 32, 2 candidate top-k + softmax +
// gather; the caller brackets stage 3 (the whole call).
cudaError_t run_forward(const pkm_shape* s, const LayerArgs& a, const ForwardWs& w, float* out,
                        int32_t* indices, float* weights, float* scores, cudaStream_t st,
                        Tracer& tr, int* nlaunch, const Opts& o, bool clear_status) {
  const void* x = a.x;
  cudaError_t e = cudaSuccess;
  int launches = 0;
  const Path path = choose_path(s, o);
  if (path == Path::kSmall) {
    tr.begin_here(2, st);
    if (small_fused_chosen(s, o)) {
      e = pkm::launch_forward_small_fused(a, w.q, w.list_s, w.list_i, w.part, out, indices,
                                          weights, scores, st);
      launches = 1;
    } else {
      e = pkm::launch_forward_small(a, w.q, w.list_s, w.list_i, out, indices, weights, scores,
                                    clear_status ? w.status : nullptr, st);
      launches = 3;
    }
    tr.end(st);
  } else if (path == Path::kSimt) {
    tr.begin_here(0, st);
    e = pkm::launch_query_bn_simt(a, w.q, st);
    tr.next(1, st);
    if (e == cudaSuccess) e = pkm::launch_subkey_topk_simt(a, w.q, w.list_s, w.list_i, st);
    tr.next(2, st);
    if (e == cudaSuccess)
      e = pkm::launch_select_gather(a, w.list_s, w.list_i, out, indices, weights, scores, st);
    tr.end(st);
    launches = 3;
  } else if (sub_batch_tokens(s->B, o) >= s->B) {
    // One batch: the three launches in order on the caller's stream.
    tr.begin_here(0, st);
    e = pkm::launch_query_tc(a, w.planes, st);
    tr.next(1, st);
    if (e == cudaSuccess) e = pkm::launch_score_topk_tc(a, w.planes, w.list_s, w.list_i, st);
    tr.next(2, st);
    if (e == cudaSuccess)
      e = pkm::launch_select_gather(a, w.list_s, w.list_i, out, indices, weights, scores, st);
    tr.end(st);
    launches = 3;
  } else {
    // Pipelined over sub-batches (PKM_OPT_SUBBATCHES > 1): the query network and
    // per-half search of sub-batch i+1 run on the caller's stream while the gather of
    // sub-batch i runs on the library's second stream (it is bound by HBM, the others
    // by the tensor cores and ALUs). The second stream waits for each sub-batch's
    // lists and the caller's stream waits for the last gather, so the call stays
    // ordered on `stream`.
    const int64_t sub = sub_batch_tokens(s->B, o);
    const int nsub = static_cast<int>((s->B + sub - 1) / sub);
    cudaStream_t aux;
    cudaEvent_t ev[5];
    if (aux_resources(nsub + 1, &aux, ev) != PKM_OK) return cudaErrorUnknown;
    const size_t xsz = s->dtype == PKM_F32 ? 4 : 2;
    const int64_t per_tok = static_cast<int64_t>(s->H) * 2 * pkm::kMaxK;
    for (int i = 0; i < nsub && e == cudaSuccess; ++i) {
      const int64_t t0 = i * sub;
      const int64_t bs = (s->B - t0 < sub) ? s->B - t0 : sub;
      LayerArgs ai = a;
      ai.B = bs;
      ai.x = static_cast<const char*>(x) + t0 * s->d_model * xsz;
      float* ls = w.list_s + t0 * per_tok;
      int* li = w.list_i + t0 * per_tok;
      tr.begin_here(0, st);
      e = pkm::launch_query_tc(ai, w.planes, st);
      tr.next(1, st);
      if (e == cudaSuccess) e = pkm::launch_score_topk_tc(ai, w.planes, ls, li, st);
      tr.end(st);
      if (e == cudaSuccess) e = cudaEventRecord(ev[i], st);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(aux, ev[i], 0);
      tr.begin(2, aux);
      const int64_t ok = t0 * s->H * static_cast<int64_t>(s->k);
      if (e == cudaSuccess)
        e = pkm::launch_select_gather(ai, ls, li, out + t0 * s->v, indices + ok, weights + ok,
                                      scores ? scores + ok : nullptr, aux);
      tr.end(aux);
      launches += 3;
    }
    // Always join, even after an error, so the caller's stream never runs ahead of
    // work already queued on the second stream.
    cudaError_t e2 = cudaEventRecord(ev[nsub], aux);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, ev[nsub], 0);
    if (e == cudaSuccess) e = e2;
  }
  *nlaunch += launches;
  return e;
}

}  // namespace

extern "C" {

int pkm_forward(const pkm_shape* s, const void* x, const void* W_q, const float* bn_mean,
                const float* bn_var, const float* bn_gamma, const float* bn_beta,
                const void* subkeys, const void* values, float* out, int32_t* indices,
                float* weights, float* scores, void* workspace, size_t workspace_bytes,
                void* stream) {
  int rc = validate_forward_args(s, x, W_q, bn_mean, bn_var, bn_gamma, bn_beta, subkeys, values,
                                 out, indices, weights, scores);
  if (rc != PKM_OK) return rc;
  const Opts o = current_options();
  const size_t need = forward_ws(s, o, nullptr, nullptr);
  if (!workspace || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PKM_ERR_WORKSPACE;
  if (s->B == 0) return PKM_OK;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ForwardWs w;
  forward_ws(s, o, &w, static_cast<char*>(workspace));
  LayerArgs a{s->B, s->d_model, s->H, s->dq, s->n, s->k, s->v, s->dtype, s->bn_eps,
              x, W_q, bn_mean, bn_var, bn_gamma, bn_beta, subkeys, values, w.status, 0};
  // The status word and the small-batch kernel's grid-barrier counter after it. The
  // small-batch three-kernel form clears the status word in its first kernel instead
  // (it does not use the counter): one operation less between back-to-back calls.
  const bool self_clear = choose_path(s, o) == Path::kSmall && !small_fused_chosen(s, o);
  if (!self_clear && cudaMemsetAsync(w.status, 0, 2 * sizeof(int), st) != cudaSuccess)
    return PKM_ERR_CUDA;
  Tracer tr(0);
  int launches = 0;
  tr.begin(3, st);
  const cudaError_t e =
      run_forward(s, a, w, out, indices, weights, scores, st, tr, &launches, o, self_clear);
  tr.end_here(st);  // the last stage's end, or a new event after the pipelined join
  tr.finish(e == cudaSuccess, launches);
  return e == cudaSuccess ? PKM_OK : PKM_ERR_CUDA;
}

int pkm_forward_train(const pkm_shape* s, const void* x, const void* W_q,
                      float* bn_running_mean, float* bn_running_var, const float* bn_gamma,
                      const float* bn_beta, float momentum, const void* subkeys,
                      const void* values, float* out, int32_t* indices, float* weights,
                      float* scores, float* batch_mean, float* batch_var, void* workspace,
                      size_t workspace_bytes, void* stream) {
  int rc = validate_forward_args(s, x, W_q, bn_running_mean, bn_running_var, bn_gamma, bn_beta,
                                 subkeys, values, out, indices, weights, scores);
  if (rc != PKM_OK) return rc;
  if (s->B == 1 || !batch_mean || !batch_var || !(momentum >= 0.f && momentum <= 1.f))
    return PKM_ERR_INVALID_ARG;
  if (!aligned16(batch_mean) || !aligned16(batch_var)) return PKM_ERR_UNSUPPORTED;
  const Opts o = current_options();
  const size_t need = forward_train_ws(s, o, nullptr, nullptr, nullptr);
  if (!workspace || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PKM_ERR_WORKSPACE;
  if (s->B == 0) return PKM_OK;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ForwardWs w;
  TrainWs tw;
  forward_train_ws(s, o, &w, &tw, static_cast<char*>(workspace));
  const int F = s->H * s->dq;
  // acc = x W_q^T without BatchNorm, its batch statistics (and the running-statistics
  // update), then the forward normalised by the batch statistics.
  LayerArgs raw{s->B, s->d_model, s->H, s->dq, s->n, s->k, s->v, s->dtype, s->bn_eps,
                x, W_q, bn_running_mean, bn_running_var, bn_gamma, bn_beta, subkeys, values,
                w.status, 1};
  LayerArgs a = raw;
  a.bn_mean = batch_mean;
  a.bn_var = batch_var;
  a.raw_acc = 0;
  if (cudaMemsetAsync(w.status, 0, 2 * sizeof(int), st) != cudaSuccess) return PKM_ERR_CUDA;
  Tracer tr(0);
  int launches = 0;
  tr.begin(3, st);
  tr.begin_here(0, st);
  const bool tensor = choose_path(s, o) == Path::kTensor;
  cudaError_t e = tensor ? pkm::launch_query_tc(raw, tw.acc, st)
                         : pkm::launch_query_bn_simt(raw, static_cast<float*>(tw.acc), st);
  if (e == cudaSuccess)
    e = pkm::launch_bn_batch_stats(tensor ? static_cast<const uint16_t*>(tw.acc) : nullptr,
                                   tensor ? nullptr : static_cast<const float*>(tw.acc), s->B, F,
                                   momentum, tw.part, batch_mean, batch_var, bn_running_mean,
                                   bn_running_var, st);
  tr.end(st);
  launches += 3;
  if (e == cudaSuccess)
    e = run_forward(s, a, w, out, indices, weights, scores, st, tr, &launches, o, false);
  tr.end_here(st);
  tr.finish(e == cudaSuccess, launches);
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
  const int64_t slots = static_cast<int64_t>(s->n) * s->n;
  // With both results asked for, the slot sort (ALU and L2 only) runs on the helper
  // stream while the kept-score gradients stream the picked value rows from HBM on the
  // caller's stream; the row sums (HBM read-modify-writes) follow on the caller's
  // stream once both are done. Two HBM-bound kernels side by side only share the
  // bandwidth, so they do not overlap each other.
  const bool split = grad_scores != nullptr;
  pkm::SideStream side;
  if (split && side_stream(&side) != PKM_OK) return PKM_ERR_CUDA;
  // Stages: 0 grad wrt kept scores, 1 slot grouping + row sums into grad_values,
  // 3 the whole call.
  Tracer tr(1);
  tr.begin(3, st);
  cudaError_t e = split ? pkm::side_fork(side, st) : cudaSuccess;
  const cudaStream_t ss = split ? side.st : st;
  tr.begin_here(1, ss);  // shares the call's first event unless on the helper stream
  if (e == cudaSuccess)
    e = pkm::launch_value_sort(s->B, s->H, s->k, slots, indices, w, status, ss);
  tr.end(ss);
  if (split) {
    tr.begin(0, st);
    if (e == cudaSuccess)
      e = pkm::launch_grad_scores(s->B, s->H, s->k, s->v, s->dtype, slots, values, indices,
                                  weights, grad_out, grad_scores, status, st);
    tr.end(st);
    // Always join, even after an error.
    const cudaError_t e2 = pkm::side_join(side, st);
    if (e == cudaSuccess) e = e2;
  }
  tr.begin(1, st);
  if (e == cudaSuccess)
    e = pkm::launch_value_segments(s->B, s->H, s->k, s->v, s->dtype, slots, weights, grad_out,
                                   grad_values, w, st);
  tr.end(st);
  tr.end_here(st);
  tr.finish(e == cudaSuccess, pkm::backward_values_launches(static_cast<int64_t>(s->n) * s->n,
                                                           grad_scores != nullptr, true));
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
