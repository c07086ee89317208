// pkm_kernels.h -- internal launcher interface between the C ABI (pkm_api.cu) and
// the kernels. Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>


namespace pkm {

struct LayerArgs {
  int64_t B;
  int d_model, H, dq, n, k, v, dtype;
  float bn_eps;
  const void* x;
  const void* W_q;
  const float* bn_mean;
  const float* bn_var;
  const float* bn_gamma;
  const float* bn_beta;
  const void* subkeys;
  const void* values;
  int* status;   // device status word
  int raw_acc;   // query kernels: write acc = x W_q^T without BatchNorm
};

// SIMT query network + per-half search (pkm_simt.cu).
cudaError_t launch_query_bn_simt(const LayerArgs& a, float* q, cudaStream_t st);
size_t subkey_topk_simt_smem(int dq);
cudaError_t launch_subkey_topk_simt(const LayerArgs& a, const float* q, float* list_s,
                                    int* list_i, cudaStream_t st);

// Candidate top-k + softmax + value gather (pkm_select_gather.cu).
bool select_gather_supported(int H, int k, int v, int dtype);
cudaError_t launch_select_gather(const LayerArgs& a, const float* list_s, const int* list_i,
                                 float* out, int* indices, float* weights, float* scores,
                                 cudaStream_t st);

// Value backward (pkm_backward.cu).
struct BackwardWs {
  // Counting sort (launch_counting_sort: the full backward's sub-key grouping).
  int* counts;    // [slots]
  int* offsets;   // [slots + 1]
  int* partials;  // [scan blocks + 1]
  int* order;     // [E] ids grouped by key
  // Value gradient: stable radix sort of the picks by slot, then work lists.
  int* keys[2];   // [E] slot ids, ping-pong between sort passes
  int* picks[2];  // [E] pick ids (t*H*k + h*k + j), ping-pong
  int* hist;      // [2048][sort blocks] digit counts, then their scan over the blocks
  int* ctr;       // [4] work-list lengths: items, huge groups, scratch rows; [64, 2112)
                  // the radix pass's digit totals
  int4* items;    // [max_items] {start, picks, slot, scratch row or -1}
  int4* huge;     // [max_huge] {slot, first scratch row, rows, 0}
  float* scratch; // [max_chunks][v] partial row sums of huge groups
  int64_t max_items, max_huge, max_chunks;
};
size_t backward_ws_bytes(int64_t B, int H, int k, int64_t slots, int v, BackwardWs* carve,
                         char* base);

// Value-gradient geometry: radix-sort tile, the largest group a warp sums inline, the
// picks per work item; and the workspace bytes for E picks and rows of v floats, laid
// out as backward_ws_bytes carves them (status word, list lengths, two key and two
// pick buffers, digit counts, work lists, partial rows). A compile-time function so
// that the fixed scratch of pkm_backward_values_noalloc is sized by the same sum.
constexpr int kSortTileKeys = 4096;
constexpr int kValueSmallGroup = 256;
constexpr int kValueChunk = 4096;
constexpr size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
constexpr int64_t value_bwd_max_items(int64_t E) {
  return E / (kValueSmallGroup + 1) + E / (kValueChunk / 2) + 2;
}
constexpr int64_t value_bwd_max_huge(int64_t E) { return E / (kValueChunk + 1) + 1; }
constexpr int64_t value_bwd_max_chunks(int64_t E) { return E / (kValueChunk / 2) + 1; }
constexpr size_t value_bwd_ws_bytes(int64_t E, int v) {
  return 256 + 8448 + 4 * round256(4 * static_cast<size_t>(E > 0 ? E : 1)) +
         round256(4 * 2048 * static_cast<size_t>(((E > 0 ? E : 1) + kSortTileKeys - 1) /
                                                 kSortTileKeys)) +
         round256(16 * static_cast<size_t>(value_bwd_max_items(E))) +
         round256(16 * static_cast<size_t>(value_bwd_max_huge(E))) +
         round256(4 * static_cast<size_t>(value_bwd_max_chunks(E)) *
                  static_cast<size_t>(v > 0 ? v : 1));
}
// Kernels one pkm_backward_values call launches.
int backward_values_launches(int64_t slots, bool grad_scores, bool grad_values);
// B1: gradients of the kept scores into grad_scores.
cudaError_t launch_grad_scores(int64_t B, int H, int k, int v, int dtype, int64_t slots,
                               const void* values, const int* indices, const float* weights,
                               const void* grad_out, float* grad_scores, int* status,
                               cudaStream_t st);
// B2: picks sorted by slot (launch_value_sort: indices only), then each slot's weighted
// grad_out rows added to grad_values (launch_value_segments, same stream order after the
// sort); launch_value_rows issues both. Independent of B1.
cudaError_t launch_value_sort(int64_t B, int H, int k, int64_t slots, const int* indices,
                              const BackwardWs& ws, int* status, cudaStream_t st);
cudaError_t launch_value_segments(int64_t B, int H, int k, int v, int dtype, int64_t slots,
                                  const float* weights, const void* grad_out, float* grad_values,
                                  const BackwardWs& ws, cudaStream_t st);
cudaError_t launch_value_rows(int64_t B, int H, int k, int v, int dtype, int64_t slots,
                              const int* indices, const float* weights, const void* grad_out,
                              float* grad_values, const BackwardWs& ws, int* status,
                              cudaStream_t st);

// A second stream for work of a call that is independent of the rest of it: `fork` is
// recorded on the caller's stream and waited on by the side stream before the side
// work; `join` is recorded on the side stream after it and waited on by the caller's
// stream, so the call stays ordered on the caller's stream.
struct SideStream {
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
inline cudaError_t side_fork(const SideStream& s, cudaStream_t st) {
  cudaError_t e = cudaEventRecord(s.fork, st);
  return e == cudaSuccess ? cudaStreamWaitEvent(s.st, s.fork, 0) : e;
}
inline cudaError_t side_join(const SideStream& s, cudaStream_t st) {
  cudaError_t e = cudaEventRecord(s.join, s.st);
  return e == cudaSuccess ? cudaStreamWaitEvent(st, s.join, 0) : e;
}

cudaError_t launch_counting_sort(const int* keys, int64_t E, int64_t slots, const BackwardWs& ws,
                                 int* status, cudaStream_t st);

// Full backward (pkm_backward_full.cu).
struct FullBackwardWs {
  BackwardWs values;  // value-gradient grouping
  float* g_s;         // [B][H][k] kept-score gradients
  float* acc;         // [B][H*dq] x W_q^T
  float* q;           // [B][H*dq] BatchNorm(acc)
  float* g_q;         // [B][H*dq] dL/dq
  float* g_acc;       // [B][H*dq] dL/dacc
  void* planes;       // tensor path: acc as three bf16 planes
  int* targets;       // [B*H*k][2] sub-key row of each pick's halves (-1: merged away)
  float* coef;        // [B*H*k][2] summed kept-score gradient of that row
  BackwardWs sub;     // sub-key grouping
  float* bn_part;     // BatchNorm column-sum partials
  float* bn_sums;     // [2][H*dq] sum_t dL/dq, sum_t dL/dq xhat
};
size_t backward_full_ws_bytes(const LayerArgs& a, bool tensor_path, FullBackwardWs* w, char* base);
cudaError_t launch_backward_full(const LayerArgs& a, bool tensor_path, bool bn_training,
                                 const int* indices,
                                 const float* weights, const void* grad_out, float* grad_x,
                                 float* grad_W, float* grad_gamma, float* grad_beta,
                                 float* grad_subkeys, float* grad_values, float* grad_scores,
                                 const FullBackwardWs& w, const SideStream& side,
                                 cudaStream_t st, int* launches);

// BatchNorm in training mode (pkm_bn_train.cu). Batch statistics of acc (three bf16
// planes, or fp32 when planes is null) in chunks of kStatChunk tokens; part holds
// [chunks][2][F] doubles.
constexpr int kStatChunk = 128;
cudaError_t launch_bn_batch_stats(const uint16_t* planes, const float* acc, int64_t B, int F,
                                  float momentum, double* part, float* batch_mean,
                                  float* batch_var, float* running_mean, float* running_var,
                                  cudaStream_t st);
cudaError_t launch_bn_train_dacc(const float* g_q, const float* acc, const float* mean,
                                 const float* var, const float* gamma, const float* sums,
                                 float eps, int64_t B, int F, float* g_acc, uint16_t* g_planes,
                                 cudaStream_t st);

// Small-batch forward (pkm_small.cu): B <= kSmallMaxB tokens, three launches that
// spread the parameters over every SM. Workspace: q fp32 [B][H*dq] and chunk lists of
// small_chunk_entries() (score, id) entries.
constexpr int kSmallMaxB = 512;
// bf16 layers whose query network and per-half scores the small-batch kernels run as
// tensor-core tiles above decode mode (d_model and dq/2 multiples of 32, dq/2 <= 256).
bool small_mma_shape(int d_model, int dq, int dtype);
// Largest batch the automatic choice sends to the small-batch kernels: the measured
// crossover with the tensor-core path (device time per call, CUDA-graph replay). With
// the tensor-core tiles: about 390 tokens with H = 4 on the 1024^2 layer (118 vs 120 us
// at 384, 127 vs 120 at 416) and 420 on the 512^2 layer (93 vs 104 us at 384, 110 vs
// 103 at 448), about 250 with H = 8 on the wide layer (197 vs 224 us at 224, 228 vs 225
// at 256). Without them (CUDA-core query and scores per token) 112 and 96 tokens.
inline int small_auto_max_b(int H, int d_model, int dq, int dtype) {
  if (small_mma_shape(d_model, dq, dtype)) return H > 4 ? 240 : 384;
  return H > 4 ? 96 : 112;
}
bool small_supported(int64_t B, int d_model, int H, int dq, int n, int k, int v, int dtype);
size_t small_chunk_entries(int64_t B, int H, int n);
// clear: the call's status word, zeroed by the first kernel once the stream's earlier
// work has finished (instead of a memset before the launch), or null.
cudaError_t launch_forward_small(const LayerArgs& a, float* q, float* chunk_s, int* chunk_i,
                                 float* out, int* idx, float* w, float* sc, int* clear,
                                 cudaStream_t st);
// The same forward as one cooperative launch with grid-wide barriers (one CTA per SM);
// the barrier counter is the int after a.status, zeroed by the caller. `part` holds
// [B][H][v] floats followed by B unsigned per-token counts (zeroed by the kernel). Taken
// only when pinned (PKM_OPT_PATH small_fused): the three kernels measured faster at
// every batch size (12.1 vs 22.6 us for one token, 18.3 vs 24.6 for 16, 25.0 vs 30.7
// for 32 on the 1024^2 layer), their first kernel overlapping the previous call's last
// through programmatic launch and clearing the status word itself, where the single
// kernel needs a memset of its barrier counter before each launch.
bool small_fused_supported(int d_model, int H, int dq, int n, int v, int dtype);
cudaError_t launch_forward_small_fused(const LayerArgs& a, float* q, float* chunk_s,
                                       int* chunk_i, float* part, float* out, int* idx, float* w,
                                       float* sc, cudaStream_t st);

// 16-byte vectors of a v-wide row each lane of a warp holds, rounded up to the kernel
// instantiations (1, 2, 4 or 8); 0 when a row is wider than 8 vectors per lane.
inline int row_vecs_per_lane(int v, int dtype) {
  const int per = dtype == 0 ? 4 : 8;
  const int m = (v / per + 31) / 32;
  if (m <= 1) return 1;
  if (m <= 2) return 2;
  if (m <= 4) return 4;
  if (m <= 8) return 8;
  return 0;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device, size)
// (pkm_util.cu).
cudaError_t set_max_smem(const void* func, size_t bytes);

// Memory utilisation (pkm_usage.cu).
size_t usage_bitmap_bytes(int64_t slots);
cudaError_t launch_slot_usage(const int* indices, int64_t E, int64_t slots, unsigned* bitmap,
                              unsigned long long* hits, int* status, cudaStream_t st);

}  // namespace pkm
