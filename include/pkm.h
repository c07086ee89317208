/*
 * pkm.h -- C ABI of the product-key memory (PKM) layer library for NVIDIA B200
 * (sm_100a). Library file: libpkm.so (product_key_memory_b200/libpkm.so).
 *
 * The layer is the one of "Large Memory Layers with Product Keys" (Lample et al.,
 * 2019). Per token and head (gptget.net summary of that paper, Methodology and the
 * Deep Analysis / Methodology list; "Product Keys Give Transformers Million-Slot
 * Memory Layers", sections "Why top-k of each half is enough" and "Implied keys
 * vs stored sub-keys"):
 *   q      = BN(x W_q^T)                query network: linear map + inference BatchNorm
 *   q1, q2 = the two halves of q_h      (dq/2 each)
 *   s1, s2 = q1 C_h^T, q2 C'_h^T        score every sub-key of each codebook
 *   keep the top-k of s1 and of s2
 *   score(i, j) = s1[i] + s2[j] over the k x k pairs; keep the exact top-k keys;
 *   the key (i, j) has flat slot i*n + j
 *   w      = softmax over the k kept scores
 *   out[t] = sum over heads h, kept j of w[t,h,j] * V[slot[t,h,j]]
 * Orders: every top-k is by score descending, ties to the lower id (sub-key id in
 * the per-half lists, flat slot in the final list). Output lists are sorted in that
 * order.
 *
 * Conventions for every entry point:
 *   - Tensors are caller-owned DEVICE pointers, row-major and contiguous, 16-byte
 *     aligned. The library allocates no device memory: scratch is the caller's
 *     `workspace` (pkm_backward_values_noalloc alone uses a fixed array compiled
 *     into the library).
 *   - Persistent state the library keeps: two process-wide option values
 *     (pkm_set_option), the tensor-map encoder's address and the SM count (looked
 *     up once), each kernel's raised shared-memory limit, and, only while tracing
 *     is on, a pool of timing events. A forward pipelined over sub-batches
 *     (PKM_OPT_SUBBATCHES > 1) also creates, on first use per device, one helper
 *     stream and a pool of ordering events; the default forward (one batch) uses
 *     neither and issues its three kernels on `stream` alone.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All work is enqueued asynchronously and ordered on it; no call synchronises.
 *   - Arguments are validated before anything is launched: a call that returns an
 *     error has launched nothing and written nothing.
 *   - Kernels that wait on hardware barriers give up after a bounded time (1 s)
 *     and record it in the workspace's status word, as do gathers that meet a slot
 *     id outside [0, n*n) (skipped); pkm_device_status() waits for the stream and
 *     returns PKM_ERR_DEVICE if either happened.
 */
#ifndef PKM_H_
#define PKM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of x, W_q, sub-keys, values and grad_out. BN vectors, scores,
 * weights, out and gradients are always fp32. */
typedef enum { PKM_F32 = 0, PKM_BF16 = 1 } pkm_dtype;

/* Status codes. */
enum {
  PKM_OK = 0,
  PKM_ERR_INVALID_ARG = -1, /* NULL pointer, size out of range, k > n, odd dq, n*n > 2^31-1 */
  PKM_ERR_UNSUPPORTED = -2, /* valid layer this library does not run (k > 32, v not a multiple of
                               16 bytes, misaligned pointer) */
  PKM_ERR_WORKSPACE = -3,   /* workspace NULL or smaller than pkm_workspace_size() */
  PKM_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
  PKM_ERR_DEVICE = -5       /* a kernel recorded a device-side error: a bounded wait ran
                               out, or a slot id outside [0, n*n) was read */
};

/* Layer sizes. */
typedef struct {
  int64_t B;       /* tokens (rows of x); 0 is allowed, launches nothing, and then the
                      per-token pointers (x, out, indices, weights, scores, grad_out,
                      grad_scores) may be NULL */
  int32_t d_model; /* input width of the query network */
  int32_t H;       /* heads */
  int32_t dq;      /* query size per head, even; each half is dq/2 */
  int32_t n;       /* sub-keys per codebook; the memory has n*n slots */
  int32_t k;       /* keys kept per half and per head, 1 <= k <= min(n, 32) */
  int32_t v;       /* value width */
  int32_t dtype;   /* pkm_dtype of x, W_q, sub-keys, values, grad_out */
  float bn_eps;    /* BatchNorm epsilon (PyTorch's default is 1e-5) */
} pkm_shape;

/*
 * Bytes of workspace pkm_forward (for_backward = 0), pkm_backward_values
 * (for_backward = 1), pkm_slot_usage (for_backward = 2), pkm_backward or
 * pkm_backward_train (for_backward = 3) or pkm_forward_train (for_backward = 4) needs
 * for this shape; 0 if the shape is invalid.
 */
size_t pkm_workspace_size(const pkm_shape* s, int for_backward);

/*
 * Forward pass of the PKM layer (the steps listed at the top of this file).
 *
 *   x        [B][d_model]            dtype
 *   W_q      [H*dq][d_model]         dtype   (q = x W_q^T; no bias)
 *   bn_mean, bn_var, bn_gamma, bn_beta  [H*dq] fp32 running statistics and affine
 *            q = (acc - mean) / sqrt(var + bn_eps) * gamma + beta
 *   subkeys  [H][2][n][dq/2]         dtype   ([h][0] = C scores q1, [h][1] = C' scores q2)
 *   values   [n*n][v]                dtype   (one table shared by all heads)
 * Outputs (overwritten):
 *   out      [B][v]     fp32   sum over heads of the weighted value rows
 *   indices  [B][H][k]  int32  flat slots i*n + j, best first
 *   weights  [B][H][k]  fp32   softmax of the kept scores
 *   scores   [B][H][k]  fp32   kept key scores s1[i] + s2[j]; may be NULL
 * workspace: device scratch of at least pkm_workspace_size(s, 0) bytes, 256-byte
 *   aligned; its contents on entry do not matter.
 * Small batches take the small-batch path, which spreads W_q, the sub-keys and the
 * heads over all SMs for latency: up to 384 tokens with H <= 4 and 240 with H <= 8 on
 * bf16 layers with d_model and dq/2 multiples of 32 and dq/2 <= 256 (whose query
 * network and per-half scores there run as warp-level tensor-core tiles of 16 tokens),
 * up to 112 / 96 tokens otherwise; a pinned form (PKM_OPT_PATH small_fused /
 * small_split) takes up to 512 tokens for any H <= 8. By default it is three kernels
 * that overlap through programmatic dependent launch on `stream`: the first waits on
 * the device for the stream's earlier work and clears the status word itself, so
 * back-to-back calls overlap too. PKM_PATH_SMALL_FUSED runs it as one cooperative
 * kernel instead (one block per SM, its query, scoring and gather phases separated by
 * grid-wide barriers whose waits are bounded like the pipelines'). Up to 4 tokens
 * with H <= 4 (8 tokens on layers without the tensor-core tiles) the query and
 * scoring stages give a warp one W_q row or 8 sub-keys for all tokens, its lanes
 * splitting the dot products (rows of 16-byte multiples). Larger batches run
 * three kernels on `stream` (query network, per-half scores and top-k, candidate
 * top-k + softmax + gather). With PKM_OPT_SUBBATCHES > 1, large batches of
 * tensor-core shapes are processed in up to that many sub-batches; the value gather
 * of one sub-batch then runs on the library's helper stream (one per device) while
 * the next sub-batch is scored on `stream`. Event waits order both
 * ways, so all of the call's work is complete when `stream` reaches the point after
 * the call.
 * Returns PKM_OK or a status code above.
 */
int pkm_forward(const pkm_shape* s, const void* x, const void* W_q, const float* bn_mean,
                const float* bn_var, const float* bn_gamma, const float* bn_beta,
                const void* subkeys, const void* values, float* out, int32_t* indices,
                float* weights, float* scores, void* workspace, size_t workspace_bytes,
                void* stream);

/*
 * Sparse value backward ("trained end-to-end with sparse updates"; only the kept
 * slots receive gradient). With L = <grad_out, out>:
 *   grad_scores[t,h,j] = w_j * (g_j - sum_l w_l g_l),  g_j = <grad_out[t], V[slot_j]>
 *   grad_values[slot] += sum over picks (t,h,j) of that slot of w[t,h,j] * grad_out[t]
 *
 *   values      [n*n][v]   dtype
 *   indices     [B][H][k]  int32  (as written by pkm_forward; each in [0, n*n))
 *   weights     [B][H][k]  fp32
 *   grad_out    [B][v]     dtype
 *   grad_values [n*n][v]   fp32   ACCUMULATED into (the caller zeroes it once)
 *   grad_scores [B][H][k]  fp32   overwritten; may be NULL
 * Picks are grouped by slot with a stable radix sort, so each slot's picks are summed
 * in pick order and each touched row is read and written once, whatever the number of
 * picks that hit it (large groups are split over several blocks whose partial sums are
 * added in a fixed order). The result is bit-for-bit the same on every run, and no
 * row is updated with atomics. Slot ids outside [0, n*n) are skipped and counted in
 * the status word (PKM_ERR_DEVICE).
 * Only B, H, n, k, v and dtype of the shape are read; d_model, dq and bn_eps are
 * ignored.
 * With grad_scores requested, the sort of the picks by slot runs on the library's
 * helper stream (one per device, highest priority) while grad_scores is computed on
 * `stream`, and the row sums follow on `stream`; event waits order both ways, so all
 * of the call's work is complete when `stream` reaches the point after the call
 * (CUDA-graph capture of `stream` takes the helper stream's work in with it).
 * workspace: at least pkm_workspace_size(s, 1) bytes, 256-byte aligned.
 */
int pkm_backward_values(const pkm_shape* s, const void* values, const int32_t* indices,
                        const float* weights, const void* grad_out, float* grad_values,
                        float* grad_scores, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * Full backward of the layer ("Large Memory Layers with Product Keys", Methodology:
 * the memory is trained end-to-end with the rest of the network). The top-k choice
 * is piecewise constant, so the picks of the forward are held fixed. With
 * L = <grad_out, out>, g_c the kept-score gradients of pkm_backward_values, key
 * (i, i') = slot i*n + i', acc = x W_q^T and s = gamma / sqrt(var + eps):
 *   dL/dq1_h = sum_j g_c[j] C_h[i_j],  dL/dq2_h = sum_j g_c[j] C'_h[i'_j]
 *   grad_subkeys[h][0][i] = sum over picks with left sub-key i of g_c q1_h (C' alike)
 *   grad_bn_beta = sum_t dL/dq,  grad_bn_gamma = sum_t dL/dq (acc - mean) / sqrt(var + eps)
 *   grad_W_q = (dL/dq s)^T x,    grad_x = (dL/dq s) W_q
 * Inputs are those of pkm_forward plus the forward's indices and weights and
 * grad_out [B][v] (dtype). Outputs, each fp32 and each may be NULL (not computed):
 *   grad_x        [B][d_model]        overwritten
 *   grad_W_q      [H*dq][d_model]     overwritten
 *   grad_bn_gamma [H*dq], grad_bn_beta [H*dq]  overwritten (inference BatchNorm:
 *                 the running statistics are constants and get no gradient)
 *   grad_subkeys  [H][2][n][dq/2]     overwritten
 *   grad_values   [n*n][v]            ACCUMULATED into, as in pkm_backward_values
 *   grad_scores   [B][H][k]           overwritten
 * acc is recomputed with the forward's query kernel (no BatchNorm), so the caller
 * keeps nothing from the forward beyond indices and weights. Sums over tokens are
 * in fp32 in a fixed order except sub-key rows shared by two 32-pick windows, which
 * are added atomically. Slot ids outside [0, n*n) are skipped and counted in the
 * status word. 2*B*H*k must stay below 2^31 (PKM_ERR_UNSUPPORTED otherwise: the
 * sub-key grouping sorts two contributions per pick with 32-bit positions).
 * The other gradients' chain of kernels runs on the library's helper stream (highest
 * priority) and grad_values, when requested, on `stream` beside it, joined back into
 * `stream` before the call's end.
 * workspace: at least pkm_workspace_size(s, 3) bytes, 256-byte aligned.
 */
int pkm_backward(const pkm_shape* s, const void* x, const void* W_q, const float* bn_mean,
                 const float* bn_var, const float* bn_gamma, const float* bn_beta,
                 const void* subkeys, const void* values, const int32_t* indices,
                 const float* weights, const void* grad_out, float* grad_x, float* grad_W_q,
                 float* grad_bn_gamma, float* grad_bn_beta, float* grad_subkeys,
                 float* grad_values, float* grad_scores, void* workspace, size_t workspace_bytes,
                 void* stream);

/*
 * Forward with BatchNorm in training mode ("Large Memory Layers with Product Keys",
 * Methodology: batch normalization in the query network; while the model trains, the
 * batch's own statistics normalise it, after Ioffe and Szegedy 2015):
 *   acc = x W_q^T,  mean_B = (1/B) sum_t acc[t],  var_B = (1/B) sum_t (acc[t] - mean_B)^2
 *   q = (acc - mean_B) / sqrt(var_B + eps) * gamma + beta, then as pkm_forward.
 * The running statistics move towards the batch's (PyTorch's convention):
 *   bn_running_mean <- (1 - momentum) bn_running_mean + momentum mean_B
 *   bn_running_var  <- (1 - momentum) bn_running_var  + momentum var_B B / (B - 1)
 * Arguments as pkm_forward, with bn_running_mean / bn_running_var [H*dq] fp32 updated
 * in place, momentum in [0, 1], and batch_mean / batch_var [H*dq] fp32 written: the
 * statistics that normalised the batch (biased variance), which pkm_backward_train
 * takes. B = 1 is rejected (PKM_ERR_INVALID_ARG: one token has no variance); B = 0
 * launches nothing and leaves every array as it was. Statistics are summed in fp64 in
 * chunks of 128 tokens and merged in chunk order (deterministic).
 * workspace: at least pkm_workspace_size(s, 4) bytes, 256-byte aligned.
 */
int pkm_forward_train(const pkm_shape* s, const void* x, const void* W_q,
                      float* bn_running_mean, float* bn_running_var, const float* bn_gamma,
                      const float* bn_beta, float momentum, const void* subkeys,
                      const void* values, float* out, int32_t* indices, float* weights,
                      float* scores, float* batch_mean, float* batch_var, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * pkm_backward for a forward run by pkm_forward_train: batch_mean / batch_var are the
 * statistics it wrote, and the gradient also flows through them (the backward of
 * batch normalisation):
 *   dL/dacc = gamma / sqrt(var_B + eps) (dL/dq - (1/B) sum_t dL/dq
 *                                        - xhat (1/B) sum_t dL/dq xhat),
 *   xhat = (acc - mean_B) / sqrt(var_B + eps).
 * dL/dgamma, dL/dbeta and everything else as in pkm_backward. B = 1 is rejected.
 * workspace: at least pkm_workspace_size(s, 3) bytes, 256-byte aligned.
 */
int pkm_backward_train(const pkm_shape* s, const void* x, const void* W_q,
                       const float* batch_mean, const float* batch_var, const float* bn_gamma,
                       const float* bn_beta, const void* subkeys, const void* values,
                       const int32_t* indices, const float* weights, const void* grad_out,
                       float* grad_x, float* grad_W_q, float* grad_bn_gamma, float* grad_bn_beta,
                       float* grad_subkeys, float* grad_values, float* grad_scores,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * pkm_backward_values without a workspace. The pages have no counterpart: this is
 * a convenience of this library. It is for callers that cannot allocate device
 * memory where they run the backward (a runtime that hands out all device memory
 * from its own pool and forbids other allocations while it executes, or a plugin
 * host that passes device pointers but no allocator). Arguments and results are
 * those of pkm_backward_values; the caller still passes inputs and outputs.
 *
 * Scratch: one fixed device array of about 44.2 MiB inside libpkm.so, held on every
 * GPU that loads the library until the process exits. Limits: n*n <= 1,048,576 slots,
 * B*H*k <= 2,097,152 picks and v <= 2048; larger shapes return PKM_ERR_UNSUPPORTED
 * before any launch. The call allocates nothing (no cudaMalloc, no library allocator).
 * The first call on a device looks up the array's device address with that device
 * current; make that first call before any stream capture. All calls share the
 * one array (each call clears what must start at zero), so calls that overlap on
 * the GPU -- on different streams, or from different threads -- race and must
 * not be issued. Slot ids outside [0, n*n) are skipped as in pkm_backward_values,
 * but the status word is not readable through pkm_device_status.
 */
int pkm_backward_values_noalloc(const pkm_shape* s, const void* values, const int32_t* indices,
                                const float* weights, const void* grad_out, float* grad_values,
                                float* grad_scores, void* stream);

/*
 * Memory utilisation of one batch ("Large Memory Layers with Product Keys", gptget.net
 * summary, Key Results: BatchNorm in the query network raises the share of memory
 * slots in use above 80 %): the number of distinct slots among the B*H*k picks.
 *   indices  [B][H][k] int32, as written by pkm_forward
 *   hits     one device uint64, overwritten with the count
 * Only B, H, n and k of the shape are read. Ids outside [0, n*n) are not counted and
 * set the status word (PKM_ERR_DEVICE).
 * workspace: at least pkm_workspace_size(s, 2) bytes (status word + one bit per slot).
 */
int pkm_slot_usage(const pkm_shape* s, const int32_t* indices, unsigned long long* hits,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, reads the status word that the kernels of the last call
 * on this workspace wrote (each call clears it when it starts), clears it and
 * returns PKM_OK, PKM_ERR_DEVICE or PKM_ERR_CUDA. This is the only entry point
 * that blocks the host.
 */
int pkm_device_status(void* workspace, void* stream);

/*
 * Stage timing (a measurement aid; the pages have no counterpart). While enabled,
 * every kernel a call launches is bracketed by two CUDA events recorded on the stream
 * it runs on, and so is the whole call (on `stream`). Forward stages: 0 query network,
 * 1 per-half scores and best 32, 2 candidate top-k + softmax + value gather, 3 the
 * whole call. Backward stages: 0 grad wrt kept scores, 1 slot grouping and row sums,
 * 3 the whole call. The events are owned by the library (host-side handles only).
 * pkm_trace_read waits for the recorded events of `pass` (0 forward, 1 backward),
 * writes the summed milliseconds per stage into stage_ms[0..max_stages) (a stage that
 * runs several launches per call, or overlaps another stage, sums their own
 * durations), the number of traced calls into *calls, and the number of kernels the
 * library launched since the last read (all passes, traced or not) into *launches;
 * then forgets them. Returns PKM_OK, PKM_ERR_INVALID_ARG or PKM_ERR_CUDA.
 */
int pkm_trace_enable(int on);
int pkm_trace_read(int pass, double* stage_ms, int max_stages, int64_t* calls,
                   int64_t* launches);

/*
 * Implementation switches (a convenience of this library; the pages have no
 * counterpart). Process-wide, for every device; a change applies to calls made after
 * it. The environment variables PKM_PATH (auto | tc | simt | small_fused | small_split) and
 * PKM_SUBBATCHES (1..4)
 * give the initial values and are read once, at the first call that needs them.
 *   PKM_OPT_PATH        PKM_PATH_AUTO (default): the small-batch kernels for small
 *                       batches (see pkm_forward), else the tensor-core kernels where
 *                       the layer fits
 *                       their tiles (bf16, d_model and dq/2 multiples of 64, n a
 *                       multiple of 256, H*dq <= 4096), else the CUDA-core kernels;
 *                       PKM_PATH_TC: never the small-batch kernels;
 *                       PKM_PATH_SIMT: always the CUDA-core kernels;
 *                       PKM_PATH_SMALL_FUSED: the small-batch path for every batch
 *                       it supports (up to 512 tokens), as the one cooperative
 *                       kernel;
 *                       PKM_PATH_SMALL_SPLIT: the same, as the three kernels.
 *   PKM_OPT_SUBBATCHES  1 (default) to 4: sub-batches of the pipelined tensor-core
 *                       forward (see pkm_forward). The forward's workspace size
 *                       depends on it: query it after setting the option.
 * pkm_set_option returns PKM_OK or PKM_ERR_INVALID_ARG (unknown option or value);
 * pkm_get_option returns the current value or PKM_ERR_INVALID_ARG.
 */
enum { PKM_OPT_PATH = 0, PKM_OPT_SUBBATCHES = 1 };
enum {
  PKM_PATH_AUTO = 0,
  PKM_PATH_TC = 1,
  PKM_PATH_SIMT = 2,
  PKM_PATH_SMALL_FUSED = 3,
  PKM_PATH_SMALL_SPLIT = 4
};
int pkm_set_option(int option, int value);
int pkm_get_option(int option);

/* Static string for a status code. */
const char* pkm_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* PKM_H_ */
