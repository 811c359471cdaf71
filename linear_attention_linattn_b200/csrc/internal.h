// Host-side declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "linattn.h"

namespace linattn {

// Launches `kern` on `st` with programmatic stream serialization: it may start while the
// previous kernel on the stream finishes (it must call grid_dependency_wait() before reading
// that kernel's results), so its set-up and its first loads of the inputs overlap that tail.
template <typename... KArgs, typename... Args>
cudaError_t launch_programmatic(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t st, Args &&...args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- forward dispatch shared by the entry points (api.cu) ---------------------------------
// Checks shared by every forward entry point: pointers (non-null, 16-byte aligned), the causal
// flag, the dtype and the sizes.  Limits keep every grid and TMA coordinate inside 32 bits.
linattn_status check_forward_args(const void *q, const void *k, const void *v, const void *out,
                                  int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                                  linattn_dtype dtype);
// What one forward pass needs: the tensor-core path's tokens per work item (0 on the fp32
// path) and the bytes of temporary state.
struct ForwardPlan {
  int64_t seg = 0;
  size_t ws_bytes = 0;
};
// dk: feature dimension of q, k (= d unless they are random features); d: value dimension.
// seg_len: tokens per work item of the tensor-core path, a multiple of 128; 0 picks the default.
ForwardPlan plan_forward(int64_t heads, int64_t n, int dk, int d, int causal, int is_bf16,
                         int64_t seg_len);
// Enqueues the pass `p` describes on `st`, with the caller's workspace (at least p.ws_bytes)
// and the word that bounded waits report a give-up in.  init_S / init_z (nullable): the state
// before each head's first token (causal) or what the rest of the sequence contributes
// (non-causal).  features != 0: q and k are non-negative features already.
// aggregates (nullable): the pass's per-segment (bf16) or per-chunk (fp32) aggregates as
// linattn_forward_state_keep left them; the aggregate launch is then skipped, the causal scan
// rewrites them in place, and ws needs only the per-head totals (non-causal).
cudaError_t run_forward(const ForwardPlan &p, const void *q, const void *k, const void *v,
                        void *out, int64_t heads, int64_t n, int dk, int d, int causal, int is_bf16,
                        const float *init_S, const float *init_z, int features, void *ws,
                        int *err, cudaStream_t st, float *aggregates = nullptr);
// The no-allocation entry point's status word (noalloc.cu): reads it for the current device
// into *word and clears it.  *word = 0 when that entry point has not run on this device.
cudaError_t noalloc_take_status(int *word);

// Failure-path self-test: one thread waits, with the kernels' bounded wait, on a barrier that
// nothing completes; the give-up is recorded in *err.
cudaError_t launch_wait_timeout_selftest(int *err, cudaStream_t st);

// Streaming multiprocessors of the current device (looked up once per device).
int sm_count();

// Launch accounting for linattn_launch_count(): every launcher adds the kernels it enqueued.
void count_launches(uint64_t n);
uint64_t launches_total();
// Records the next caller-supplied profiling event (linattn_profile_events) on `st`.
void record_launch_event(cudaStream_t st);

// Tokens per chunk of the fp32 (CUDA-core) path.
constexpr int kSimtChunk = 64;

// ---- CUDA-core path (simt_forward.cu); is_bf16 selects bf16 I/O, else fp32 ------------
// Chunk aggregates into ws[head][chunk][D*D + D] (S row-major, then z).  features != 0:
// k holds non-negative features already (no phi applied), likewise q below.
cudaError_t launch_simt_chunk_state(const void *k, const void *v, float *ws, int64_t heads,
                                    int64_t n, int d, int is_bf16, int features,
                                    cudaStream_t st);
// States [heads][nseg][dk*dv + dk] (S [dk][dv] row-major, then z [dk]).  In-place exclusive
// prefix over the segments of each head (mode 0), or the per-head total written to
// S_out + head*S_hs ([dk][dv]) and z_out + head*z_hs ([dk]) (mode 1); both start from the
// state (init_S [heads][dk][dv], init_z [heads][dk]) when init_S is not null.
// Mode 2: in-place exclusive suffix (sum of the later segments; no starting state).
cudaError_t launch_scan_states(float *ws, int64_t heads, int64_t nseg, int dk, int dv, int mode,
                               float *S_out, int64_t S_hs, float *z_out, int64_t z_hs,
                               const float *init_S, const float *init_z, cudaStream_t st);
// Per-head sum of gathered states [count][heads][D*d + D], skipping index `skip`.
cudaError_t launch_sum_states(const float *states, int64_t count, int64_t skip, int64_t heads,
                              int d, float *S_out, float *z_out, cudaStream_t st);
// Outputs from per-chunk prefixes (causal) or the per-head totals (non-causal).
cudaError_t launch_simt_chunk_out(const void *q, const void *k, const void *v, void *out,
                                  const float *S, const float *z, int64_t S_chunk_stride,
                                  int64_t S_head_stride, int64_t z_chunk_stride,
                                  int64_t z_head_stride, int64_t heads, int64_t n, int d,
                                  int causal, int is_bf16, int features, cudaStream_t st);
// FAVOR+ positive random features: out[t][i] = exp(W[i] . x[t] - |x[t]|^2 / 2) / sqrt(m) for
// rows t < rows, i < m; W [m][d] float32; x [rows][d], out [rows][m] of type bf16 (tensor
// cores) or fp32 (CUDA cores).  d, m in {64, 128}.
cudaError_t launch_favor_features(const void *x, const float *W, void *out, int64_t rows, int d,
                                  int m, int is_bf16, int *err, cudaStream_t st);

// ---- backward pass with fp32 I/O (backward.cu), CUDA cores; is_bf16 selects bf16 I/O ------
// Workspace floats linattn_backward needs.
size_t backward_workspace_floats(int64_t heads, int64_t n, int d, int causal);
cudaError_t backward(const void *q, const void *k, const void *v, const void *g, void *dq,
                     void *dk, void *dv, int64_t heads, int64_t n, int d, int causal, int is_bf16,
                     float *ws, cudaStream_t st);

// ---- decode (decode.cu) ----------------------------------------------------------------
cudaError_t launch_decode_step(float *S, float *z, const void *q, const void *k, const void *v,
                               void *out, int64_t heads, int d, cudaStream_t st);

// ---- bf16 I/O, tensor cores (tc_forward.cu, tc_causal.cu) ---------------------------------
// Chunk length of the tensor-core aggregate and non-causal kernels.
constexpr int kTcChunk = 64;
// Chunk length of the causal kernel on features of their own dimension (tc_causal.cu);
// segments are multiples of it.
constexpr int kTcFeatureChunk = 128;
// Causal outputs on features whose dimension dk differs from the value dimension dv, from the
// exclusive prefix state of every segment (prefix: [heads][segments][dk*dv + dk] fp32, S
// row-major then z).  q, k: [heads][n][dk] features; v, out: [heads][n][dv].  seg: a multiple
// of kTcFeatureChunk.
cudaError_t tc_causal_features(const void *q, const void *k, const void *v, void *out,
                               int64_t heads, int64_t n, int dk, int dv, int64_t seg,
                               const float *prefix, int *err, cudaStream_t st);
// Default tokens per work item (segment) of the tensor-core path (a multiple of 256, or the
// whole head rounded up to kTcFeatureChunk).
int64_t tc_default_segment(int64_t heads, int64_t n, int d);
// Workspace bytes the tensor-core forward needs.
size_t tc_workspace_bytes(int64_t heads, int64_t n, int dk, int dv, int64_t seg, int causal);
// q, k: [heads][n][dk]; v, out: [heads][n][dv].  init_S / init_z (nullable): the state before
// the first token of every head.  features != 0: q and k are non-negative features already
// (no phi applied; dk may differ from dv), else dk = dv.
cudaError_t tc_forward(const void *q, const void *k, const void *v, void *out, int64_t heads,
                       int64_t n, int dk, int dv, int causal, int64_t seg, void *ws, int *err,
                       const float *init_S, const float *init_z, int features,
                       cudaStream_t st, float *aggregates = nullptr);
cudaError_t tc_forward_state(const void *k, const void *v, float *S_out, float *z_out,
                             int64_t heads, int64_t n, int d, int64_t seg, void *ws, int *err,
                             cudaStream_t st);
// Segment aggregates [S | z] = sum phi(k)^T [v | 1] of k, v: [heads][n][d] bf16 into
// out: [heads][ceil(n / seg)][d*d + d] fp32 (one launch; seg a multiple of kTcChunk).
cudaError_t tc_segment_aggregates(const void *k, const void *v, int64_t heads, int64_t n, int d,
                                  int64_t seg, float *out, int *err, cudaStream_t st);

// ---- bf16 I/O backward on the tensor cores (tc_backward.cu) --------------------------------
struct TcBackwardLayout {
  // [heads][segments][d*d + 3d + 4]: the forward records [Psi | zeta | vs | sigma | kappa] and
  // the reverse records [Phi | rho | as | tau | bs] of the segments (tc_backward.cu)
  float *s_rec, *r_rec;
  float *s_tot, *r_tot;           // [heads][d*d + 3d + 4]: per-head totals (non-causal)
  __nv_bfloat16 *a_hi, *a_lo;     // [heads][n][d]: a_i = g_i / den_i as a bf16 pair
  float *b;                       // [heads][n]: -(a_i . out_i)
  // [heads][chunks][3d + 4]: per chunk, the vectors of the forward record before it within
  // its segment, and the chunk's own reverse-record vectors
  float *s_vec, *r_vec;
  __nv_bfloat16 *psi_q, *psi_k;  // [heads][n][d]: psi = phi - 1 of q and k, rounded to bf16
  float *sq, *sk;                // [heads][n]: their row sums
};
// Tokens per work item of the backward (a multiple of 256, or n rounded up to kTcChunk).
int64_t tc_backward_segment(int64_t heads, int64_t n, int d);
// The workspace's parts at ws (null: sizes only); *bytes = the workspace size.
TcBackwardLayout tc_backward_layout(void *ws, int64_t heads, int64_t n, int d, int64_t seg,
                                    size_t *bytes);
// q, k, v, g, dq, dk, dv: [heads][n][d] bf16, d in {64, 128}.
cudaError_t tc_backward(const void *q, const void *k, const void *v, const void *g, void *dq,
                        void *dk, void *dv, int64_t heads, int64_t n, int d, int causal,
                        int64_t seg, void *ws, int *err, cudaStream_t st);

}  // namespace linattn
