// Host-side declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace linattn {

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
// In-place exclusive prefix over the segments of each head (mode 0), or the per-head total
// written to S_out + head*S_hs ([D][d]) and z_out + head*z_hs ([D]) (mode 1); both start
// from the state (init_S [heads][D][d], init_z [heads][D]) when init_S is not null.
// Mode 2: in-place exclusive suffix (sum of the later segments; no starting state).
cudaError_t launch_scan_states(float *ws, int64_t heads, int64_t nseg, int d, int mode,
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
// FAVOR+ positive random features: out[t][i] = exp(W[i] . x[t] - |x[t]|^2 / 2) / sqrt(d)
// for rows t < rows; W [d][d] float32 (m = d features); x, out of type bf16 or fp32.
cudaError_t launch_favor_features(const void *x, const float *W, void *out, int64_t rows, int d,
                                  int is_bf16, cudaStream_t st);

// ---- backward pass (backward.cu), CUDA cores; is_bf16 selects bf16 I/O, else fp32 ------
// Workspace floats linattn_backward needs.
size_t backward_workspace_floats(int64_t heads, int64_t n, int d, int causal);
cudaError_t backward(const void *q, const void *k, const void *v, const void *g, void *dq,
                     void *dk, void *dv, int64_t heads, int64_t n, int d, int causal, int is_bf16,
                     float *ws, cudaStream_t st);

// ---- decode (decode.cu) ----------------------------------------------------------------
cudaError_t launch_decode_step(float *S, float *z, const void *q, const void *k, const void *v,
                               void *out, int64_t heads, int d, cudaStream_t st);

// ---- bf16 I/O, tensor cores (tc_forward.cu) ----------------------------------------------
// Chunk length of the tensor-core path.
constexpr int kTcChunk = 64;
// Default tokens per work item (segment) of the tensor-core path.
int64_t tc_default_segment(int64_t heads, int64_t n, int d);
// Workspace bytes the tensor-core forward needs.
size_t tc_workspace_bytes(int64_t heads, int64_t n, int d, int64_t seg, int causal);
// init_S / init_z (nullable): the state before the first token of every head.
// features != 0: q and k are non-negative features already (no phi applied).
cudaError_t tc_forward(const void *q, const void *k, const void *v, void *out, int64_t heads,
                       int64_t n, int d, int causal, int64_t seg, void *ws, int *err,
                       const float *init_S, const float *init_z, int features,
                       cudaStream_t st);
cudaError_t tc_forward_state(const void *k, const void *v, float *S_out, float *z_out,
                             int64_t heads, int64_t n, int d, int64_t seg, void *ws, int *err,
                             cudaStream_t st);

}  // namespace linattn
