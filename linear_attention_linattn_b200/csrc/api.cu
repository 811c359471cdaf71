// C ABI of linattn (see include/linattn.h): argument checks, workspace, dispatch.
//
// Dispatch is by I/O type only: float32 I/O runs the CUDA-core kernels (simt_forward.cu),
// bfloat16 I/O runs the tensor-core kernels (tc_forward.cu).  There is no host fallback:
// every step of the pass runs in this library's kernels on the caller's stream.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "linattn.h"

namespace linattn {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  std::once_flag once;
  std::atomic<bool> ready{false};
  cudaError_t init_err = cudaSuccess;
  int *err_word = nullptr;     // kernels' error word (device memory)
  cudaMemPool_t pool = nullptr;  // stream-ordered workspace pool
  // linattn_forward_host: the streams its head groups run on (created on its first call)
  std::once_flag streams_once;
  cudaError_t streams_err = cudaSuccess;
  cudaStream_t group_streams[3] = {nullptr, nullptr, nullptr};
};
DeviceState g_dev[kMaxDevices];

// Per-device set-up on first use: the kernels' error word and a workspace pool that keeps
// its memory between calls (so steady-state calls do not go back to the driver).
cudaError_t device_state(DeviceState **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceState &s = g_dev[dev];
  std::call_once(s.once, [&]() {
    cudaError_t r = cudaMalloc(&s.err_word, sizeof(int));
    if (r == cudaSuccess) r = cudaMemset(s.err_word, 0, sizeof(int));
    if (r == cudaSuccess) {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.handleTypes = cudaMemHandleTypeNone;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      r = cudaMemPoolCreate(&s.pool, &props);
    }
    if (r == cudaSuccess) {
      uint64_t keep = ~0ull;
      r = cudaMemPoolSetAttribute(s.pool, cudaMemPoolAttrReleaseThreshold, &keep);
    }
    if (r == cudaSuccess) r = cudaDeviceSynchronize();
    s.init_err = r;
    s.ready.store(r == cudaSuccess, std::memory_order_release);
  });
  if (s.init_err != cudaSuccess) return s.init_err;
  *out = &s;
  return cudaSuccess;
}

// The current device's state if device_state() has set it up already, else null (no set-up,
// so nothing is allocated).
DeviceState *device_state_if_ready() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  return g_dev[dev].ready.load(std::memory_order_acquire) ? &g_dev[dev] : nullptr;
}

// Stream-ordered scratch: allocated on `st` before the kernels, released on `st` after.
struct Workspace {
  void *ptr = nullptr;
  cudaStream_t st = nullptr;
  ~Workspace() {
    if (ptr) cudaFreeAsync(ptr, st);
  }
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

linattn_status to_status(cudaError_t e) { return e == cudaSuccess ? LINATTN_OK : LINATTN_ERR_CUDA; }

// Forward pass with its workspace taken from the device's pool on `st`.
linattn_status forward_pooled(const void *q, const void *k, const void *v, void *out,
                              int64_t heads, int64_t n, int dk, int d, int causal, int is_bf16,
                              int64_t seg_len, const float *init_S, const float *init_z,
                              int features, DeviceState *ds, cudaStream_t st) {
  const ForwardPlan p = plan_forward(heads, n, dk, d, causal, is_bf16, seg_len);
  Workspace ws;
  ws.st = st;
  if (cudaMallocFromPoolAsync(&ws.ptr, p.ws_bytes, ds->pool, st) != cudaSuccess)
    return LINATTN_ERR_CUDA;
  return to_status(run_forward(p, q, k, v, out, heads, n, dk, d, causal, is_bf16, init_S, init_z,
                               features, ws.ptr, ds->err_word, st));
}

// Failure-path self-test: one thread waits, with the kernels' own bounded wait, on an mbarrier
// that nothing ever arrives at.  The wait gives up after its limit and records
// LINATTN_ERR_TIMEOUT in the device's error word, exactly as a stalled kernel would.
__global__ void wait_timeout_selftest_kernel(int *err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err);
}

}  // namespace

// The forward's shape, mode and type checks (the pointers are checked by the callers).
linattn_status check_forward_shape(int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                                   linattn_dtype dtype) {
  if (causal != 0 && causal != 1) return LINATTN_ERR_INVALID_ARG;
  if (dtype != LINATTN_F32 && dtype != LINATTN_BF16) return LINATTN_ERR_INVALID_ARG;
  // n < 2^31, B*H < 2^24, total elements < 2^40
  if (B <= 0 || H <= 0 || n <= 0 || d <= 0) return LINATTN_ERR_INVALID_ARG;
  if (B > (1 << 24) || H > (1 << 24) || n >= (int64_t(1) << 31)) return LINATTN_ERR_INVALID_ARG;
  const int64_t heads = B * H;
  if (heads > (1 << 24)) return LINATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LINATTN_ERR_UNSUPPORTED;
  if (heads * n > (int64_t(1) << 40) / d) return LINATTN_ERR_INVALID_ARG;
  const int64_t nchunks = (n + kSimtChunk - 1) / kSimtChunk;
  if (nchunks * heads >= (int64_t(1) << 31)) return LINATTN_ERR_INVALID_ARG;
  return LINATTN_OK;
}

linattn_status check_forward_args(const void *q, const void *k, const void *v, const void *out,
                                  int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                                  linattn_dtype dtype) {
  if (!q || !k || !v || !out) return LINATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return LINATTN_ERR_INVALID_ARG;
  return check_forward_shape(B, H, n, d, causal, dtype);
}

ForwardPlan plan_forward(int64_t heads, int64_t n, int dk, int d, int causal, int is_bf16,
                         int64_t seg_len) {
  ForwardPlan p;
  if (is_bf16) {
    p.seg = seg_len > 0 ? seg_len
                        : tc_default_segment(heads, n, d);
    p.ws_bytes = tc_workspace_bytes(heads, n, dk, d, p.seg, causal);
    return p;
  }
  // fp32 path: one state per 64-token chunk; non-causal adds one total per head
  const int64_t nchunks = (n + kSimtChunk - 1) / kSimtChunk;
  const int64_t per = (int64_t)d * d + d;
  p.ws_bytes = (size_t)(heads * nchunks * per + (causal ? 0 : heads * per)) * sizeof(float);
  return p;
}

cudaError_t run_forward(const ForwardPlan &p, const void *q, const void *k, const void *v,
                        void *out, int64_t heads, int64_t n, int dk, int d, int causal, int is_bf16,
                        const float *init_S, const float *init_z, int features, void *ws,
                        int *err, cudaStream_t st, float *aggregates) {
  if (is_bf16)
    return tc_forward(q, k, v, out, heads, n, dk, d, causal, p.seg, ws, err, init_S, init_z,
                      features, st, aggregates);
  if (dk != d) return cudaErrorInvalidValue;  // the CUDA-core kernels keep one dimension
  const int64_t nchunks = (n + kSimtChunk - 1) / kSimtChunk;
  const int64_t per = (int64_t)d * d + d;
  float *w = aggregates ? aggregates : static_cast<float *>(ws);
  cudaError_t e = cudaSuccess;
  if (!aggregates) e = launch_simt_chunk_state(k, v, w, heads, n, d, 0, features, st);
  if (e != cudaSuccess) return e;
  if (causal) {
    e = launch_scan_states(w, heads, nchunks, d, d, 0, nullptr, 0, nullptr, 0, init_S, init_z, st);
    if (e != cudaSuccess) return e;
    return launch_simt_chunk_out(q, k, v, out, w, w + (int64_t)d * d, per, nchunks * per, per,
                                 nchunks * per, heads, n, d, 1, 0, features, st);
  }
  float *tot = aggregates ? static_cast<float *>(ws) : w + heads * nchunks * per;
  float *tot_z = tot + heads * (int64_t)d * d;
  e = launch_scan_states(w, heads, nchunks, d, d, 1, tot, (int64_t)d * d, tot_z, d, init_S, init_z,
                         st);
  if (e != cudaSuccess) return e;
  return launch_simt_chunk_out(q, k, v, out, tot, tot_z, 0, (int64_t)d * d, 0, d, heads, n, d, 0,
                               0, features, st);
}

cudaError_t launch_wait_timeout_selftest(int *err, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(err);
  count_launches(1);
  return cudaGetLastError();
}

int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return 148;  // not cached: asked again next time
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

}  // namespace linattn

using namespace linattn;

extern "C" {

linattn_status linattn_selftest_wait_timeout(linattn_stream_t stream) {
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  return to_status(launch_wait_timeout_selftest(ds->err_word,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

linattn_status linattn_forward_ex(const void *q, const void *k, const void *v, void *out,
                                  int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                                  linattn_dtype dtype, int64_t segment_len,
                                  linattn_stream_t stream) {
  linattn_status s = check_forward_args(q, k, v, out, B, H, n, d, causal, dtype);
  if (s != LINATTN_OK) return s;
  if (segment_len < 0 || segment_len % kTcFeatureChunk != 0) return LINATTN_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  return forward_pooled(q, k, v, out, B * H, n, (int)d, (int)d, causal, dtype == LINATTN_BF16,
                        segment_len, nullptr, nullptr, 0, ds,
                        reinterpret_cast<cudaStream_t>(stream));
}

linattn_status linattn_forward_host(const void *q, const void *k, const void *v, void *out,
                                    int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                                    linattn_dtype dtype, linattn_stream_t stream) {
  if (!q || !k || !v || !out) return LINATTN_ERR_INVALID_ARG;  // host buffers: any alignment
  linattn_status s = check_forward_shape(B, H, n, d, causal, dtype);
  if (s != LINATTN_OK) return s;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  std::call_once(ds->streams_once, [&]() {
    for (cudaStream_t &gs : ds->group_streams) {
      ds->streams_err = cudaStreamCreateWithFlags(&gs, cudaStreamNonBlocking);
      if (ds->streams_err != cudaSuccess) break;
    }
  });
  if (ds->streams_err != cudaSuccess) return LINATTN_ERR_CUDA;
  const cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
  constexpr int kSlots = 3;  // head groups in flight, one per stream
  const int64_t heads = B * H;
  const size_t head_bytes = static_cast<size_t>(n) * d * (dtype == LINATTN_BF16 ? 2 : 4);
  // about eight groups, so that all but one group's copies overlap others' work, each at most
  // 1 GiB of the four tensors
  int64_t g = (heads + 7) / 8;
  const int64_t g_cap = static_cast<int64_t>((size_t(1) << 30) / (4 * head_bytes));
  if (g > g_cap) g = g_cap > 0 ? g_cap : 1;
  const int64_t ngroups = (heads + g - 1) / g;
  const size_t group_bytes = static_cast<size_t>(g) * head_bytes;
  const auto *hq = static_cast<const unsigned char *>(q);
  const auto *hk = static_cast<const unsigned char *>(k);
  const auto *hv = static_cast<const unsigned char *>(v);
  auto *ho = static_cast<unsigned char *>(out);

  // the group streams start after the work enqueued on the caller's stream so far
  cudaEvent_t start = nullptr, done[kSlots] = {nullptr, nullptr, nullptr};
  cudaError_t e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(start, user);
  for (int i = 0; i < kSlots && e == cudaSuccess; ++i)
    e = cudaStreamWaitEvent(ds->group_streams[i], start, 0);
  // per stream: device buffers for one group's q, k, v, out
  unsigned char *buf[kSlots] = {nullptr, nullptr, nullptr};
  const int used = static_cast<int>(ngroups < kSlots ? ngroups : kSlots);
  for (int i = 0; i < used && e == cudaSuccess; ++i)
    e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&buf[i]), 4 * group_bytes, ds->pool,
                                ds->group_streams[i]);
  // group j on stream j % kSlots: copy in, forward, copy out (the stream orders the reuse of
  // its buffers; the copies of one group overlap the work of the others)
  linattn_status st = e == cudaSuccess ? LINATTN_OK : LINATTN_ERR_CUDA;
  for (int64_t j = 0; j < ngroups && st == LINATTN_OK; ++j) {
    const int i = static_cast<int>(j % kSlots);
    const cudaStream_t gs = ds->group_streams[i];
    const int64_t h0 = j * g, gh = heads - h0 < g ? heads - h0 : g;
    const size_t off = static_cast<size_t>(h0) * head_bytes, bytes = gh * head_bytes;
    unsigned char *dq = buf[i], *dk = dq + group_bytes, *dv = dk + group_bytes,
                  *dout = dv + group_bytes;
    if (cudaMemcpyAsync(dq, hq + off, bytes, cudaMemcpyHostToDevice, gs) != cudaSuccess ||
        cudaMemcpyAsync(dk, hk + off, bytes, cudaMemcpyHostToDevice, gs) != cudaSuccess ||
        cudaMemcpyAsync(dv, hv + off, bytes, cudaMemcpyHostToDevice, gs) != cudaSuccess) {
      st = LINATTN_ERR_CUDA;
      break;
    }
    st = forward_pooled(dq, dk, dv, dout, gh, n, (int)d, (int)d, causal, dtype == LINATTN_BF16,
                        0, nullptr, nullptr, 0, ds, gs);
    if (st == LINATTN_OK &&
        cudaMemcpyAsync(ho + off, dout, bytes, cudaMemcpyDeviceToHost, gs) != cudaSuccess)
      st = LINATTN_ERR_CUDA;
  }
  // release the buffers in stream order; the caller's stream waits for every group
  for (int i = 0; i < kSlots; ++i) {
    if (buf[i] && cudaFreeAsync(buf[i], ds->group_streams[i]) != cudaSuccess)
      st = LINATTN_ERR_CUDA;
    if (cudaEventCreateWithFlags(&done[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventRecord(done[i], ds->group_streams[i]) != cudaSuccess ||
        cudaStreamWaitEvent(user, done[i], 0) != cudaSuccess)
      st = LINATTN_ERR_CUDA;
  }
  for (cudaEvent_t ev : done)
    if (ev) cudaEventDestroy(ev);
  if (start) cudaEventDestroy(start);
  return st;
}

linattn_status linattn_forward_init(const void *q, const void *k, const void *v, void *out,
                                    const float *state_S, const float *state_z, int64_t B,
                                    int64_t H, int64_t n, int64_t d, int causal,
                                    linattn_dtype dtype, linattn_stream_t stream) {
  linattn_status s = check_forward_args(q, k, v, out, B, H, n, d, causal, dtype);
  if (s != LINATTN_OK) return s;
  if (!state_S || !state_z || !aligned16(state_S) || !aligned16(state_z))
    return LINATTN_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  return forward_pooled(q, k, v, out, B * H, n, (int)d, (int)d, causal, dtype == LINATTN_BF16,
                        0, state_S, state_z, 0, ds, reinterpret_cast<cudaStream_t>(stream));
}

linattn_status linattn_forward_features(const void *phi_q, const void *phi_k, const void *v,
                                        void *out, int64_t B, int64_t H, int64_t n, int64_t m,
                                        int64_t d, int causal, linattn_dtype dtype,
                                        linattn_stream_t stream) {
  linattn_status s = check_forward_args(phi_q, phi_k, v, out, B, H, n, d, causal, dtype);
  if (s != LINATTN_OK) return s;
  if (m <= 0) return LINATTN_ERR_INVALID_ARG;
  if (m != 64 && m != 128) return LINATTN_ERR_UNSUPPORTED;
  if (m != d && dtype != LINATTN_BF16) return LINATTN_ERR_UNSUPPORTED;  // fp32: m = d only
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  return forward_pooled(phi_q, phi_k, v, out, B * H, n, (int)m, (int)d, causal,
                        dtype == LINATTN_BF16, 0, nullptr, nullptr, 1, ds,
                        reinterpret_cast<cudaStream_t>(stream));
}

linattn_status linattn_favor_features(const void *x, const float *W, void *out, int64_t rows,
                                      int64_t d, int64_t m, linattn_dtype dtype,
                                      linattn_stream_t stream) {
  if (!x || !W || !out) return LINATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W) || !aligned16(out)) return LINATTN_ERR_INVALID_ARG;
  if (dtype != LINATTN_F32 && dtype != LINATTN_BF16) return LINATTN_ERR_INVALID_ARG;
  if (rows <= 0 || d <= 0 || m <= 0) return LINATTN_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || (m != 64 && m != 128)) return LINATTN_ERR_UNSUPPORTED;
  if (rows >= (int64_t(1) << 31) || rows > (int64_t(1) << 40) / m) return LINATTN_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  return to_status(launch_favor_features(x, W, out, rows, (int)d, (int)m, dtype == LINATTN_BF16,
                                         ds->err_word, reinterpret_cast<cudaStream_t>(stream)));
}

linattn_status linattn_backward(const void *q, const void *k, const void *v, const void *dout,
                                void *dq, void *dk, void *dv, int64_t B, int64_t H, int64_t n,
                                int64_t d, int causal, linattn_dtype dtype,
                                linattn_stream_t stream) {
  return linattn_backward_ex(q, k, v, dout, dq, dk, dv, B, H, n, d, causal, dtype, 0, stream);
}

linattn_status linattn_backward_ex(const void *q, const void *k, const void *v,
                                   const void *dout, void *dq, void *dk, void *dv, int64_t B,
                                   int64_t H, int64_t n, int64_t d, int causal,
                                   linattn_dtype dtype, int64_t segment_len,
                                   linattn_stream_t stream) {
  linattn_status s = check_forward_args(q, k, v, dout, B, H, n, d, causal, dtype);
  if (s != LINATTN_OK) return s;
  if (segment_len < 0 || segment_len % kTcChunk != 0) return LINATTN_ERR_INVALID_ARG;
  if (!dq || !dk || !dv || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return LINATTN_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t heads = B * H;
  Workspace ws;
  ws.st = st;
  if (dtype == LINATTN_BF16) {  // tensor cores
    const int64_t seg = segment_len > 0 ? segment_len : tc_backward_segment(heads, n, (int)d);
    size_t bytes = 0;
    tc_backward_layout(nullptr, heads, n, (int)d, seg, &bytes);
    if (cudaMallocFromPoolAsync(&ws.ptr, bytes, ds->pool, st) != cudaSuccess)
      return LINATTN_ERR_CUDA;
    return to_status(tc_backward(q, k, v, dout, dq, dk, dv, heads, n, (int)d, causal, seg,
                                 ws.ptr, ds->err_word, st));
  }
  const size_t bytes = backward_workspace_floats(heads, n, (int)d, causal) * sizeof(float);
  if (cudaMallocFromPoolAsync(&ws.ptr, bytes, ds->pool, st) != cudaSuccess)
    return LINATTN_ERR_CUDA;
  return to_status(backward(q, k, v, dout, dq, dk, dv, heads, n, (int)d, causal, 0,
                            static_cast<float *>(ws.ptr), st));
}

linattn_status linattn_sum_states(const float *states, int64_t count, int64_t skip, int64_t B,
                                  int64_t H, int64_t d, float *state_S, float *state_z,
                                  linattn_stream_t stream) {
  if (!state_S || !state_z || (count > 0 && !states)) return LINATTN_ERR_INVALID_ARG;
  if ((states && !aligned16(states)) || !aligned16(state_S) || !aligned16(state_z))
    return LINATTN_ERR_INVALID_ARG;
  if (count < 0 || count > (1 << 20) || skip < -1 || B <= 0 || H <= 0 || B > (1 << 24) ||
      H > (1 << 24) || B * H > (1 << 24))
    return LINATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LINATTN_ERR_UNSUPPORTED;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  return to_status(launch_sum_states(states, count, skip, B * H, (int)d, state_S, state_z,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

linattn_status linattn_forward(const void *q, const void *k, const void *v, void *out, int64_t B,
                               int64_t H, int64_t n, int64_t d, int causal, linattn_dtype dtype,
                               linattn_stream_t stream) {
  return linattn_forward_ex(q, k, v, out, B, H, n, d, causal, dtype, 0, stream);
}

// The block state of k, v into state_S / state_z, its aggregates left in agg (bf16: per
// segment, fp32: per 64-token chunk; [heads][..][d*d + d] fp32).
static cudaError_t forward_state_into(const void *k, const void *v, float *state_S,
                                      float *state_z, int64_t heads, int64_t n, int64_t d,
                                      int is_bf16, float *agg, int *err, cudaStream_t st) {
  if (is_bf16) {
    const int64_t seg = tc_default_segment(heads, n, (int)d);
    return tc_forward_state(k, v, state_S, state_z, heads, n, (int)d, seg, agg, err, st);
  }
  const int64_t nchunks = (n + kSimtChunk - 1) / kSimtChunk;
  cudaError_t e = launch_simt_chunk_state(k, v, agg, heads, n, (int)d, 0, 0, st);
  if (e == cudaSuccess)
    e = launch_scan_states(agg, heads, nchunks, (int)d, (int)d, 1, state_S, d * d, state_z, d,
                           nullptr, nullptr, st);
  return e;
}

static size_t block_aggregate_bytes(int64_t heads, int64_t n, int64_t d, int is_bf16) {
  const int64_t per = d * d + d;
  const int64_t units = is_bf16 ? (n + tc_default_segment(heads, n, (int)d) - 1) /
                                      tc_default_segment(heads, n, (int)d)
                                : (n + kSimtChunk - 1) / kSimtChunk;
  return (size_t)(heads * units * per) * sizeof(float);
}

linattn_status linattn_forward_state(const void *k, const void *v, float *state_S,
                                     float *state_z, int64_t B, int64_t H, int64_t n, int64_t d,
                                     linattn_dtype dtype, linattn_stream_t stream) {
  linattn_status s = check_forward_args(k, k, v, state_S, B, H, n, d, 0, dtype);
  if (s != LINATTN_OK) return s;
  if (!state_z || !aligned16(state_z)) return LINATTN_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t heads = B * H;
  const int is_bf16 = dtype == LINATTN_BF16;
  Workspace ws;
  ws.st = st;
  if (cudaMallocFromPoolAsync(&ws.ptr, block_aggregate_bytes(heads, n, d, is_bf16), ds->pool,
                              st) != cudaSuccess)
    return LINATTN_ERR_CUDA;
  return to_status(forward_state_into(k, v, state_S, state_z, heads, n, d, is_bf16,
                                      static_cast<float *>(ws.ptr), ds->err_word, st));
}

size_t linattn_block_aggregates_bytes(int64_t B, int64_t H, int64_t n, int64_t d,
                                      linattn_dtype dtype) {
  if (B <= 0 || H <= 0 || n <= 0 || B > (1 << 24) || H > (1 << 24) || B * H > (1 << 24) ||
      n >= (int64_t(1) << 31) || (d != 64 && d != 128) ||
      (dtype != LINATTN_F32 && dtype != LINATTN_BF16))
    return 0;
  return block_aggregate_bytes(B * H, n, d, dtype == LINATTN_BF16);
}

linattn_status linattn_forward_state_keep(const void *k, const void *v, float *state_S,
                                          float *state_z, float *aggregates, int64_t B,
                                          int64_t H, int64_t n, int64_t d, linattn_dtype dtype,
                                          linattn_stream_t stream) {
  linattn_status s = check_forward_args(k, k, v, state_S, B, H, n, d, 0, dtype);
  if (s != LINATTN_OK) return s;
  if (!state_z || !aligned16(state_z) || !aggregates || !aligned16(aggregates))
    return LINATTN_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  return to_status(forward_state_into(k, v, state_S, state_z, B * H, n, d,
                                      dtype == LINATTN_BF16, aggregates, ds->err_word,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

linattn_status linattn_forward_init_from(const void *q, const void *k, const void *v,
                                         void *out, const float *state_S, const float *state_z,
                                         float *aggregates, int64_t B, int64_t H, int64_t n,
                                         int64_t d, int causal, linattn_dtype dtype,
                                         linattn_stream_t stream) {
  linattn_status s = check_forward_args(q, k, v, out, B, H, n, d, causal, dtype);
  if (s != LINATTN_OK) return s;
  if (!state_S || !state_z || !aligned16(state_S) || !aligned16(state_z) || !aggregates ||
      !aligned16(aggregates))
    return LINATTN_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  if (device_state(&ds) != cudaSuccess) return LINATTN_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t heads = B * H;
  const int is_bf16 = dtype == LINATTN_BF16;
  const ForwardPlan p = plan_forward(heads, n, (int)d, (int)d, causal, is_bf16, 0);
  // the aggregates are given: the workspace holds only the non-causal per-head totals
  Workspace ws;
  ws.st = st;
  if (!causal && cudaMallocFromPoolAsync(&ws.ptr, (size_t)(heads * (d * d + d)) * sizeof(float),
                                         ds->pool, st) != cudaSuccess)
    return LINATTN_ERR_CUDA;
  return to_status(run_forward(p, q, k, v, out, heads, n, (int)d, (int)d, causal, is_bf16,
                               state_S, state_z, 0, ws.ptr, ds->err_word, st, aggregates));
}

linattn_status linattn_decode_step(float *state_S, float *state_z, const void *q, const void *k,
                                   const void *v, void *out, int64_t Bseq, int64_t H, int64_t d,
                                   linattn_stream_t stream) {
  if (!state_S || !state_z || !q || !k || !v || !out) return LINATTN_ERR_INVALID_ARG;
  if (!aligned16(state_S) || !aligned16(state_z) || !aligned16(q) || !aligned16(k) ||
      !aligned16(v) || !aligned16(out))
    return LINATTN_ERR_INVALID_ARG;
  if (Bseq <= 0 || H <= 0 || d <= 0) return LINATTN_ERR_INVALID_ARG;
  if (Bseq > (1 << 24) || H > (1 << 24) || Bseq * H >= (int64_t(1) << 31))
    return LINATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LINATTN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return to_status(launch_decode_step(state_S, state_z, q, k, v, out, Bseq * H, (int)d, st));
}

size_t linattn_state_bytes(int64_t d) {
  if (d <= 0) return 0;
  return (size_t)(d * d * 4 + d * 4);
}

const char *linattn_status_string(linattn_status status) {
  switch (status) {
    case LINATTN_OK: return "ok";
    case LINATTN_ERR_INVALID_ARG: return "invalid argument";
    case LINATTN_ERR_UNSUPPORTED: return "unsupported head dimension (d must be 64 or 128)";
    case LINATTN_ERR_CUDA: return "CUDA error";
    case LINATTN_ERR_TIMEOUT: return "a kernel's bounded wait gave up";
  }
  return "unknown status";
}

linattn_status linattn_device_error(linattn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return LINATTN_ERR_CUDA;
  int word = 0;
  // the pooled entry points' word, if any of them has run on this device
  if (DeviceState *ds = device_state_if_ready()) {
    if (cudaMemcpy(&word, ds->err_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
      return LINATTN_ERR_CUDA;
    if (word != 0 && cudaMemset(ds->err_word, 0, sizeof(int)) != cudaSuccess)
      return LINATTN_ERR_CUDA;
  }
  // linattn_forward_noalloc's word, in its static block
  int noalloc_word = 0;
  if (noalloc_take_status(&noalloc_word) != cudaSuccess) return LINATTN_ERR_CUDA;
  return (word | noalloc_word) == 0 ? LINATTN_OK : LINATTN_ERR_TIMEOUT;
}

int linattn_version(void) { return 100; }

uint64_t linattn_launch_count(void) { return linattn::launches_total(); }

}  // extern "C"

namespace linattn {
namespace {
std::atomic<uint64_t> g_launches{0};
// per-thread event list of linattn_profile_events
thread_local void *const *t_events = nullptr;
thread_local int t_event_count = 0;
thread_local int t_event_next = 0;
}  // namespace
void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
uint64_t launches_total() { return g_launches.load(std::memory_order_relaxed); }
void record_launch_event(cudaStream_t st) {
  if (t_event_count > 0 && t_event_next < t_event_count)
    cudaEventRecord(static_cast<cudaEvent_t>(t_events[t_event_next++]), st);
}
}  // namespace linattn

extern "C" linattn_status linattn_profile_events(void *const *events, int count) {
  if (count < 0 || (count > 0 && !events)) return LINATTN_ERR_INVALID_ARG;
  linattn::t_events = count > 0 ? events : nullptr;
  linattn::t_event_count = count;
  linattn::t_event_next = 0;
  return LINATTN_OK;
}
