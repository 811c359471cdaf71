// linattn_forward_noalloc: the forward pass for callers that must not allocate memory.
//
// Some callers cannot call cudaMalloc or any allocating routine: real-time or embedded hosts
// that reserve every byte of device memory up front, and runtimes that own the device
// allocator and forbid libraries from reaching it.  linattn_forward takes its temporary state
// (one fp32 D x d state plus z per head and segment) from a stream-ordered pool, which is an
// allocation.  This entry point runs the same kernels, through the same dispatch, with that
// workspace placed in a fixed block of device memory declared in this file instead, so it
// allocates nothing.
//
// The block is a file-scope __device__ array of LINATTN_NOALLOC_SCRATCH_BYTES.  Every GPU
// that loads the library holds one copy until the process exits.  All calls on a device
// share it and it keeps the last call's contents; nothing in it needs to start at zero
// (each kernel writes every scratch value before any kernel reads it), except the status
// word, which starts at zero and is cleared whenever it is read.  Calls whose work overlaps
// on the GPU race on the block, so issue them on one stream, or otherwise order them.  The
// first call on each device looks the block's device address up (cudaGetSymbolAddress) with
// that device current; make that first call before any stream capture.  A failed look-up is
// not remembered: the next call tries again.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "linattn.h"

namespace linattn {
namespace {

// First 256 bytes: the kernels' status word (a bounded wait that gives up ORs
// LINATTN_ERR_TIMEOUT's flag into it); the rest: the workspace.
constexpr size_t kStatusBytes = 256;
constexpr size_t kScratchBytes = LINATTN_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes > kStatusBytes, "scratch block size");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
// Device address of each device's block, once looked up (null until then).
std::atomic<unsigned char *> g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of this device's scratch block.  In host code g_noalloc_scratch names a
// host-side stand-in, never the device memory itself, so the address is asked for.  Only a
// successful look-up is kept.
cudaError_t scratch_address(unsigned char **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned char *p = g_scratch[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    p = g_scratch[dev].load(std::memory_order_acquire);
    if (!p) {
      void *addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
      if (e != cudaSuccess || !addr) return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
      p = static_cast<unsigned char *>(addr);
      g_scratch[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

cudaError_t noalloc_take_status(int *word) {
  *word = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned char *p = g_scratch[dev].load(std::memory_order_acquire);
  if (!p) return cudaSuccess;  // the entry point has not run on this device
  e = cudaMemcpy(word, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && *word != 0) e = cudaMemset(p, 0, sizeof(int));
  return e;
}

}  // namespace linattn

using namespace linattn;

extern "C" linattn_status linattn_forward_noalloc(const void *q, const void *k, const void *v,
                                                  void *out, int64_t B, int64_t H, int64_t n,
                                                  int64_t d, int causal, linattn_dtype dtype,
                                                  linattn_stream_t stream) {
  linattn_status s = check_forward_args(q, k, v, out, B, H, n, d, causal, dtype);
  if (s != LINATTN_OK) return s;
  const int64_t heads = B * H;
  const int is_bf16 = dtype == LINATTN_BF16;
  const int di = static_cast<int>(d);

  // Plan the workspace and reject what does not fit in the scratch block.
  const size_t cap = kScratchBytes - kStatusBytes;
  ForwardPlan p = plan_forward(heads, n, di, di, causal, is_bf16, 0);
  if (p.ws_bytes > cap && is_bf16) {
    // the tensor-core path: lengthen the segments until one state per segment (and, non-causal,
    // a total per head) fits
    const int64_t per = (int64_t)(d * d + d) * (int64_t)sizeof(float);  // one (S, z) state
    const int64_t nseg_max = (int64_t)(cap / per) / heads - (causal ? 0 : 1);
    if (nseg_max < 1) return LINATTN_ERR_INVALID_ARG;
    const int64_t seg =
        ((n + nseg_max - 1) / nseg_max + kTcFeatureChunk - 1) / kTcFeatureChunk * kTcFeatureChunk;
    p = plan_forward(heads, n, di, di, causal, is_bf16, seg);
  }
  if (p.ws_bytes > cap) return LINATTN_ERR_INVALID_ARG;

  unsigned char *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return LINATTN_ERR_CUDA;
  int *status_word = reinterpret_cast<int *>(scratch);
  void *ws = scratch + kStatusBytes;
  cudaError_t e = run_forward(p, q, k, v, out, heads, n, di, di, causal, is_bf16, nullptr, nullptr,
                              0, ws, status_word, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LINATTN_OK : LINATTN_ERR_CUDA;
}

extern "C" linattn_status linattn_selftest_noalloc_wait_timeout(linattn_stream_t stream) {
  unsigned char *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return LINATTN_ERR_CUDA;
  cudaError_t e = launch_wait_timeout_selftest(reinterpret_cast<int *>(scratch),
                                               reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LINATTN_OK : LINATTN_ERR_CUDA;
}
