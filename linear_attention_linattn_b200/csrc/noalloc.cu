// linattn_forward_noalloc: the forward pass for callers that must not allocate memory.
//
// Some callers cannot call cudaMalloc or any allocating routine: code running while a
// stream is being captured into a CUDA graph whose memory is fixed up front, real-time or
// embedded hosts that pre-reserve every byte, and runtimes that own the device allocator
// and forbid libraries from reaching it.  linattn_forward takes its temporary state
// (one fp32 D x d state plus z per head and segment) from a stream-ordered pool, which is
// an allocation.  This entry point runs the same kernels with that workspace placed in a
// fixed block of device memory declared in this file instead, so it allocates nothing.
//
// The block is a file-scope __device__ array of LINATTN_NOALLOC_SCRATCH_BYTES.  Every GPU
// that loads the library holds one copy until the process exits.  All calls on a device
// share it and it keeps the last call's contents; nothing in it needs to start at zero
// (each kernel writes every scratch value before any kernel reads it).  Calls whose work
// overlaps on the GPU race on the block, so issue them on one stream, or otherwise order
// them.  The first call on each device looks the block's device address up
// (cudaGetSymbolAddress) with that device current; make that first call before any stream
// capture.
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
struct ScratchAddress {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  unsigned char *ptr = nullptr;
};
ScratchAddress g_scratch[kMaxDevices];

// Device address of this device's scratch block (looked up once per device).  In host
// code g_noalloc_scratch names a host-side stand-in, never the device memory itself.
cudaError_t scratch_address(unsigned char **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  ScratchAddress &s = g_scratch[dev];
  std::call_once(s.once, [&]() {
    void *p = nullptr;
    s.err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    s.ptr = static_cast<unsigned char *>(p);
  });
  if (s.err != cudaSuccess) return s.err;
  *out = s.ptr;
  return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace linattn

using namespace linattn;

extern "C" linattn_status linattn_forward_noalloc(const void *q, const void *k, const void *v,
                                                  void *out, int64_t B, int64_t H, int64_t n,
                                                  int64_t d, int causal, linattn_dtype dtype,
                                                  linattn_stream_t stream) {
  if (!q || !k || !v || !out) return LINATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return LINATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return LINATTN_ERR_INVALID_ARG;
  if (dtype != LINATTN_F32 && dtype != LINATTN_BF16) return LINATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || n <= 0 || d <= 0) return LINATTN_ERR_INVALID_ARG;
  if (B > (1 << 24) || H > (1 << 24) || n >= (int64_t(1) << 31)) return LINATTN_ERR_INVALID_ARG;
  const int64_t heads = B * H;
  if (heads > (1 << 24)) return LINATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LINATTN_ERR_UNSUPPORTED;
  if (heads * n > (int64_t(1) << 40) / d) return LINATTN_ERR_INVALID_ARG;

  // Plan the workspace and reject what does not fit in the scratch block.
  const int64_t per = d * d + d;  // floats of one (S, z) state
  const int64_t cap_states = (int64_t)((kScratchBytes - kStatusBytes) / (per * sizeof(float)));
  const int64_t totals = causal ? 0 : heads;  // non-causal keeps one total per head as well
  int64_t seg = 0, nseg = 0;
  if (dtype == LINATTN_BF16) {
    // the tensor-core path: lengthen segments until heads * segments fits
    const int64_t nseg_max = cap_states / heads - (causal ? 0 : 1);
    if (nseg_max < 1) return LINATTN_ERR_INVALID_ARG;
    seg = tc_default_segment(heads, n, (int)d);
    nseg = (n + seg - 1) / seg;
    if (nseg > nseg_max) {
      seg = ((n + nseg_max - 1) / nseg_max + kTcChunk - 1) / kTcChunk * kTcChunk;
      nseg = (n + seg - 1) / seg;
    }
    if (heads * nseg + totals > cap_states) return LINATTN_ERR_INVALID_ARG;
  } else {
    // the CUDA-core path keeps one state per 64-token chunk
    nseg = (n + kSimtChunk - 1) / kSimtChunk;
    if (nseg * heads >= (int64_t(1) << 31)) return LINATTN_ERR_INVALID_ARG;
    if (heads * nseg + totals > cap_states) return LINATTN_ERR_INVALID_ARG;
  }

  unsigned char *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return LINATTN_ERR_CUDA;
  int *status_word = reinterpret_cast<int *>(scratch);
  float *ws = reinterpret_cast<float *>(scratch + kStatusBytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int di = static_cast<int>(d);

  cudaError_t e;
  if (dtype == LINATTN_BF16) {
    e = tc_forward(q, k, v, out, heads, n, di, causal, seg, ws, status_word, nullptr, nullptr, 0,
                   st);
  } else {
    e = launch_simt_chunk_state(k, v, ws, heads, n, di, 0, 0, st);
    if (e == cudaSuccess && causal) {
      e = launch_scan_states(ws, heads, nseg, di, 0, nullptr, 0, nullptr, 0, nullptr, nullptr,
                             st);
      if (e == cudaSuccess)
        e = launch_simt_chunk_out(q, k, v, out, ws, ws + d * d, per, nseg * per, per,
                                  nseg * per, heads, n, di, 1, 0, 0, st);
    } else if (e == cudaSuccess) {
      float *tot = ws + heads * nseg * per;
      float *tot_z = tot + heads * d * d;
      e = launch_scan_states(ws, heads, nseg, di, 1, tot, d * d, tot_z, d, nullptr, nullptr,
                             st);
      if (e == cudaSuccess)
        e = launch_simt_chunk_out(q, k, v, out, tot, tot_z, 0, d * d, 0, d, heads, n, di, 0, 0,
                                  0, st);
    }
  }
  return e == cudaSuccess ? LINATTN_OK : LINATTN_ERR_CUDA;
}
