// Pieces shared by the tensor-core kernels (tc_forward.cu, tc_causal.cu, tc_backward.cu):
// shared-memory matrix descriptors, the packed-bf16 feature map, 32-byte global stores, the
// all-lane read of M = 64 accumulators, warp-uniform waits, the (head, segment) work items, and
// the TMA tensor maps of [heads][n][d] bf16.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace linattn {
namespace tc {

constexpr int kMaxSmem = 227 * 1024;  // dynamic shared memory of one CTA
constexpr uint32_t kTmemCols = 512;   // every column of the SM's tensor memory

// Shared-memory descriptors are built once per operand base (make_sw128_desc) and then
// stepped by adding (byte offset >> 4) to the 14-bit start-address field, which never
// carries: shared addresses stay below 2^18 bytes.
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t byte_off) {
  return desc + static_cast<uint64_t>(byte_off >> 4);
}
// K-major operand, K-step ks of a tile made of 64-column atoms of `atom_bytes` each: four
// K-steps of 32 bytes inside one 128-byte swizzle row, then the next atom.
__device__ __forceinline__ uint32_t kmajor_off(int ks, uint32_t atom_bytes) {
  return (ks >> 2) * atom_bytes + (ks & 3) * 32;
}
// MN-major operand, K-step ks: 16 K-rows = two 8-row groups of 1024 bytes.
__device__ __forceinline__ uint32_t mnmajor_off(int ks) { return ks * 2048; }
__device__ __forceinline__ uint64_t kmajor_base(uint32_t addr) {
  return make_sw128_desc(addr, 16, 1024);
}
// lbo: byte stride between the operand's 64-wide M/N blocks (its atoms)
__device__ __forceinline__ uint64_t mnmajor_base(uint32_t addr, uint32_t lbo) {
  return make_sw128_desc(addr, lbo, 1024);
}

// phi on two packed bf16 values: exp(min(x, 0)) + max(x, 0), which is x + 1 above zero and
// exp(x) at or below zero.  Everything is packed bf16 arithmetic:
//   t = min(x, 0) * log2(e), with log2(e) split into a bf16 head and tail so that the product
//       is rounded once (fma of the head onto the tail's product);
//   e = 2^t with the packed bf16 exponential (one MUFU operation for two elements);
//   phi = e + max(x, 0)  (above zero e = 1 exactly, so this is 1 + x rounded once).
// The bf16 rounding of t perturbs exp(x) by at most |x| * 2^-9 relative; over the sums of
// the method this stays far below the bf16 I/O tolerance (modelled and tested).
__device__ __forceinline__ uint32_t phi_bf16x2(uint32_t u) {
  const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(&u);
  const __nv_bfloat162 zero = __float2bfloat162_rn(0.f);
  const __nv_bfloat162 log2e_hi = __float2bfloat162_rn(1.4453125f);      // bf16(log2 e)
  const __nv_bfloat162 log2e_lo = __float2bfloat162_rn(-0.0026174592f);  // log2 e - head
  const __nv_bfloat162 m = __hmin2(x, zero);
  const __nv_bfloat162 p = __hmax2(x, zero);
  const __nv_bfloat162 t = __hfma2(m, log2e_hi, __hmul2(m, log2e_lo));
  uint32_t e;
  asm("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(e) : "r"(*reinterpret_cast<const uint32_t *>(&t)));
  const __nv_bfloat162 r = __hadd2(*reinterpret_cast<const __nv_bfloat162 *>(&e), p);
  return *reinterpret_cast<const uint32_t *>(&r);
}
__device__ __forceinline__ uint4 phi_bf16x8(uint4 x) {
  x.x = phi_bf16x2(x.x);
  x.y = phi_bf16x2(x.y);
  x.z = phi_bf16x2(x.z);
  x.w = phi_bf16x2(x.w);
  return x;
}

__device__ __forceinline__ uint4 pack8(const float *f) {
  uint4 u;
  u.x = pack_bf16x2(f[0], f[1]);
  u.y = pack_bf16x2(f[2], f[3]);
  u.z = pack_bf16x2(f[4], f[5]);
  u.w = pack_bf16x2(f[6], f[7]);
  return u;
}
// 32 bytes (16 bf16 values) to global memory: one full-sector store where the buffer is
// 32-byte aligned (a32), else two 16-byte stores.  Callers promise only 16-byte aligned
// buffers; a row's alignment is its buffer's (rows are 128 or 256 bytes long), so kernels
// test their output pointer once and pass the result, uniform over the launch.
__device__ __forceinline__ bool aligned32(const void *p) {
  return (reinterpret_cast<uintptr_t>(p) & 31u) == 0;
}
__device__ __forceinline__ void st_global_32B(void *p, uint4 a, uint4 b, bool a32) {
  if (a32) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x),
                 "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
  } else {
    uint4 *q = static_cast<uint4 *>(p);
    q[0] = a;
    q[1] = b;
  }
}

// 16 lanes x 32 consecutive fp32 columns of an M = 64 accumulator (it lives in lanes 0..15 of
// each TMEM sub-partition; taddr: the calling warp's lane base and the first column), read by
// all 32 threads (warp-collective), where the 32x32b loads would leave half the warp idle:
// thread t gets rows t/4 and 8 + t/4 of the 16, columns 8k + 2(t%4) + {0, 1} for k = 0..3, as
// f[4k + {0, 1}] (first row) and f[4k + {2, 3}] (second row).
__device__ __forceinline__ void tmem_quad32(uint32_t taddr, float *f) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  tmem_ld_wait();
  tmem_reg_fence<16>(r);
#pragma unroll
  for (int e = 0; e < 16; ++e) f[e] = __uint_as_float(r[e]);
}

// mbarrier wait of a whole warp whose outcome the lanes share (warp-uniform control flow);
// a lane whose bounded wait gave up makes the warp give up.  Two forms, chosen per kernel by
// measurement (the faster one differs with the shape of the work between waits):
//   LANE0 = false  every lane waits on the barrier itself;
//   LANE0 = true   lane 0 waits (suspending while the phase is pending), then every lane
//                  tests the completed phase once, which orders its later reads after the
//                  barrier like its own wait would.
template <bool LANE0>
struct WarpWaiterT {
  volatile int *abort;
  int *err;
  int lane;
  bool ok = true;
  __device__ __forceinline__ bool operator()(uint64_t *b, uint32_t parity) {
    if (LANE0) {
      int r = 1;
      if (lane == 0) r = (ok && mbar_wait(b, parity, abort, err)) ? 1 : 0;
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r) mbar_try_wait(b, parity);
      ok = ok && (r != 0);
    } else {
      const int r = (ok && mbar_wait(b, parity, abort, err)) ? 1 : 0;
      ok = __all_sync(0xffffffffu, r) != 0;
    }
    return ok;
  }
};
using WarpWaiter = WarpWaiterT<false>;

// One work item: tokens [t_begin, t_end) of one head (one segment), in chunks of CH tokens.
struct Item {
  int64_t head, seg, t_begin, t_end;
  int nchunks;
};
template <int CH>
__device__ __forceinline__ Item item_at(int64_t it, int64_t n, int64_t seg_len, int64_t nseg) {
  Item I;
  I.head = it / nseg;
  I.seg = it % nseg;
  I.t_begin = I.seg * seg_len;
  I.t_end = n < I.t_begin + seg_len ? n : I.t_begin + seg_len;
  I.nchunks = static_cast<int>((I.t_end - I.t_begin + CH - 1) / CH);
  return I;
}

}  // namespace tc

// [heads][n][d] bf16 as a 3-D TMA tensor (d innermost), boxes of 64 columns x box_rows rows,
// 128-byte swizzle.  Rows beyond n read as zero and are never written.  (tc_forward.cu)
cudaError_t make_tmap_bf16(CUtensorMap *m, const void *ptr, int64_t heads, int64_t n, int d,
                           int box_rows);

}  // namespace linattn
