// Recurrent decode step (page "Efficient Transformers: Linear Attention and Flash
// Attention", section "The recurrent view: attention as an RNN"):
//
//   S' = S + phi(k) v^T,   z' = z + phi(k),   out = phi(q) S' / (phi(q) . z')
//
// for Bseq*H independent (sequence, head) states.  The step is pure streaming: the fp32
// state (D*d*4 + D*4 bytes) is read once and written once, plus four bf16 token vectors.
// Its floor is those bytes over the HBM bandwidth (the "bytes transferred per decode step"
// bound of the page "Let's Stop Calling Everything Linear Attention").
//
// One CTA of 256 threads per state.  Thread (rg, cg) owns the 4 value columns
// [4cg, 4cg + 4) of the rows r = rg + RG*i, so each warp reads and writes whole 512-byte
// (d = 128) or 256-byte (d = 64) rows with 16-byte accesses.  All of a thread's rows are
// loaded before any is used, so every thread keeps D/RG 16-byte loads in flight.
#include "common.cuh"
#include "internal.h"

namespace linattn {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float4 ld_stream(const float4 *p) {
  float4 r;
  asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ void st_stream(float4 *p, float4 v) {
  asm volatile("st.global.L1::no_allocate.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads) decode_step_kernel(
    float *__restrict__ S, float *__restrict__ z, const __nv_bfloat16 *__restrict__ q,
    const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
    __nv_bfloat16 *__restrict__ out) {
  constexpr int CG = D / 4;            // column groups of 4 floats
  constexpr int RG = kThreads / CG;    // row groups
  constexpr int ROWS = D / RG;         // rows per thread
  __shared__ float s_pk[D], s_pq[D], s_v[D];
  __shared__ float s_part[RG][D];
  __shared__ float s_den[kThreads / 32];

  const int64_t head = blockIdx.x;
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;
  float4 *Sh = reinterpret_cast<float4 *>(S + head * D * D);

  // issue the state loads first; the token vectors arrive meanwhile
  float4 s[ROWS];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) s[i] = ld_stream(Sh + (rg + RG * i) * CG + cg);

  if (tid < D) {
    s_pk[tid] = phi_fast(__bfloat162float(k[head * D + tid]));
    s_pq[tid] = phi_fast(__bfloat162float(q[head * D + tid]));
    s_v[tid] = __bfloat162float(v[head * D + tid]);
  }
  __syncthreads();

  const float4 vv = reinterpret_cast<const float4 *>(s_v)[cg];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < ROWS; ++i) {
    const int r = rg + RG * i;
    const float pk = s_pk[r], pq = s_pq[r];
    float4 t = s[i];
    t.x = fmaf(pk, vv.x, t.x);
    t.y = fmaf(pk, vv.y, t.y);
    t.z = fmaf(pk, vv.z, t.z);
    t.w = fmaf(pk, vv.w, t.w);
    st_stream(Sh + r * CG + cg, t);
    acc.x = fmaf(pq, t.x, acc.x);
    acc.y = fmaf(pq, t.y, acc.y);
    acc.z = fmaf(pq, t.z, acc.z);
    acc.w = fmaf(pq, t.w, acc.w);
  }
  reinterpret_cast<float4 *>(s_part[rg])[cg] = acc;

  // normaliser: z' = z + phi(k), den = phi(q) . z'
  float dz = 0.f;
  if (tid < D) {
    const float zn = z[head * D + tid] + s_pk[tid];
    z[head * D + tid] = zn;
    dz = s_pq[tid] * zn;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dz += __shfl_xor_sync(0xffffffffu, dz, o);
  if ((tid & 31) == 0) s_den[tid >> 5] = dz;
  __syncthreads();

  if (tid < D) {
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) den += s_den[w];
    float num = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) num += s_part[g][tid];
    out[head * D + tid] = __float2bfloat16_rn(num / den);
  }
}

}  // namespace

cudaError_t launch_decode_step(float *S, float *z, const void *q, const void *k, const void *v,
                               void *out, int64_t heads, int d, cudaStream_t st) {
  const auto *qb = static_cast<const __nv_bfloat16 *>(q);
  const auto *kb = static_cast<const __nv_bfloat16 *>(k);
  const auto *vb = static_cast<const __nv_bfloat16 *>(v);
  auto *ob = static_cast<__nv_bfloat16 *>(out);
  if (d == 64)
    decode_step_kernel<64><<<(unsigned)heads, kThreads, 0, st>>>(S, z, qb, kb, vb, ob);
  else
    decode_step_kernel<128><<<(unsigned)heads, kThreads, 0, st>>>(S, z, qb, kb, vb, ob);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

}  // namespace linattn
