// FAVOR+ positive random features on the CUDA cores.
//
// Performer's FAVOR+ is named on the page "Efficient Transformers: Linear Attention and Flash
// Attention" (section "Linear attention: reordering the matmuls, not shrinking them") as a
// feature map whose dot products approximate the softmax kernel exp(q . k).  Its
// positive-feature form, with m = d random rows w_i of W (the caller draws them):
//
//     phi(x)_i = exp(w_i . x - |x|^2 / 2) / sqrt(m)
//
// The features are positive, so linattn_forward_features runs the linear-attention pass on
// them with no further feature map.  Each CTA holds W (transposed) in shared memory and walks
// tiles of 64 rows; thread (ti, tc) computes rows ti + 16a and features tc + 16b.
#include "common.cuh"
#include "internal.h"

namespace linattn {
namespace {

constexpr int kRows = 64;
constexpr int kThreads = 256;

__device__ __forceinline__ float4 ldx(const float *p) {
  return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ float4 ldx(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}
__device__ __forceinline__ void stx(float *p, float x) { *p = x; }
__device__ __forceinline__ void stx(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

template <int D, typename T>
__global__ void __launch_bounds__(kThreads) favor_features_kernel(const T *__restrict__ x,
                                                                  const float *__restrict__ W,
                                                                  T *__restrict__ out,
                                                                  int64_t rows) {
  constexpr int PD = D + 1;
  extern __shared__ float4 smem_f4[];
  float *sX = reinterpret_cast<float *>(smem_f4);  // x rows            [kRows][PD]
  float *sWT = sX + kRows * PD;                     // W transposed      [D][D]: sWT[r][i]
  float *sHalfSq = sWT + D * D;                     // |x_t|^2 / 2       [kRows]
  // W once per CTA (the CTA then walks many row tiles); read transposed from global memory
  // (64 KB at d = 128, L2-resident) so the shared-memory writes are consecutive
  for (int e = threadIdx.x; e < D * D; e += kThreads) {
    const int r = e / D, i = e % D;
    sWT[e] = W[i * D + r];
  }
  constexpr int RB = D / 16;
  const int ti = threadIdx.x / 16, tc = threadIdx.x % 16;
  const float scale = rsqrtf(static_cast<float>(D));  // 1 / sqrt(m), m = D
  const int64_t ntiles = (rows + kRows - 1) / kRows;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int64_t r0 = tile * kRows;
    const int valid = rows - r0 < kRows ? static_cast<int>(rows - r0) : kRows;
    __syncthreads();  // the previous tile is done with sX
    for (int i = threadIdx.x; i < kRows * D / 4; i += kThreads) {
      const int row = i / (D / 4), c4 = i % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row < valid) v = ldx(x + (r0 + row) * D + 4 * c4);
      float *p = sX + row * PD + 4 * c4;
      p[0] = v.x;
      p[1] = v.y;
      p[2] = v.z;
      p[3] = v.w;
    }
    __syncthreads();
    if (threadIdx.x < kRows) {
      float sq = 0.f;
      for (int r = 0; r < D; ++r) sq = fmaf(sX[threadIdx.x * PD + r], sX[threadIdx.x * PD + r], sq);
      sHalfSq[threadIdx.x] = 0.5f * sq;
    }
    __syncthreads();
    float acc[4][RB];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[a][b] = 0.f;
    for (int r = 0; r < D; ++r) {
      float xa[4], wb[RB];
#pragma unroll
      for (int a = 0; a < 4; ++a) xa[a] = sX[(ti + 16 * a) * PD + r];
#pragma unroll
      for (int b = 0; b < RB; ++b) wb[b] = sWT[r * D + tc + 16 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(xa[a], wb[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int t = ti + 16 * a;
      if (t < valid) {
#pragma unroll
        for (int b = 0; b < RB; ++b)
          stx(out + (r0 + t) * D + tc + 16 * b, expf(acc[a][b] - sHalfSq[t]) * scale);
      }
    }
  }
}

template <int D, typename T>
cudaError_t favor_impl(const void *x, const float *W, void *out, int64_t rows, cudaStream_t st) {
  const size_t smem = ((size_t)kRows * (D + 1) + (size_t)D * D + kRows) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(favor_features_kernel<D, T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (rows + kRows - 1) / kRows;
  const int64_t cap = 4 * 148;  // a few CTAs per SM, each walking many row tiles
  const unsigned grid = static_cast<unsigned>(ntiles < cap ? ntiles : cap);
  favor_features_kernel<D, T><<<grid, kThreads, smem, st>>>(
      static_cast<const T *>(x), W, static_cast<T *>(out), rows);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_favor_features(const void *x, const float *W, void *out, int64_t rows, int d,
                                  int is_bf16, cudaStream_t st) {
  if (is_bf16)
    return d == 64 ? favor_impl<64, __nv_bfloat16>(x, W, out, rows, st)
                   : favor_impl<128, __nv_bfloat16>(x, W, out, rows, st);
  return d == 64 ? favor_impl<64, float>(x, W, out, rows, st)
                 : favor_impl<128, float>(x, W, out, rows, st);
}

}  // namespace linattn
