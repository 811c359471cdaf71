// fp32-I/O forward pass on the CUDA cores (float32 FFMA end to end).
//
// Kernelised attention (page "Efficient Transformers: Linear Attention and Flash
// Attention", section "Linear attention: reordering the matmuls, not shrinking them"),
// causal as the chunked form of the running state of that page's section "The recurrent
// view: attention as an RNN":
//
//   K1  chunk aggregates  S_c = phi(K_c)^T V_c,  z_c = sum_{j in c} phi(k_j)
//   K2  exclusive prefix  S_<c = sum_{c' < c} S_c'   (or the per-head total)
//   K3  chunk outputs     num_i = phi(q_i) S_<c + sum_{j <= i, j in c} (phi(q_i).phi(k_j)) v_j
//                         den_i = phi(q_i).z_<c + sum_{j <= i, j in c}  phi(q_i).phi(k_j)
//                         out_i = num_i / den_i
//
// Non-causal runs K1, K2 (total) and K3 with the total state and no in-chunk term.
// This path serves float32 I/O, where the bf16 tensor-core products would not hold
// a 1e-4 relative error.  Tokens beyond n in the last chunk are masked.
#include "common.cuh"
#include "internal.h"

namespace linattn {
namespace {

constexpr int C = kSimtChunk;
constexpr int kThreads = 256;

// Four consecutive elements as floats.
__device__ __forceinline__ float4 load4(const float *p) {
  return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}
__device__ __forceinline__ void store1(float *p, float x) { *p = x; }
__device__ __forceinline__ void store1(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// Loads rows [t0, t0 + C) of one head into shared memory as floats (zero beyond n);
// applies phi when `apply_phi`, and leaves masked rows at zero either way.
template <int D, typename T>
__device__ __forceinline__ void load_rows(float *dst, const T *src, int valid, bool apply_phi) {
  for (int i = threadIdx.x; i < C * D / 4; i += kThreads) {
    const int row = i / (D / 4);
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < valid) {
      x = load4(src + 4 * i);
      if (apply_phi) {
        x.x = phi(x.x);
        x.y = phi(x.y);
        x.z = phi(x.z);
        x.w = phi(x.w);
      }
    }
    reinterpret_cast<float4 *>(dst)[i] = x;
  }
}

// K1: one CTA per (chunk, head).  Each thread owns a (D/16) x (D/16) block of S_c with
// rows r = tr + 16a and columns c = tc + 16b, so a warp reads consecutive columns.
template <int D, typename T>
__global__ void __launch_bounds__(kThreads) simt_chunk_state_kernel(const T *__restrict__ k,
                                                                    const T *__restrict__ v,
                                                                    float *__restrict__ ws,
                                                                    int64_t n, int64_t nchunks,
                                                                    int apply_phi) {
  extern __shared__ float4 smem_f4[];
  float *sK = reinterpret_cast<float *>(smem_f4);  // phi(K_c) [C][D]
  float *sV = sK + C * D;                          // V_c [C][D]
  const int64_t chunk = blockIdx.x % nchunks;
  const int64_t head = blockIdx.x / nchunks;
  const int64_t t0 = chunk * C;
  const int valid = n - t0 < C ? static_cast<int>(n - t0) : C;
  load_rows<D, T>(sK, k + (head * n + t0) * D, valid, apply_phi != 0);
  load_rows<D, T>(sV, v + (head * n + t0) * D, valid, false);
  __syncthreads();

  constexpr int R = D / 16;
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  float acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;
  for (int t = 0; t < valid; ++t) {
    float kr[R], vc[R];
#pragma unroll
    for (int a = 0; a < R; ++a) kr[a] = sK[t * D + tr + 16 * a];
#pragma unroll
    for (int b = 0; b < R; ++b) vc[b] = sV[t * D + tc + 16 * b];
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
      for (int b = 0; b < R; ++b) acc[a][b] = fmaf(kr[a], vc[b], acc[a][b]);
  }
  float *out = ws + (head * nchunks + chunk) * (int64_t)(D * D + D);
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) out[(tr + 16 * a) * D + tc + 16 * b] = acc[a][b];
  if (threadIdx.x < D) {
    float zs = 0.f;
    for (int t = 0; t < valid; ++t) zs += sK[t * D + threadIdx.x];
    out[D * D + threadIdx.x] = zs;
  }
}

// K2: per head, a sequential sweep over the segments for each group of 4 state elements
// (16-byte loads and stores; a state is [dk][dv] then [dk] floats with dk, dv multiples of 4, so
// a group never straddles S and z).  One thread per group keeps the running sum in registers:
// the sums over segments are independent per element, so no cross-thread scan is needed, and
// the sweep reads each aggregate once.
//   mode 0: ws[h][s] <- init[h] + sum_{s' < s} ws[h][s'] (exclusive prefix, in place)
//   mode 1: S_out + h*S_hs, z_out + h*z_hs <- init[h] + sum_s ws[h][s] (the total)
//   mode 2: ws[h][s] <- sum_{s' > s} ws[h][s'] (exclusive suffix, in place; the backward
//           pass's states of the later chunks)
// init[h] is the state before the first segment: (init_S[h] [dk][dv], init_z[h] [dk]), or zero
// when init_S is null.  The segments are summed in order, one group of elements per thread.
__global__ void __launch_bounds__(256) scan_states_kernel(float *__restrict__ ws, int64_t nseg,
                                                          int dk, int dv, int mode,
                                                          float *__restrict__ S_out, int64_t S_hs,
                                                          float *__restrict__ z_out, int64_t z_hs,
                                                          const float *__restrict__ init_S,
                                                          const float *__restrict__ init_z) {
  // launched programmatically: the next kernel may start now; this one reads the aggregates
  // of the kernel before it only once that kernel has finished
  grid_dependency_launch();
  grid_dependency_wait();
  const int64_t per4 = ((int64_t)dk * dv + dk) / 4;
  const int64_t blocks_per_head = (per4 + blockDim.x - 1) / blockDim.x;
  const int64_t head = blockIdx.x / blocks_per_head;
  const int64_t e4 = (blockIdx.x % blocks_per_head) * (int64_t)blockDim.x + threadIdx.x;
  if (e4 >= per4) return;
  float4 *base = reinterpret_cast<float4 *>(ws) + head * nseg * per4 + e4;
  constexpr int kBatch = 8;  // independent 16-byte loads in flight per thread
  float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
  if (init_S != nullptr) {
    const int64_t e = e4 * 4, dd = (int64_t)dk * dv;
    run = e < dd ? *reinterpret_cast<const float4 *>(init_S + head * dd + e)
                 : *reinterpret_cast<const float4 *>(init_z + head * dk + (e - dd));
  }
  const bool rev = mode == 2;
  for (int64_t s0 = 0; s0 < nseg; s0 += kBatch) {
    float4 x[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t s = rev ? nseg - 1 - (s0 + i) : s0 + i;
      x[i] = s0 + i < nseg ? base[s * per4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t s = rev ? nseg - 1 - (s0 + i) : s0 + i;
      if (mode != 1 && s0 + i < nseg) base[s * per4] = run;
      run.x += x[i].x;
      run.y += x[i].y;
      run.z += x[i].z;
      run.w += x[i].w;
    }
  }
  if (mode == 1) {
    const int64_t e = e4 * 4;
    const int64_t dd = (int64_t)dk * dv;
    float *dst = e < dd ? S_out + head * S_hs + e : z_out + head * z_hs + (e - dd);
    dst[0] = run.x;
    dst[1] = run.y;
    dst[2] = run.z;
    dst[3] = run.w;
  }
}

// K3: one CTA per (chunk, head).  Thread (ti, tc) owns rows i = ti + 16a (a < 4) and
// columns c = tc + 16b (b < D/16) of the chunk's output.
template <int D, bool CAUSAL, typename T>
__global__ void __launch_bounds__(kThreads) simt_chunk_out_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    T *__restrict__ out, const float *__restrict__ S, const float *__restrict__ z,
    int64_t S_chunk_stride, int64_t S_head_stride, int64_t z_chunk_stride,
    int64_t z_head_stride, int64_t n, int64_t nchunks, int apply_phi) {
  extern __shared__ float4 smem_f4[];
  float *sQ = reinterpret_cast<float *>(smem_f4);  // phi(Q_c) [C][D]
  float *sS = sQ + C * D;                          // S_<c [D][D]
  float *sz = sS + D * D;                          // z_<c [D]
  float *sDen = sz + D;                            // [C]
  float *sK = sDen + C;                            // phi(K_c)^T [D][C] (causal)
  float *sV = sK + C * D;                          // V_c [C][D]        (causal)
  float *sP = sV + C * D;                          // masked scores [C][C + 1] (causal)
  const int64_t chunk = blockIdx.x % nchunks;
  const int64_t head = blockIdx.x / nchunks;
  const int64_t t0 = chunk * C;
  const int valid = n - t0 < C ? static_cast<int>(n - t0) : C;
  const int64_t row0 = (head * n + t0) * D;

  load_rows<D, T>(sQ, q + row0, valid, apply_phi != 0);
  const float *Sg = S + head * S_head_stride + chunk * S_chunk_stride;
  const float *zg = z + head * z_head_stride + chunk * z_chunk_stride;
  for (int i = threadIdx.x; i < D * D / 4; i += kThreads)
    reinterpret_cast<float4 *>(sS)[i] = reinterpret_cast<const float4 *>(Sg)[i];
  if (threadIdx.x < D) sz[threadIdx.x] = zg[threadIdx.x];
  if (CAUSAL) {
    // phi(K_c) transposed, sK[r][j], so the score loop below reads consecutive j
    for (int i = threadIdx.x; i < C * D / 4; i += kThreads) {
      const int t = i % C, cg = i / C;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < valid) {
        x = load4(k + row0 + (int64_t)t * D + 4 * cg);
        if (apply_phi) {
          x.x = phi(x.x);
          x.y = phi(x.y);
          x.z = phi(x.z);
          x.w = phi(x.w);
        }
      }
      sK[(4 * cg + 0) * C + t] = x.x;
      sK[(4 * cg + 1) * C + t] = x.y;
      sK[(4 * cg + 2) * C + t] = x.z;
      sK[(4 * cg + 3) * C + t] = x.w;
    }
    load_rows<D, T>(sV, v + row0, valid, false);
  }
  __syncthreads();

  if (CAUSAL) {
    // scores P[i][j] = phi(q_i).phi(k_j) for j <= i, 0 above the diagonal
    for (int e = threadIdx.x; e < C * C; e += kThreads) {
      const int i = e / C, j = e % C;
      float s = 0.f;
      if (j <= i) {
#pragma unroll 8
        for (int r = 0; r < D; ++r) s = fmaf(sQ[i * D + r], sK[r * C + j], s);
      }
      sP[i * (C + 1) + j] = s;
    }
  }
  // denominators: phi(q_i).z_<c + sum_{j<=i} P[i][j]
  if (threadIdx.x < C) {
    const int i = threadIdx.x;
    float den = 0.f;
    for (int r = 0; r < D; ++r) den = fmaf(sQ[i * D + r], sz[r], den);
    sDen[i] = den;
  }
  __syncthreads();
  if (CAUSAL && threadIdx.x < C) {
    const int i = threadIdx.x;
    float add = 0.f;
    for (int j = 0; j <= i; ++j) add += sP[i * (C + 1) + j];
    sDen[i] += add;
  }

  constexpr int RB = D / 16;
  const int ti = threadIdx.x / 16, tc = threadIdx.x % 16;
  float acc[4][RB];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < RB; ++b) acc[a][b] = 0.f;
  for (int r = 0; r < D; ++r) {
    float qa[4], sb[RB];
#pragma unroll
    for (int a = 0; a < 4; ++a) qa[a] = sQ[(ti + 16 * a) * D + r];
#pragma unroll
    for (int b = 0; b < RB; ++b) sb[b] = sS[r * D + tc + 16 * b];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(qa[a], sb[b], acc[a][b]);
  }
  if (CAUSAL) {
    for (int j = 0; j < valid; ++j) {
      float pa[4], vb[RB];
#pragma unroll
      for (int a = 0; a < 4; ++a) pa[a] = sP[(ti + 16 * a) * (C + 1) + j];
#pragma unroll
      for (int b = 0; b < RB; ++b) vb[b] = sV[j * D + tc + 16 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(pa[a], vb[b], acc[a][b]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = ti + 16 * a;
    if (i < valid) {
      const float inv = 1.f / sDen[i];
#pragma unroll
      for (int b = 0; b < RB; ++b) store1(out + row0 + (int64_t)i * D + tc + 16 * b, acc[a][b] * inv);
    }
  }
}

template <int D>
size_t chunk_out_smem(bool causal) {
  size_t f = (size_t)C * D + (size_t)D * D + D + C;
  if (causal) f += 2 * (size_t)C * D + (size_t)C * (C + 1);
  return f * sizeof(float);
}

template <int D, typename T>
cudaError_t chunk_state_impl(const void *k, const void *v, float *ws, int64_t heads, int64_t n,
                             int apply_phi, cudaStream_t st) {
  const int64_t nchunks = (n + C - 1) / C;
  const size_t smem = 2 * (size_t)C * D * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(simt_chunk_state_kernel<D, T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  simt_chunk_state_kernel<D, T><<<(unsigned)(nchunks * heads), kThreads, smem, st>>>(
      static_cast<const T *>(k), static_cast<const T *>(v), ws, n, nchunks, apply_phi);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

template <int D, bool CAUSAL, typename T>
cudaError_t chunk_out_impl(const void *q, const void *k, const void *v, void *out,
                           const float *S, const float *z, int64_t Scs, int64_t Shs,
                           int64_t zcs, int64_t zhs, int64_t heads, int64_t n, int apply_phi,
                           cudaStream_t st) {
  const int64_t nchunks = (n + C - 1) / C;
  const size_t smem = chunk_out_smem<D>(CAUSAL);
  cudaError_t e = cudaFuncSetAttribute(simt_chunk_out_kernel<D, CAUSAL, T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  simt_chunk_out_kernel<D, CAUSAL, T><<<(unsigned)(nchunks * heads), kThreads, smem, st>>>(
      static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v),
      static_cast<T *>(out), S, z, Scs, Shs, zcs, zhs, n, nchunks, apply_phi);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

template <typename T>
cudaError_t chunk_state_t(const void *k, const void *v, float *ws, int64_t heads, int64_t n,
                          int d, int apply_phi, cudaStream_t st) {
  return d == 64 ? chunk_state_impl<64, T>(k, v, ws, heads, n, apply_phi, st)
                 : chunk_state_impl<128, T>(k, v, ws, heads, n, apply_phi, st);
}

template <typename T>
cudaError_t chunk_out_t(const void *q, const void *k, const void *v, void *out, const float *S,
                        const float *z, int64_t Scs, int64_t Shs, int64_t zcs, int64_t zhs,
                        int64_t heads, int64_t n, int d, int causal, int apply_phi,
                        cudaStream_t st) {
  if (d == 64)
    return causal ? chunk_out_impl<64, true, T>(q, k, v, out, S, z, Scs, Shs, zcs, zhs, heads,
                                                n, apply_phi, st)
                  : chunk_out_impl<64, false, T>(q, k, v, out, S, z, Scs, Shs, zcs, zhs, heads,
                                                 n, apply_phi, st);
  return causal ? chunk_out_impl<128, true, T>(q, k, v, out, S, z, Scs, Shs, zcs, zhs, heads, n,
                                               apply_phi, st)
                : chunk_out_impl<128, false, T>(q, k, v, out, S, z, Scs, Shs, zcs, zhs, heads, n,
                                                apply_phi, st);
}

}  // namespace

cudaError_t launch_simt_chunk_state(const void *k, const void *v, float *ws, int64_t heads,
                                    int64_t n, int d, int is_bf16, int features,
                                    cudaStream_t st) {
  return is_bf16 ? chunk_state_t<__nv_bfloat16>(k, v, ws, heads, n, d, !features, st)
                 : chunk_state_t<float>(k, v, ws, heads, n, d, !features, st);
}

cudaError_t launch_scan_states(float *ws, int64_t heads, int64_t nseg, int dk, int dv, int mode,
                               float *S_out, int64_t S_hs, float *z_out, int64_t z_hs,
                               const float *init_S, const float *init_z, cudaStream_t st) {
  const int64_t per4 = ((int64_t)dk * dv + dk) / 4;
  cudaError_t e = launch_programmatic(scan_states_kernel,
                                      dim3((unsigned)(((per4 + 255) / 256) * heads)), dim3(256), 0,
                                      st, ws, nseg, dk, dv, mode, S_out, S_hs, z_out, z_hs, init_S,
                                      init_z);
  if (e != cudaSuccess) return e;
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

// Sum of gathered states: for each head h, (S_out[h], z_out[h]) <- sum over i in [0, count),
// i != skip, of states[i][h] (each [D*d + D]: S row-major then z), added in order of i; zero
// when no state is summed.
__global__ void __launch_bounds__(256) sum_states_kernel(const float *__restrict__ states,
                                                         int64_t count, int64_t skip,
                                                         int64_t heads, int d,
                                                         float *__restrict__ S_out,
                                                         float *__restrict__ z_out) {
  const int64_t per4 = ((int64_t)d * d + d) / 4;
  const int64_t blocks_per_head = (per4 + blockDim.x - 1) / blockDim.x;
  const int64_t head = blockIdx.x / blocks_per_head;
  const int64_t e4 = (blockIdx.x % blocks_per_head) * (int64_t)blockDim.x + threadIdx.x;
  if (e4 >= per4) return;
  const float4 *src = reinterpret_cast<const float4 *>(states) + head * per4 + e4;
  float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t i = 0; i < count; ++i) {
    if (i == skip) continue;
    const float4 x = src[i * heads * per4];
    run.x += x.x;
    run.y += x.y;
    run.z += x.z;
    run.w += x.w;
  }
  const int64_t e = e4 * 4, dd = (int64_t)d * d;
  float4 *dst = e < dd ? reinterpret_cast<float4 *>(S_out + head * dd + e)
                       : reinterpret_cast<float4 *>(z_out + head * d + (e - dd));
  *dst = run;
}

cudaError_t launch_sum_states(const float *states, int64_t count, int64_t skip, int64_t heads,
                              int d, float *S_out, float *z_out, cudaStream_t st) {
  const int64_t per4 = ((int64_t)d * d + d) / 4;
  sum_states_kernel<<<(unsigned)(((per4 + 255) / 256) * heads), 256, 0, st>>>(
      states, count, skip, heads, d, S_out, z_out);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

cudaError_t launch_simt_chunk_out(const void *q, const void *k, const void *v, void *out,
                                  const float *S, const float *z, int64_t Scs, int64_t Shs,
                                  int64_t zcs, int64_t zhs, int64_t heads, int64_t n, int d,
                                  int causal, int is_bf16, int features, cudaStream_t st) {
  return is_bf16 ? chunk_out_t<__nv_bfloat16>(q, k, v, out, S, z, Scs, Shs, zcs, zhs, heads, n,
                                               d, causal, !features, st)
                 : chunk_out_t<float>(q, k, v, out, S, z, Scs, Shs, zcs, zhs, heads, n, d,
                                      causal, !features, st);
}

}  // namespace linattn
