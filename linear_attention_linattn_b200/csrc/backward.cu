// Backward pass of the forward on the CUDA cores (float32 FFMA; bf16 or fp32 I/O).
//
// The pages define the forward only; its gradients follow by the chain rule.  Per head, with
// the forward written as weights w_ij = phi(q_i).phi(k_j) (j <= i when causal),
// den_i = sum_j w_ij and out_i = sum_j w_ij v_j / den_i, and g = dL/dout:
//
//   a_i = g_i / den_i,   b_i = -(g_i . out_i) / den_i,   dL/dw_ij = v_j . a_i + b_i
//   dphi(q_i) = sum_j dL/dw_ij phi(k_j)  = S_i a_i + z_i b_i          (S_i, z_i: the state)
//   dphi(k_j) = sum_i dL/dw_ij phi(q_i)  = R_j v_j + r_j              (R_j, r_j: see below)
//   dv_j      = sum_i w_ij a_i           = R_j^T phi(k_j)
//   dq = dphi(q) * phi'(q),  dk = dphi(k) * phi'(k),  phi'(x) = 1 above zero, exp(x) below
//
// with the "reverse state" R_j = sum_{i >= j} phi(q_i) a_i^T (D x d) and r_j = sum_{i >= j}
// phi(q_i) b_i (D), summed over every i in the non-causal mode.  So the backward is two
// chunked passes in the shape of the forward: a prefix pass over (phi(K), V) that yields dq
// (and stores a, b), and a suffix pass over (phi(Q), a, b) that yields dk and dv:
//
//   K1  forward chunk states (simt_forward.cu)       K2  exclusive prefix (or total)
//   B1  per chunk: den, out, a, b; dq
//   B2  per chunk: R_c = phi(Q_c)^T A_c, r_c = phi(Q_c)^T b_c
//   K2  exclusive suffix (or total) of (R_c, r_c)
//   B3  per chunk: dk, dv
//
// phi'(x) is read off phi(x): phi > 1 exactly when x > 0 (phi = x + 1), and phi = exp(x) at or
// below zero, so phi'(x) = phi(x) > 1 ? 1 : phi(x).  Rows past n are masked (their a, b are
// zero, so they add nothing to any sum).
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace linattn {
namespace {

constexpr int C = kSimtChunk;  // tokens per chunk (64)
constexpr int kThreads = 256;

__device__ __forceinline__ float4 ld4(const float *p) {
  return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}
__device__ __forceinline__ void st1(float *p, float x) { *p = x; }
__device__ __forceinline__ void st1(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ float dphi_from_phi(float f) { return f > 1.f ? 1.f : f; }

// Rows [0, C) of a chunk into shared memory with a padded row stride of D + 1 floats (so that
// both row- and column-wise sweeps are free of bank conflicts); zero past `valid`; phi
// applied when asked.
template <int D, typename T>
__device__ __forceinline__ void load_pad(float *dst, const T *src, int valid, bool apply_phi) {
  for (int i = threadIdx.x; i < C * D / 4; i += kThreads) {
    const int row = i / (D / 4), c4 = i % (D / 4);
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < valid) {
      x = ld4(src + (int64_t)row * D + 4 * c4);
      if (apply_phi) {
        x.x = phi(x.x);
        x.y = phi(x.y);
        x.z = phi(x.z);
        x.w = phi(x.w);
      }
    }
    float *p = dst + row * (D + 1) + 4 * c4;
    p[0] = x.x;
    p[1] = x.y;
    p[2] = x.z;
    p[3] = x.w;
  }
}

// A [D][d] state from global memory, transposed into shared memory: dst[c][r] = S[r][c]
// (row stride D + 1).
template <int D>
__device__ __forceinline__ void load_state_t(float *dst, const float *S) {
  for (int e = threadIdx.x; e < D * D; e += kThreads) {
    const int r = e / D, c = e % D;
    dst[c * (D + 1) + r] = S[e];
  }
}

// W[i][j] = sum_r X[i][r] Y[j][r] + add[i] for j <= i, zero above the diagonal (X, Y: [C][D+1]
// tiles; add may be null).  Each thread computes a 4 x 4 block, rows ti + 16a and columns
// tj + 16b, so a sweep over r loads 8 values for 16 FMAs.
template <int D>
__device__ __forceinline__ void masked_products(float *W, const float *X, const float *Y,
                                                const float *add) {
  constexpr int PD = D + 1;
  const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 4
  for (int r = 0; r < D; ++r) {
    float x[4], y[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) x[a] = X[(ti + 16 * a) * PD + r];
#pragma unroll
    for (int b = 0; b < 4; ++b) y[b] = Y[(tj + 16 * b) * PD + r];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(x[a], y[b], acc[a][b]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = ti + 16 * a;
    const float ad = add ? add[i] : 0.f;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = tj + 16 * b;
      W[i * (C + 1) + j] = j <= i ? acc[a][b] + ad : 0.f;
    }
  }
}

template <int D>
constexpr size_t bwd_smem_floats(bool causal) {
  // four [C][D+1] tiles, one transposed state [D][D+1], z or r [D], [C] den and b,
  // and the [C][C+1] score block (causal)
  return 4 * (size_t)C * (D + 1) + (size_t)D * (D + 1) + D + 2 * C +
         (causal ? (size_t)C * (C + 1) : 0);
}

// B1: one CTA per (chunk, head).  S, z: the state before the chunk (causal: the exclusive
// prefix; non-causal: the total) at S + head*S_hs + chunk*S_cs, z likewise.
template <int D, bool CAUSAL, typename T>
__global__ void __launch_bounds__(kThreads) bwd_q_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const T *__restrict__ g, T *__restrict__ dq, const float *__restrict__ S,
    const float *__restrict__ z, int64_t S_cs, int64_t S_hs, int64_t z_cs, int64_t z_hs,
    float *__restrict__ a_out, float *__restrict__ b_out, int64_t n, int64_t nchunks) {
  constexpr int PD = D + 1;
  extern __shared__ float4 smem_f4[];
  float *sQ = reinterpret_cast<float *>(smem_f4);  // phi(Q_c)            [C][PD]
  float *sK = sQ + C * PD;                          // phi(K_c)            [C][PD]
  float *sV = sK + C * PD;                          // V_c                 [C][PD]
  float *sA = sV + C * PD;                          // G_c, then A_c       [C][PD]
  float *sST = sA + C * PD;                         // S^T                 [D][PD]
  float *sz = sST + D * PD;                         // z                   [D]
  float *sDen = sz + D;                             // den                 [C]
  float *sB = sDen + C;                             // b                   [C]
  float *sW = sB + C;                               // scores, then dL/dw  [C][C+1]
  const int64_t chunk = blockIdx.x % nchunks;
  const int64_t head = blockIdx.x / nchunks;
  const int64_t t0 = chunk * C;
  const int valid = n - t0 < C ? static_cast<int>(n - t0) : C;
  const int64_t row0 = (head * n + t0) * D;

  load_pad<D, T>(sQ, q + row0, valid, true);
  load_pad<D, T>(sA, g + row0, valid, false);
  if (CAUSAL) {
    load_pad<D, T>(sK, k + row0, valid, true);
    load_pad<D, T>(sV, v + row0, valid, false);
  }
  load_state_t<D>(sST, S + head * S_hs + chunk * S_cs);
  if (threadIdx.x < D) sz[threadIdx.x] = z[head * z_hs + chunk * z_cs + threadIdx.x];
  __syncthreads();

  if (CAUSAL) {
    masked_products<D>(sW, sQ, sK, nullptr);  // P[i][j] = phi(q_i).phi(k_j), j <= i
    __syncthreads();
  }
  if (threadIdx.x < C) {
    const int i = threadIdx.x;
    float den = 0.f;
    for (int r = 0; r < D; ++r) den = fmaf(sQ[i * PD + r], sz[r], den);
    if (CAUSAL)
      for (int j = 0; j <= i; ++j) den += sW[i * (C + 1) + j];
    sDen[i] = i < valid ? den : 1.f;  // rows past n: any finite value (their g is zero)
  }
  __syncthreads();

  // out = (phi(Q) S + P V) / den; then a = g / den and b = -(g . out) / den
  constexpr int RB = D / 16;
  const int ti = threadIdx.x / 16, tx = threadIdx.x % 16;
  {
    float acc[4][RB];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[a][b] = 0.f;
    for (int r = 0; r < D; ++r) {
      float qa[4], sb[RB];
#pragma unroll
      for (int a = 0; a < 4; ++a) qa[a] = sQ[(ti + 16 * a) * PD + r];
#pragma unroll
      for (int b = 0; b < RB; ++b) sb[b] = sST[(tx + 16 * b) * PD + r];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(qa[a], sb[b], acc[a][b]);
    }
    if (CAUSAL) {
      for (int j = 0; j < valid; ++j) {
        float pa[4], vb[RB];
#pragma unroll
        for (int a = 0; a < 4; ++a) pa[a] = sW[(ti + 16 * a) * (C + 1) + j];
#pragma unroll
        for (int b = 0; b < RB; ++b) vb[b] = sV[j * PD + tx + 16 * b];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(pa[a], vb[b], acc[a][b]);
      }
    }
    float gdot[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = ti + 16 * a;
      const float inv = 1.f / sDen[i];
      gdot[a] = 0.f;
#pragma unroll
      for (int b = 0; b < RB; ++b) gdot[a] = fmaf(sA[i * PD + tx + 16 * b], acc[a][b] * inv, gdot[a]);
    }
    // the 16 threads of a row are lanes tx = 0..15 of one half-warp
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int m = 8; m >= 1; m >>= 1) gdot[a] += __shfl_xor_sync(0xffffffffu, gdot[a], m);
    __syncthreads();  // every thread has read G before A overwrites it
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = ti + 16 * a;
      const bool live = i < valid;
      const float inv = 1.f / sDen[i];
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        const int c = tx + 16 * b;
        const float av = live ? sA[i * PD + c] * inv : 0.f;
        sA[i * PD + c] = av;
        if (live) a_out[(head * n + t0 + i) * D + c] = av;
      }
      if (tx == 0) {
        const float bv = live ? -gdot[a] * inv : 0.f;
        sB[i] = bv;
        if (live) b_out[head * n + t0 + i] = bv;
      }
    }
  }
  __syncthreads();

  if (CAUSAL) {
    masked_products<D>(sW, sA, sV, sB);  // dL/dw[i][j] = v_j . a_i + b_i, j <= i
    __syncthreads();
  }

  // dphi(q_i)[r] = sum_c S[r][c] a_i[c] + z[r] b_i + sum_{j <= i} dL/dw[i][j] phi(k_j)[r]
  {
    float acc[4][RB];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[a][b] = sz[tx + 16 * b] * sB[ti + 16 * a];
    for (int c = 0; c < D; ++c) {
      float aa[4], sr[RB];
#pragma unroll
      for (int a = 0; a < 4; ++a) aa[a] = sA[(ti + 16 * a) * PD + c];
#pragma unroll
      for (int b = 0; b < RB; ++b) sr[b] = sST[c * PD + tx + 16 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(aa[a], sr[b], acc[a][b]);
    }
    if (CAUSAL) {
      for (int j = 0; j < valid; ++j) {
        float m[4], kr[RB];
#pragma unroll
        for (int a = 0; a < 4; ++a) m[a] = sW[(ti + 16 * a) * (C + 1) + j];
#pragma unroll
        for (int b = 0; b < RB; ++b) kr[b] = sK[j * PD + tx + 16 * b];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(m[a], kr[b], acc[a][b]);
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = ti + 16 * a;
      if (i < valid) {
#pragma unroll
        for (int b = 0; b < RB; ++b) {
          const int r = tx + 16 * b;
          st1(dq + row0 + (int64_t)i * D + r, acc[a][b] * dphi_from_phi(sQ[i * PD + r]));
        }
      }
    }
  }
}

// B2: the reverse state of one chunk, R_c[r][c] = sum_i phi(q_i)[r] a_i[c] and
// r_c[r] = sum_i phi(q_i)[r] b_i, into ws[head][chunk][D*D + D].
template <int D, typename T>
__global__ void __launch_bounds__(kThreads) bwd_state_kernel(const T *__restrict__ q,
                                                             const float *__restrict__ a_in,
                                                             const float *__restrict__ b_in,
                                                             float *__restrict__ ws, int64_t n,
                                                             int64_t nchunks) {
  extern __shared__ float4 smem_f4[];
  float *sQ = reinterpret_cast<float *>(smem_f4);  // phi(Q_c) [C][D]
  float *sA = sQ + C * D;                          // A_c      [C][D]
  float *sB = sA + C * D;                          // b_c      [C]
  const int64_t chunk = blockIdx.x % nchunks;
  const int64_t head = blockIdx.x / nchunks;
  const int64_t t0 = chunk * C;
  const int valid = n - t0 < C ? static_cast<int>(n - t0) : C;
  for (int i = threadIdx.x; i < C * D / 4; i += kThreads) {
    const int row = i / (D / 4);
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
    if (row < valid) {
      x = ld4(q + (head * n + t0) * D + 4 * i);
      x.x = phi(x.x);
      x.y = phi(x.y);
      x.z = phi(x.z);
      x.w = phi(x.w);
      y = ld4(a_in + (head * n + t0) * D + 4 * i);
    }
    reinterpret_cast<float4 *>(sQ)[i] = x;
    reinterpret_cast<float4 *>(sA)[i] = y;
  }
  if (threadIdx.x < C) sB[threadIdx.x] = threadIdx.x < valid ? b_in[head * n + t0 + threadIdx.x] : 0.f;
  __syncthreads();

  constexpr int R = D / 16;
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  float acc[R][R];
#pragma unroll
  for (int x = 0; x < R; ++x)
#pragma unroll
    for (int y = 0; y < R; ++y) acc[x][y] = 0.f;
  for (int t = 0; t < valid; ++t) {
    float qr[R], ac[R];
#pragma unroll
    for (int x = 0; x < R; ++x) qr[x] = sQ[t * D + tr + 16 * x];
#pragma unroll
    for (int y = 0; y < R; ++y) ac[y] = sA[t * D + tc + 16 * y];
#pragma unroll
    for (int x = 0; x < R; ++x)
#pragma unroll
      for (int y = 0; y < R; ++y) acc[x][y] = fmaf(qr[x], ac[y], acc[x][y]);
  }
  float *out = ws + (head * nchunks + chunk) * (int64_t)(D * D + D);
#pragma unroll
  for (int x = 0; x < R; ++x)
#pragma unroll
    for (int y = 0; y < R; ++y) out[(tr + 16 * x) * D + tc + 16 * y] = acc[x][y];
  if (threadIdx.x < D) {
    float rs = 0.f;
    for (int t = 0; t < valid; ++t) rs = fmaf(sQ[t * D + threadIdx.x], sB[t], rs);
    out[D * D + threadIdx.x] = rs;
  }
}

// B3: one CTA per (chunk, head).  R, r: the reverse state after the chunk (causal: the
// exclusive suffix; non-causal: the total).
template <int D, bool CAUSAL, typename T>
__global__ void __launch_bounds__(kThreads) bwd_kv_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const float *__restrict__ a_in, const float *__restrict__ b_in, const float *__restrict__ R,
    const float *__restrict__ rz, int64_t R_cs, int64_t R_hs, int64_t r_cs, int64_t r_hs,
    T *__restrict__ dk, T *__restrict__ dv, int64_t n, int64_t nchunks) {
  constexpr int PD = D + 1;
  extern __shared__ float4 smem_f4[];
  float *sQ = reinterpret_cast<float *>(smem_f4);  // phi(Q_c)            [C][PD]
  float *sK = sQ + C * PD;                          // phi(K_c)            [C][PD]
  float *sV = sK + C * PD;                          // V_c                 [C][PD]
  float *sA = sV + C * PD;                          // A_c                 [C][PD]
  float *sRT = sA + C * PD;                         // R^T                 [D][PD]
  float *sr = sRT + D * PD;                         // r                   [D]
  float *sB = sr + D;                               // b                   [C]
  float *sW = sB + 2 * C;                           // scores, then dL/dw  [C][C+1]
  const int64_t chunk = blockIdx.x % nchunks;
  const int64_t head = blockIdx.x / nchunks;
  const int64_t t0 = chunk * C;
  const int valid = n - t0 < C ? static_cast<int>(n - t0) : C;
  const int64_t row0 = (head * n + t0) * D;

  load_pad<D, T>(sK, k + row0, valid, true);
  load_pad<D, T>(sV, v + row0, valid, false);
  if (CAUSAL) {
    load_pad<D, T>(sQ, q + row0, valid, true);
    load_pad<D, float>(sA, a_in + row0, valid, false);
    if (threadIdx.x < C) sB[threadIdx.x] = threadIdx.x < valid ? b_in[head * n + t0 + threadIdx.x] : 0.f;
  }
  load_state_t<D>(sRT, R + head * R_hs + chunk * R_cs);
  if (threadIdx.x < D) sr[threadIdx.x] = rz[head * r_hs + chunk * r_cs + threadIdx.x];
  __syncthreads();

  constexpr int RB = D / 16;
  const int tj = threadIdx.x / 16, tx = threadIdx.x % 16;
  if (CAUSAL) {
    masked_products<D>(sW, sQ, sK, nullptr);  // P[i][j] = phi(q_i).phi(k_j), i >= j
    __syncthreads();
  }
  // dv_j[c] = sum_r R[r][c] phi(k_j)[r] + sum_{i >= j} P[i][j] a_i[c]
  {
    float acc[4][RB];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[a][b] = 0.f;
    for (int r = 0; r < D; ++r) {
      float ka[4], rb[RB];
#pragma unroll
      for (int a = 0; a < 4; ++a) ka[a] = sK[(tj + 16 * a) * PD + r];
#pragma unroll
      for (int b = 0; b < RB; ++b) rb[b] = sRT[(tx + 16 * b) * PD + r];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(ka[a], rb[b], acc[a][b]);
    }
    if (CAUSAL) {
      for (int i = 0; i < valid; ++i) {
        float p[4], ab[RB];
#pragma unroll
        for (int a = 0; a < 4; ++a) p[a] = sW[i * (C + 1) + tj + 16 * a];
#pragma unroll
        for (int b = 0; b < RB; ++b) ab[b] = sA[i * PD + tx + 16 * b];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(p[a], ab[b], acc[a][b]);
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int j = tj + 16 * a;
      if (j < valid) {
#pragma unroll
        for (int b = 0; b < RB; ++b) st1(dv + row0 + (int64_t)j * D + tx + 16 * b, acc[a][b]);
      }
    }
  }
  if (CAUSAL) {
    __syncthreads();  // every thread is done with P
    masked_products<D>(sW, sA, sV, sB);  // dL/dw[i][j] = v_j . a_i + b_i, i >= j
    __syncthreads();
  }
  // dphi(k_j)[r] = sum_c R[r][c] v_j[c] + r[r] + sum_{i >= j} dL/dw[i][j] phi(q_i)[r]
  {
    float acc[4][RB];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[a][b] = sr[tx + 16 * b];
    for (int c = 0; c < D; ++c) {
      float va[4], rb[RB];
#pragma unroll
      for (int a = 0; a < 4; ++a) va[a] = sV[(tj + 16 * a) * PD + c];
#pragma unroll
      for (int b = 0; b < RB; ++b) rb[b] = sRT[c * PD + tx + 16 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(va[a], rb[b], acc[a][b]);
    }
    if (CAUSAL) {
      for (int i = 0; i < valid; ++i) {
        float m[4], qb[RB];
#pragma unroll
        for (int a = 0; a < 4; ++a) m[a] = sW[i * (C + 1) + tj + 16 * a];
#pragma unroll
        for (int b = 0; b < RB; ++b) qb[b] = sQ[i * PD + tx + 16 * b];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(m[a], qb[b], acc[a][b]);
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int j = tj + 16 * a;
      if (j < valid) {
#pragma unroll
        for (int b = 0; b < RB; ++b) {
          const int r = tx + 16 * b;
          st1(dk + row0 + (int64_t)j * D + r, acc[a][b] * dphi_from_phi(sK[j * PD + r]));
        }
      }
    }
  }
}

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int D, bool CAUSAL, typename T>
cudaError_t backward_impl(const T *q, const T *k, const T *v, const T *g, T *dq, T *dk, T *dv,
                          int64_t heads, int64_t n, float *ws, cudaStream_t st) {
  const int64_t nchunks = (n + C - 1) / C;
  const int64_t per = (int64_t)D * D + D;
  float *Sf = ws;                          // forward chunk states  [heads][nchunks][per]
  float *Sr = Sf + heads * nchunks * per;  // reverse chunk states  [heads][nchunks][per]
  float *A = Sr + heads * nchunks * per;   // a                     [heads][n][D]
  float *Bv = A + heads * n * D;           // b                     [heads][n]
  float *tot = Bv + heads * n;             // non-causal: forward total, then reverse total
  const unsigned grid = static_cast<unsigned>(nchunks * heads);
  const size_t smem_big = bwd_smem_floats<D>(CAUSAL) * sizeof(float);
  const size_t smem_state = (2 * (size_t)C * D + C) * sizeof(float);
  cudaError_t e;
  if ((e = set_smem(bwd_q_kernel<D, CAUSAL, T>, smem_big)) != cudaSuccess) return e;
  if ((e = set_smem(bwd_kv_kernel<D, CAUSAL, T>, smem_big)) != cudaSuccess) return e;
  if ((e = set_smem(bwd_state_kernel<D, T>, smem_state)) != cudaSuccess) return e;

  // K1 + K2: the forward states of the chunks (prefix) or the head (total)
  e = launch_simt_chunk_state(k, v, Sf, heads, n, D, std::is_same<T, __nv_bfloat16>::value, 0,
                              st);
  if (e != cudaSuccess) return e;
  int64_t Scs = per, Shs = nchunks * per;
  const float *Sbase = Sf;
  if (CAUSAL) {
    e = launch_scan_states(Sf, heads, nchunks, D, D, 0, nullptr, 0, nullptr, 0, nullptr, nullptr, st);
  } else {
    e = launch_scan_states(Sf, heads, nchunks, D, D, 1, tot, per, tot + (int64_t)D * D, per, nullptr,
                           nullptr, st);
    Scs = 0;
    Shs = per;
    Sbase = tot;
  }
  if (e != cudaSuccess) return e;
  // B1: dq, a, b
  bwd_q_kernel<D, CAUSAL, T><<<grid, kThreads, smem_big, st>>>(
      q, k, v, g, dq, Sbase, Sbase + (int64_t)D * D, Scs, Shs, Scs, Shs, A, Bv, n, nchunks);
  count_launches(1);
  record_launch_event(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // B2 + K2: the reverse states (suffix) or their total
  bwd_state_kernel<D, T><<<grid, kThreads, smem_state, st>>>(q, A, Bv, Sr, n, nchunks);
  count_launches(1);
  record_launch_event(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int64_t Rcs = per, Rhs = nchunks * per;
  const float *Rbase = Sr;
  if (CAUSAL) {
    e = launch_scan_states(Sr, heads, nchunks, D, D, 2, nullptr, 0, nullptr, 0, nullptr, nullptr, st);
  } else {
    e = launch_scan_states(Sr, heads, nchunks, D, D, 1, tot, per, tot + (int64_t)D * D, per, nullptr,
                           nullptr, st);
    Rcs = 0;
    Rhs = per;
    Rbase = tot;
  }
  if (e != cudaSuccess) return e;
  // B3: dk, dv
  bwd_kv_kernel<D, CAUSAL, T><<<grid, kThreads, smem_big, st>>>(
      q, k, v, A, Bv, Rbase, Rbase + (int64_t)D * D, Rcs, Rhs, Rcs, Rhs, dk, dv, n, nchunks);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

template <int D, typename T>
cudaError_t backward_d(const void *q, const void *k, const void *v, const void *g, void *dq,
                       void *dk, void *dv, int64_t heads, int64_t n, int causal, float *ws,
                       cudaStream_t st) {
  const T *q_ = static_cast<const T *>(q), *k_ = static_cast<const T *>(k);
  const T *v_ = static_cast<const T *>(v), *g_ = static_cast<const T *>(g);
  T *dq_ = static_cast<T *>(dq), *dk_ = static_cast<T *>(dk), *dv_ = static_cast<T *>(dv);
  return causal ? backward_impl<D, true, T>(q_, k_, v_, g_, dq_, dk_, dv_, heads, n, ws, st)
                : backward_impl<D, false, T>(q_, k_, v_, g_, dq_, dk_, dv_, heads, n, ws, st);
}

}  // namespace

size_t backward_workspace_floats(int64_t heads, int64_t n, int d, int causal) {
  const int64_t nchunks = (n + C - 1) / C;
  const int64_t per = (int64_t)d * d + d;
  return (size_t)(2 * heads * nchunks * per + heads * n * d + heads * n +
                  (causal ? 0 : heads * per));
}

cudaError_t backward(const void *q, const void *k, const void *v, const void *g, void *dq,
                     void *dk, void *dv, int64_t heads, int64_t n, int d, int causal, int is_bf16,
                     float *ws, cudaStream_t st) {
  if (is_bf16)
    return d == 64 ? backward_d<64, __nv_bfloat16>(q, k, v, g, dq, dk, dv, heads, n, causal, ws, st)
                   : backward_d<128, __nv_bfloat16>(q, k, v, g, dq, dk, dv, heads, n, causal, ws,
                                                    st);
  return d == 64 ? backward_d<64, float>(q, k, v, g, dq, dk, dv, heads, n, causal, ws, st)
                 : backward_d<128, float>(q, k, v, g, dq, dk, dv, heads, n, causal, ws, st);
}

}  // namespace linattn
