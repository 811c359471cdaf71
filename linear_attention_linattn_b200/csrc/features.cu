// FAVOR+ positive random features.
//
// Performer's FAVOR+ is named on the page "Efficient Transformers: Linear Attention and Flash
// Attention" (section "Linear attention: reordering the matmuls, not shrinking them") as a
// feature map whose dot products approximate the softmax kernel exp(q . k).  Its
// positive-feature form, with m random rows w_i of W (the caller draws them):
//
//     phi(x)_i = exp(w_i . x - |x|^2 / 2) / sqrt(m),   i < m
//
// The features are positive, so linattn_forward_features runs the linear-attention pass on
// them with no further feature map.
//
// fp32 I/O: CUDA cores.  Each CTA holds W (transposed) in shared memory and walks tiles of 64
// rows; thread (ti, tc) computes rows ti + 16a and features tc + 16b.
// bf16 I/O: tensor cores.  X W^T is a [rows x d] x [d x m] product: tcgen05.mma (M = 128 rows,
// N = m, K = d) into tensor memory, with W split into two bf16 parts (W = W_hi + W_lo, both
// products accumulated) so the exponent sees W to about 2^-16; x is bf16 already, so the
// product is exact up to fp32 accumulation.  The epilogue takes |x|^2 from the x tile in
// shared memory, applies exp(. - |x|^2/2)/sqrt(m), and stores bf16 rows.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace linattn {
namespace {

constexpr int kRows = 64;
constexpr int kThreads = 256;

__device__ __forceinline__ float4 ldx(const float *p) {
  return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ void stx(float *p, float x) { *p = x; }

template <int D, int M, typename T>
__global__ void __launch_bounds__(kThreads) favor_features_kernel(const T *__restrict__ x,
                                                                  const float *__restrict__ W,
                                                                  T *__restrict__ out,
                                                                  int64_t rows) {
  constexpr int PD = D + 1;
  extern __shared__ float4 smem_f4[];
  float *sX = reinterpret_cast<float *>(smem_f4);  // x rows            [kRows][PD]
  float *sWT = sX + kRows * PD;                     // W transposed      [D][M]: sWT[r][i]
  float *sHalfSq = sWT + D * M;                     // |x_t|^2 / 2       [kRows]
  // W once per CTA (the CTA then walks many row tiles); read transposed from global memory
  // (L2-resident) so the shared-memory writes are consecutive
  for (int e = threadIdx.x; e < D * M; e += kThreads) {
    const int r = e / M, i = e % M;
    sWT[e] = W[i * D + r];
  }
  constexpr int RB = M / 16;
  const int ti = threadIdx.x / 16, tc = threadIdx.x % 16;
  const float scale = rsqrtf(static_cast<float>(M));  // 1 / sqrt(m)
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
      for (int b = 0; b < RB; ++b) wb[b] = sWT[r * M + tc + 16 * b];
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
          stx(out + (r0 + t) * M + tc + 16 * b, expf(acc[a][b] - sHalfSq[t]) * scale);
      }
    }
  }
}

template <int D, int M>
cudaError_t favor_simt(const void *x, const float *W, void *out, int64_t rows, cudaStream_t st) {
  const size_t smem = ((size_t)kRows * (D + 1) + (size_t)D * M + kRows) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(favor_features_kernel<D, M, float>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (rows + kRows - 1) / kRows;
  const int64_t cap = 4 * (int64_t)sm_count();  // a few CTAs per SM, each walking many row tiles
  const unsigned grid = static_cast<unsigned>(ntiles < cap ? ntiles : cap);
  favor_features_kernel<D, M, float><<<grid, kThreads, smem, st>>>(
      static_cast<const float *>(x), W, static_cast<float *>(out), rows);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ tensor-core features
using namespace tc;

constexpr int kFRows = 128;           // rows per tile (the M of the product)
constexpr int kFAtom = kFRows * 128;  // one [128 rows][64 bf16] 128B-swizzled atom: 16 KB
constexpr int kFNS = 4;               // stages of x tiles
constexpr int kFWarpTMA = 0, kFWarpMMA = 1, kFWarpEpi0 = 2;
constexpr int kFThreads = (kFWarpEpi0 + 4) * 32;

template <int D, int M>
struct FCfg {
  static constexpr int A = D / 64;             // 64-column atoms of an x tile / of W
  static constexpr int XTILE = A * kFAtom;     // bf16 [128][D]
  static constexpr int WATOM = M * 128;        // [M rows][64 bf16] atom of W
  static constexpr int WBYTES = A * WATOM;     // bf16 [M][D]
  static constexpr int OFF_WHI = kFNS * XTILE;
  static constexpr int OFF_WLO = OFF_WHI + WBYTES;
  static constexpr int OFF_BAR = OFF_WLO + WBYTES;
  static constexpr int SMEM = OFF_BAR + 256;
  static_assert(SMEM <= kMaxSmem, "shared memory budget");
  static_assert(OFF_WHI % 1024 == 0 && WATOM % 1024 == 0, "128B-swizzled operands need 1024 B");
};

struct FBars {
  uint64_t full[kFNS], empty[kFNS], acc_full[2], acc_empty[2], fin;
  uint32_t tmem_base;
  int abort;
};

// out[t][i] = exp(w_i . x_t - |x_t|^2 / 2) / sqrt(M) for tiles of 128 rows; CTA b takes tiles
// b, b + gridDim.x, ...
template <int D, int M>
__global__ void __launch_bounds__(kFThreads, 1)
    favor_tc_kernel(const __grid_constant__ CUtensorMap tmX, const float *__restrict__ W,
                    __nv_bfloat16 *__restrict__ out, int64_t rows, int *err) {
  const bool a32 = aligned32(out);  // output rows take full-sector stores
  using G = FCfg<D, M>;
  constexpr int KS = D / 16;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(err, kErrLayout);
    return;
  }
  FBars &bar = *reinterpret_cast<FBars *>(smem + G::OFF_BAR);
  volatile int *abort = &bar.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (rows + kFRows - 1) / kFRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFNS; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.acc_full[b], 1);
      mbar_init(&bar.acc_empty[b], 128);
    }
    mbar_init(&bar.fin, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  // W (fp32, [M][D]) -> W_hi = bf16(W), W_lo = bf16(W - W_hi): K-major B operands
  for (int e = threadIdx.x; e < M * D / 8; e += kFThreads) {
    const int row = e / (D / 8), c8 = (e % (D / 8)) * 8;
    float hi[8], lo[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float w = W[(int64_t)row * D + c8 + i];
      hi[i] = __bfloat162float(__float2bfloat16_rn(w));
      lo[i] = w - hi[i];
    }
    const uint32_t off = (c8 >> 6) * G::WATOM + sw128_offset(row, c8 & 63);
    *reinterpret_cast<uint4 *>(smem + G::OFF_WHI + off) = pack8(hi);
    *reinterpret_cast<uint4 *>(smem + G::OFF_WLO + off) = pack8(lo);
  }
  fence_proxy_async_smem();
  if (warp == kFWarpMMA) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kFWarpTMA && lane == 0) prefetch_tmap(&tmX);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp == kFWarpTMA) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int g = 0;
      for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++g) {
        const int s = g % kFNS;
        if (g >= kFNS && !mbar_wait(&bar.empty[s], ((g / kFNS) - 1) & 1, abort, err)) break;
        mbar_arrive_expect_tx(&bar.full[s], G::XTILE);
#pragma unroll
        for (int a = 0; a < G::A; ++a)
          tma_load_3d(smem + s * G::XTILE + a * kFAtom, &tmX, &bar.full[s], a * 64,
                      static_cast<int>(tile * kFRows), 0, pol);
      }
      for (int gg = (g > kFNS ? g - kFNS : 0); gg < g; ++gg)
        mbar_wait_drain(&bar.full[gg % kFNS], (gg / kFNS) & 1, err);
    }
  } else if (warp == kFWarpMMA) {
    if (lane == 0) {
      constexpr uint32_t I_F = make_idesc_bf16(128, M, false, false);
      const uint64_t dWhi = kmajor_base(smem_u32(smem + G::OFF_WHI));
      const uint64_t dWlo = kmajor_base(smem_u32(smem + G::OFF_WLO));
      int g = 0;
      for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++g) {
        const int s = g % kFNS, b = g & 1;
        if (!mbar_wait(&bar.full[s], (g / kFNS) & 1, abort, err)) break;
        if (g >= 2 && !mbar_wait(&bar.acc_empty[b], ((g >> 1) - 1) & 1, abort, err)) break;
        tc_fence_after();
        const uint64_t dX = kmajor_base(smem_u32(smem + s * G::XTILE));
        const uint32_t tA = tmem + b * M;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const uint64_t a = desc_add(dX, kmajor_off(ks, kFAtom));
          mma_bf16_ss(tA, a, desc_add(dWhi, kmajor_off(ks, G::WATOM)), I_F, ks > 0 ? 1u : 0u);
          mma_bf16_ss(tA, a, desc_add(dWlo, kmajor_off(ks, G::WATOM)), I_F, 1u);
        }
        mma_commit(&bar.acc_full[b]);
      }
      mma_commit(&bar.fin);
      mbar_wait_drain(&bar.fin, 0, err);
    }
  } else {
    // epilogue: thread = row (tensor-memory lane) of the tile
    const int sp = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const int r = 32 * sp + lane;
    const float scale = rsqrtf(static_cast<float>(M));
    WarpWaiter wait{abort, err, lane};
    int g = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++g) {
      const int s = g % kFNS, b = g & 1;
      if (!wait(&bar.acc_full[b], (g >> 1) & 1)) break;
      tc_fence_after();
      // |x_r|^2 / 2 from the x tile, still in shared memory (this group releases the stage)
      const uint8_t *xt = smem + s * G::XTILE;
      float sq = 0.f;
#pragma unroll
      for (int a = 0; a < G::A; ++a)
#pragma unroll
        for (int c8 = 0; c8 < 64; c8 += 8) {
          const uint4 u = *reinterpret_cast<const uint4 *>(xt + a * kFAtom + sw128_offset(r, c8));
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = bf16_lo(w[e]), x1 = bf16_hi(w[e]);
            sq = fmaf(x0, x0, fmaf(x1, x1, sq));
          }
        }
      const float half_sq = 0.5f * sq;
      mbar_arrive(&bar.empty[s]);
      const int64_t row = tile * kFRows + r;
      const bool live = row < rows;
      __nv_bfloat16 *orow = out + (live ? row : 0) * M;
      const uint32_t tA = tmem + lane_off + b * M;
#pragma unroll 1
      for (int c0 = 0; c0 < M; c0 += 32) {
        uint32_t v[32];
        tmem_ld16_async(tA + c0, v);
        tmem_ld16_async(tA + c0 + 16, v + 16);
        tmem_ld_wait();
        tmem_reg_fence<32>(v);
        if (live) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float f[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) f[e] = expf(__uint_as_float(v[16 * q + e]) - half_sq) * scale;
            st_global_32B(orow + c0 + 16 * q, pack8(f), pack8(f + 8), a32);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.acc_empty[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kFWarpMMA) tmem_dealloc(tmem, kTmemCols);
}

template <int D, int M>
cudaError_t favor_tc(const void *x, const float *W, void *out, int64_t rows, int *err,
                     cudaStream_t st) {
  using G = FCfg<D, M>;
  CUtensorMap tx;
  cudaError_t e = make_tmap_bf16(&tx, x, 1, rows, D, kFRows);
  if (e != cudaSuccess) return e;
  auto kern = favor_tc_kernel<D, M>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (rows + kFRows - 1) / kFRows;
  const int64_t sms = sm_count();
  const unsigned grid = static_cast<unsigned>(ntiles < sms ? ntiles : sms);
  kern<<<grid, kFThreads, G::SMEM, st>>>(tx, W, static_cast<__nv_bfloat16 *>(out), rows, err);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_favor_features(const void *x, const float *W, void *out, int64_t rows, int d,
                                  int m, int is_bf16, int *err, cudaStream_t st) {
  if (is_bf16) {
    if (d == 64)
      return m == 64 ? favor_tc<64, 64>(x, W, out, rows, err, st)
                     : favor_tc<64, 128>(x, W, out, rows, err, st);
    return m == 64 ? favor_tc<128, 64>(x, W, out, rows, err, st)
                   : favor_tc<128, 128>(x, W, out, rows, err, st);
  }
  if (d == 64)
    return m == 64 ? favor_simt<64, 64>(x, W, out, rows, st)
                   : favor_simt<64, 128>(x, W, out, rows, st);
  return m == 64 ? favor_simt<128, 64>(x, W, out, rows, st)
                 : favor_simt<128, 128>(x, W, out, rows, st);
}

}  // namespace linattn
