// Backward pass with bf16 I/O on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// The pages define the forward only ("Efficient Transformers: Linear Attention and Flash
// Attention", sections "Linear attention: reordering the matmuls, not shrinking them" and "The
// recurrent view: attention as an RNN"; "Linear Attention", section "Memory Efficiency", notes
// that training keeps the forward's tensors for backpropagation).  Its gradients follow by the
// chain rule.  Per head, with w_ij = phi(q_i).phi(k_j) (j <= i when causal), den_i = sum_j w_ij,
// out_i = sum_j w_ij v_j / den_i and g = dL/dout:
//
//   a_i = g_i / den_i,   b_i = -(a_i . out_i),   dW_ij = a_i . v_j + b_i
//   dphi(q_i) = sum_j dW_ij phi(k_j),   dphi(k_j) = sum_i dW_ij phi(q_i),   dv_j = sum_i w_ij a_i
//   dq = dphi(q) * phi'(q),  dk = dphi(k) * phi'(k),  phi'(x) = 1 above zero, exp(x) below.
//
// Precision.  With inputs of the usual scale phi(x) = 1 + psi(x) is 1 plus a small psi
// (psi = elu: x above zero, exp(x) - 1 below), so w_ij is d plus a small varying part and the
// gradients live in that part: rounded to bf16, phi itself would keep only a few bits of it.
// So every tensor-core operand here is a psi quantity (small, kept to bf16's relative
// precision) and the 1's are summed analytically in fp32 on the CUDA cores.  With
// sq_i = sum_r psi(q_i)_r and sk_j likewise,
//   w_ij = d + sq_i + sk_j + psi(q_i).psi(k_j)
//   dphi(q_i) = C_i 1 + [ sum_j dW_ij psi(k_j) ],   C_i  = sum_j dW_ij
//   dphi(k_j) = C'_j 1 + [ sum_i dW_ij psi(q_i) ],  C'_j = sum_i dW_ij
// where C_i and C'_j, sums of terms that nearly cancel, are taken in fp32 from the exact a.
// a itself enters the products as a bf16 pair (hi + lo), which keeps it to about 16 bits.
//
// The pass, per head; causal sums run over the chunks before (prefix) or after (suffix):
//   K1  per segment, the forward record [Psi | zeta | vs | sigma | kappa] of the keys:
//       Psi = sum psi(k_j) v_j^T, zeta = sum psi(k_j), vs = sum v_j, sigma = sum sk_j v_j,
//       kappa = sum sk_j; psi(k) (rounded to bf16) and its row sums sk to the workspace
//   K2  its exclusive prefix over segments (causal) or the head's total
//   B1  prefix walk: per segment, chunks in order, Psi in TMEM: den, out, a, b, dq; a (hi, lo),
//       b and (causal) psi(q) with its row sums sq to the workspace; the segment's reverse record [Phi | rho | as | tau | bs]:
//       Phi = sum psi(q_i) a_i^T, rho = sum psi(q_i) b_i, as = sum a_i, tau = sum sq_i a_i,
//       bs = sum b_i
//   K2  its exclusive suffix (causal) or the head's total
//   B3  suffix walk: per segment, chunks in reverse order, Phi in TMEM: dk, dv
// psi(q) and psi(k) are each computed once: B1 and B3 read psi(k) from K1, B3 psi(q) from B1
// (tile stores by TMA from the shared-memory tiles the kernel computed them in).
//
// Products of one 64-token chunk (tcgen05.mma kind::f16, bf16 operands, fp32 in TMEM):
//   B1  P' = psi(Q) psi(K)^T;  Psi += psi(K)^T V;  LV = L V (L: the lower triangle of ones);
//       O' = psi(Q) Psi + M V with M = mask(P' + sk);  dW = A V^T;  dQ' = A Psi^T + mask(dW + b)
//       psi(K);  Phi += psi(Q)^T A  (A = [a_hi; a_lo] along the contraction)
//   B3  P'^T = psi(K) psi(Q)^T;  dW^T = V A^T;  Phi += psi(Q)^T A;  dV' = psi(K) Phi +
//       mask(w^T) A_hi;  dK' = V Phi^T + mask(dW^T + b) psi(Q)
// and the fp32 rest, e.g. den_i = N_i (d + sq_i) + kappa + psi(q_i).zeta + rowsum(M)_i and
// out_i = ((d + sq_i)(vs + LV_i) + sigma + O'_i) / den_i, N_i the keys row i sees.
//
// Each CTA runs 8 warps through a chunk's phases in step (warps w and w + 4 share TMEM
// sub-partition w & 3 and split the columns), thread 0 issuing the TMA loads (one chunk ahead,
// two stages) and lane 0 of warps 0-2 the MMAs of each phase.  Two CTAs share an SM at d = 64, so one CTA's products run while
// the other drains its accumulators.  Every wait is bounded (2 s); a CTA whose wait gave up lets
// its copies and products land and exits.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace linattn {
namespace {

using namespace tc;

constexpr int C = kTcChunk;     // tokens per chunk (64)
constexpr int kAtom = C * 128;  // one [64 rows][64 bf16] 128B-swizzled atom: 8 KB
constexpr int kThreads = 256;   // 8 warps, two per TMEM sub-partition
// The walks' products of one phase go to different accumulators and are issued by lane 0 of
// warps 0, 1 and 2 in parallel: one thread issues a tcgen05.mma about every 55 cycles, slower
// than the tensor pipe runs these small products.
constexpr int kIssuers = 3;

// A state record: [M (D x D, row-major) | three D-vectors | a scalar, three zeros].
template <int D>
__host__ __device__ constexpr int64_t rec_floats() {
  return (int64_t)D * D + 3 * D + 4;
}

// A chunk's vectors: [three D-vectors | a scalar, three zeros] (the vector part of a record).
template <int D>
__host__ __device__ constexpr int64_t vec_floats() {
  return 3 * D + 4;
}

struct BwdShared {
  uint64_t full[2];      // stage loaded (TMA transaction bytes)
  uint64_t mma;          // the products issued since the last wait are done
  uint64_t fin;          // drain at exit
  float vec[3][128];     // the record's three vectors (current state)
  float sq[64], sk[64];  // row sums of psi(Q), psi(K) of the chunk
  float part[2][64];     // per column half, per row: partial sums
  float gd[2][64];
  float cd[2][64];
  float bv[64];          // b of the chunk's rows
  float acc[3][128];     // column sums being gathered (atomically) for a chunk or an item
  float racc[3][128];    // the prefix walk: the item's reverse-record vectors
  float scal;            // the record's scalar
  uint32_t tmem_base;
  int abort;
};
// pairs of columns are read as float2
static_assert(offsetof(BwdShared, vec) % 8 == 0 && offsetof(BwdShared, sq) % 8 == 0 &&
                  offsetof(BwdShared, sk) % 8 == 0 && offsetof(BwdShared, bv) % 8 == 0,
              "float2 reads of the shared vectors");

template <int D>
struct BCfg {
  static constexpr int AT = D / 64;        // 64-column atoms per [64][D] tile
  static constexpr int TILE = AT * kAtom;  // one bf16 [64][D] tile
  static constexpr int S_ATOM = D * 128;   // [D rows][64 columns] block of a D x D operand
  static constexpr int STATE = AT * S_ATOM;
  // prefix walk: stages of Q, G, K, V; the Psi operand; A hi, A lo; the M / dW operand; L
  static constexpr int P_STAGE = 4 * TILE;
  static constexpr int P_ST = 2 * P_STAGE;
  static constexpr int P_A = P_ST + STATE;
  static constexpr int P_AL = P_A + TILE;
  static constexpr int P_W = P_AL + TILE;
  static constexpr int P_L = P_W + kAtom;
  static constexpr int P_SH = P_L + kAtom;
  // suffix walk: stages of Q, A hi, A lo, K, V; the Phi operand; two [64][64] operands
  static constexpr int S_STAGE = 5 * TILE;
  static constexpr int S_ST = 2 * S_STAGE;
  static constexpr int S_W0 = S_ST + STATE;
  static constexpr int S_W1 = S_W0 + kAtom;
  static constexpr int S_SH = S_W1 + kAtom;
  // aggregate: stages of K, V; D = 64: the E atom and the ones atom of the extended product
  static constexpr bool G_XT = D == 64;
  static constexpr int G_STAGE = 2 * TILE;
  static constexpr int G_E = 2 * G_STAGE;
  static constexpr int G_ONES = G_E + kAtom;
  static constexpr int G_SH = G_XT ? G_ONES + kAtom : 2 * G_STAGE;
  static constexpr uint32_t G_TCOLS = G_XT ? 128 : D;  // the aggregate's TMEM
  static constexpr int SLACK = 1024;  // alignment of the dynamic shared memory base
  static constexpr int P_SMEM = P_SH + (int)sizeof(BwdShared) + SLACK;
  static constexpr int S_SMEM = S_SH + (int)sizeof(BwdShared) + SLACK;
  static constexpr int G_SMEM = G_SH + (int)sizeof(BwdShared) + SLACK;
  static constexpr uint32_t TCOLS = D == 64 ? 256 : 512;  // the walks' TMEM
  static constexpr int CTAS = D == 64 ? 2 : 1;            // walk CTAs per SM
  static constexpr int G_CTAS = D == 64 ? 4 : 2;          // aggregate CTAs per SM
  static constexpr int kSmPerSm = 228 * 1024;             // an SM's shared memory
  static_assert(P_SMEM <= kMaxSmem && S_SMEM <= kMaxSmem, "shared memory");
  static_assert(CTAS * (P_SMEM + 1024) <= kSmPerSm && CTAS * (S_SMEM + 1024) <= kSmPerSm,
                "CTAS walk CTAs fit on an SM");
  static_assert(D == 128 || (3 * (P_SMEM + 1024) > kSmPerSm && 3 * (S_SMEM + 1024) > kSmPerSm),
                "at most two walk CTAs per SM share its TMEM");
  static_assert(G_CTAS * (G_SMEM + 1024) <= kSmPerSm && G_CTAS * G_TCOLS <= 512,
                "G_CTAS aggregate CTAs fit on an SM");
  static_assert(P_ST % 1024 == 0 && P_A % 1024 == 0 && P_AL % 1024 == 0 && P_W % 1024 == 0 &&
                    P_L % 1024 == 0 && S_ST % 1024 == 0 && S_W0 % 1024 == 0 &&
                    S_W1 % 1024 == 0,
                "128B-swizzled operands need 1024-byte alignment");
};

// ---------------------------------------------------------------- shared helpers
// 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tmem_row32(uint32_t taddr, float *f) {
  uint32_t r[32];
  tmem_ld16_async(taddr, r);
  tmem_ld16_async(taddr + 16, r + 16);
  tmem_ld_wait();
  tmem_reg_fence<32>(r);
#pragma unroll
  for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(r[e]);
}

__device__ __forceinline__ void unpack8(uint4 u, float *f) {
  f[0] = bf16_lo(u.x);
  f[1] = bf16_hi(u.x);
  f[2] = bf16_lo(u.y);
  f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z);
  f[5] = bf16_hi(u.z);
  f[6] = bf16_lo(u.w);
  f[7] = bf16_hi(u.w);
}
// Byte offset of (row, col) in a token tile of 64-column atoms (col a multiple of 8 for
// 16-byte accesses).
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
  return (col >> 6) * kAtom + sw128_offset(row, col & 63);
}
__device__ __forceinline__ void tile_row8(const uint8_t *tile, int row, int col, float *f) {
  unpack8(*reinterpret_cast<const uint4 *>(tile + tile_off(row, col)), f);
}
// phi'(x) from psi(x) = phi(x) - 1: 1 above zero, exp(x) = 1 + psi(x) at or below.
__device__ __forceinline__ float dphi_from_psi(float p) { return p > 0.f ? 1.f : 1.f + p; }

// psi in place on the 64 rows of a [64][D] token tile, in fp32 and rounded to bf16; rows at or
// after `keep` zeroed.  rowsum (if not null) receives each row's sum of the rounded values.
// Thread t takes rows t / 8 and 32 + t / 8 (16-byte chunk t % 8 of each atom), so the 8
// threads of a row are 8 consecutive lanes.
template <int D>
__device__ __forceinline__ void psi_tile(uint8_t *tile, int keep, float *rowsum) {
  uint4 *p = reinterpret_cast<uint4 *>(tile);
  float s[2] = {0.f, 0.f};
#pragma unroll
  for (int m = 0; m < 2 * (D / 64); ++m) {
    const int i = threadIdx.x + kThreads * m;
    const int row = (i % (kAtom / 16)) >> 3;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (row < keep) {
      float f[8];
      unpack8(p[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = f[e] > 0.f ? f[e] : __expf(f[e]) - 1.f;
      x = pack8(f);
      unpack8(x, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) s[m & 1] += f[e];
    }
    p[i] = x;
  }
  if (rowsum != nullptr) {
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      s[0] += __shfl_xor_sync(0xffffffffu, s[0], o);
      s[1] += __shfl_xor_sync(0xffffffffu, s[1], o);
    }
    if ((threadIdx.x & 7) == 0) {
      rowsum[threadIdx.x >> 3] = s[0];
      rowsum[32 + (threadIdx.x >> 3)] = s[1];
    }
  }
}

// Rows at or after `keep` of a [64][D] token tile zeroed.
template <int D>
__device__ __forceinline__ void zero_rows(uint8_t *tile, int keep) {
  if (keep >= C) return;
  uint4 *p = reinterpret_cast<uint4 *>(tile);
#pragma unroll
  for (int m = 0; m < 2 * (D / 64); ++m) {
    const int i = threadIdx.x + kThreads * m;
    if (((i % (kAtom / 16)) >> 3) >= keep) p[i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Per-thread roles: warps w and w + 4 read TMEM sub-partition w & 3; the first four take the
// low half of every accumulator's columns, the others the high half.
struct Lanes {
  int warp, lane, sp, hf;
  uint32_t lane_off;  // TMEM lane field of this warp's sub-partition
  bool v64;           // lane holds a row of an M = 64 accumulator (lanes 0..15)
  int r64;            // that row (token within the chunk)
  int rS;             // row of a D x D accumulator
  bool vS;
  int qa, qb;         // rows of an M = 64 accumulator this thread gets from tmem_quad32
  int cq;             // its first column within each group of 8 (2 (lane % 4))
  template <int D>
  __device__ __forceinline__ static Lanes make() {
    Lanes L;
    L.warp = threadIdx.x >> 5;
    L.lane = threadIdx.x & 31;
    L.sp = L.warp & 3;
    L.hf = L.warp >> 2;
    L.lane_off = static_cast<uint32_t>(32 * L.sp) << 16;
    L.v64 = L.lane < 16;
    L.r64 = 16 * L.sp + L.lane;
    L.rS = D == 128 ? 32 * L.sp + L.lane : L.r64;
    L.vS = D == 128 || L.v64;
    L.qa = 16 * L.sp + (L.lane >> 2);
    L.qb = L.qa + 8;
    L.cq = 2 * (L.lane & 3);
    return L;
  }
};

// A record from global memory: M into the bf16 operand (and, when to_tmem, TMEM at tM), the
// three vectors into sh.vec, the scalar into sh.scal.  Rows rS, this half's columns of M.
template <int D>
__device__ __forceinline__ void load_record(const float *src, uint8_t *sOp, uint32_t tM,
                                            bool to_tmem, const Lanes &L, BwdShared &sh) {
  constexpr int HD = D / 2;
#pragma unroll 1
  for (int c0 = L.hf * HD; c0 < L.hf * HD + HD; c0 += 32) {
    uint32_t r[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (L.vS) f = *reinterpret_cast<const float4 *>(src + (int64_t)L.rS * D + c0 + 4 * q);
      r[4 * q + 0] = __float_as_uint(f.x);
      r[4 * q + 1] = __float_as_uint(f.y);
      r[4 * q + 2] = __float_as_uint(f.z);
      r[4 * q + 3] = __float_as_uint(f.w);
    }
    if (to_tmem) {
      tmem_st16(tM + c0, *reinterpret_cast<const uint32_t(*)[16]>(r));
      tmem_st16(tM + c0 + 16, *reinterpret_cast<const uint32_t(*)[16]>(r + 16));
    }
    if (L.vS) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * q + e]);
        *reinterpret_cast<uint4 *>(sOp + (c0 >> 6) * (D * 128) +
                                   sw128_offset(L.rS, (c0 & 63) + 8 * q)) = pack8(f);
      }
    }
  }
  if (to_tmem) tmem_st_wait();
  if (threadIdx.x < D) {
#pragma unroll
    for (int k = 0; k < 3; ++k) sh.vec[k][threadIdx.x] = src[(int64_t)D * D + k * D + threadIdx.x];
  }
  if (threadIdx.x == 0) sh.scal = src[(int64_t)D * D + 3 * D];
}

// TMEM state (rows rS, this half's columns) -> its bf16 operand (warp-collective loads).
// D = 64: the state is an M = 64 accumulator, read by all 32 lanes (tmem_quad32).
template <int D>
__device__ __forceinline__ void state_to_operand(uint32_t tM, uint8_t *sOp, const Lanes &L) {
  constexpr int HD = D / 2;
  if constexpr (D == 64) {
    float f[16];
    tmem_quad32(tM + L.hf * HD, f);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = L.hf * HD + 8 * q + L.cq;
      *reinterpret_cast<uint32_t *>(sOp + sw128_offset(L.qa, c)) =
          pack_bf16x2(f[4 * q], f[4 * q + 1]);
      *reinterpret_cast<uint32_t *>(sOp + sw128_offset(L.qb, c)) =
          pack_bf16x2(f[4 * q + 2], f[4 * q + 3]);
    }
  } else {
#pragma unroll 1
    for (int c0 = L.hf * HD; c0 < L.hf * HD + HD; c0 += 32) {
      float f[32];
      tmem_row32(tM + c0, f);
      if (L.vS) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(sOp + (c0 >> 6) * (D * 128) +
                                     sw128_offset(L.rS, (c0 & 63) + 8 * q)) = pack8(f + 8 * q);
      }
    }
  }
}

// TMEM state (rows rS, this half's columns) -> fp32 row-major D x D at dst.
template <int D>
__device__ __forceinline__ void state_to_global(uint32_t tM, float *dst, const Lanes &L) {
  constexpr int HD = D / 2;
#pragma unroll 1
  for (int c0 = L.hf * HD; c0 < L.hf * HD + HD; c0 += 32) {
    float f[32];
    tmem_row32(tM + c0, f);
    if (L.vS) {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4 *>(dst + (int64_t)L.rS * D + c0 + e) =
            make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
    }
  }
}

// Adds to acc[0..2][col] the column sums over the chunk's 64 rows of three per-row terms:
// terms(i, c, t) adds row i's terms for columns [c, c + 8) into t[0..2][0..7].  Warp w owns
// D / 64 groups of 8 columns; the lanes of a group split its rows and then reduce-scatter their
// 8 partial sums (each halving step sends half of them to the partner lane), so that every
// column's total ends in one lane, which adds it to acc: no two lanes write the same column.
template <int D, typename F>
__device__ __forceinline__ void column_sums3(float (*acc)[128], F &&terms) {
  constexpr int CPW = D / 64;    // column groups per warp
  constexpr int LPG = 32 / CPW;  // lanes per column group
  constexpr int RPL = C / LPG;   // rows per lane
  const int lane = threadIdx.x & 31;
  const int cg = (threadIdx.x >> 5) * CPW + lane / LPG;
  float t[3][8];
#pragma unroll
  for (int k = 0; k < 3; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) t[k][e] = 0.f;
#pragma unroll
  for (int m = 0; m < RPL; ++m) terms(lane % LPG + m * LPG, 8 * cg, t);
  int col = 0;
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const int h = 4 >> r, o = LPG >> (r + 1);
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int k = 0; k < 3; ++k)
#pragma unroll
      for (int j = 0; j < h; ++j) {
        const float keep = up ? t[k][j + h] : t[k][j];
        const float send = up ? t[k][j] : t[k][j + h];
        t[k][j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    col += up ? h : 0;
  }
#pragma unroll
  for (int o = LPG / 16; o >= 1; o >>= 1)
#pragma unroll
    for (int k = 0; k < 3; ++k) t[k][0] += __shfl_xor_sync(0xffffffffu, t[k][0], o);
  if ((lane & (LPG / 8 - 1)) == 0) {
#pragma unroll
    for (int k = 0; k < 3; ++k) acc[k][8 * cg + col] += t[k][0];
  }
}
// Sum of x(i) over i in [0, 64), in every lane of the calling warp.
template <typename F>
__device__ __forceinline__ float warp_sum64(F &&x) {
  const int l = threadIdx.x & 31;
  float s = x(l) + x(l + 32);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}
// The three vectors of acc into dst, and acc cleared (threads t < D, column t).
template <int D>
__device__ __forceinline__ void drain_acc(float (*acc)[128], float *dst, int64_t stride) {
  if (threadIdx.x < D) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      dst[k * stride + threadIdx.x] = acc[k][threadIdx.x];
      acc[k][threadIdx.x] = 0.f;
    }
  }
}

// Common set-up of the three kernels: barriers, TMEM, and the CTA-wide agreement on whether
// every wait so far has succeeded.
struct Sync {
  BwdShared &sh;
  WarpWaiter wait;
  uint32_t mph = 0;  // commits to sh.mma waited for
  __device__ __forceinline__ Sync(BwdShared &s, int *err, int lane)
      : sh(s), wait{&s.abort, err, lane} {}
  // CTA barrier; false (for every thread) once any thread's wait has given up
  __device__ __forceinline__ bool barrier() {
    tc_fence_before();
    const int bad = __syncthreads_or(wait.ok ? 0 : 1);
    tc_fence_after();
    if (bad) wait.ok = false;
    return bad == 0;
  }
  __device__ __forceinline__ void wait_mma() {
    wait(&sh.mma, mph & 1);
    ++mph;
  }
};

// issuers: the threads (lane 0 of the first warps) that issue MMAs; sh.mma and sh.fin take
// one arrival from each.
__device__ __forceinline__ void init_barriers(BwdShared &sh, int issuers) {
  for (int i = threadIdx.x; i < 3 * 128; i += kThreads) {
    sh.acc[i / 128][i % 128] = 0.f;
    sh.racc[i / 128][i % 128] = 0.f;
  }
  if (threadIdx.x == 0) {
    mbar_init(&sh.full[0], 1);
    mbar_init(&sh.full[1], 1);
    mbar_init(&sh.mma, issuers);
    mbar_init(&sh.fin, issuers);
    sh.abort = 0;
    fence_barrier_init();
  }
}

// An issuer's end of an MMA phase: its products of the phase committed to `bar`, or (none
// issued) an arrival at once.
__device__ __forceinline__ void phase_done(uint64_t *bar, bool issued_any) {
  if (issued_any)
    mma_commit(bar);
  else
    mbar_arrive(bar);
}

// Lets every copy and product a CTA issued land (thread 0: `landed` of `issued` loads had
// been waited for; each of the `issuers` MMA-issuing threads: my_mma, whether it issued any),
// then releases its TMEM.
__device__ __forceinline__ void finish(BwdShared &sh, int landed, int issued, uint32_t tmem,
                                       uint32_t cols, int *err, int issuers, bool my_mma) {
  if (threadIdx.x == 0)
    for (int l = landed; l < issued; ++l) mbar_wait_drain(&sh.full[l & 1], (l >> 1) & 1, err);
  if ((threadIdx.x & 31) == 0 && (threadIdx.x >> 5) < issuers) phase_done(&sh.fin, my_mma);
  if (threadIdx.x == 0) mbar_wait_drain(&sh.fin, 0, err);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if ((threadIdx.x >> 5) == 0) tmem_dealloc(tmem, cols);
}

__device__ __forceinline__ uint64_t kdesc(uint32_t base, int ks, uint32_t atom) {
  return desc_add(kmajor_base(base), kmajor_off(ks, atom));
}
__device__ __forceinline__ uint64_t mdesc(uint32_t base, int ks, uint32_t atom) {
  return desc_add(mnmajor_base(base, atom), mnmajor_off(ks));
}

// ---------------------------------------------------------------- K1: forward records
// k, v: [heads][n][D] via tmK, tmV.  Writes each item's record [Psi | zeta | vs | sigma |
// kappa] to rec + (head * nseg + seg) * rec_floats<D>(), the item's vectors before each of its
// chunks to chunk_vec, and psi(k) (rounded to bf16, via the store map tmPK) with its row sums
// (skg, [heads][n]) for the walks.
// D = 64: the whole record comes from one product per K-step, A = [psi(K) | E] (M = 128, E's row
// j = [1, hi(sk_j), lo(sk_j), 0 ...], sk_j split into two bf16) times B = [V | 1] (N = 80):
// accumulator rows 0..63 hold [Psi | zeta], row 64 [vs | count], rows 65 and 66 the two halves
// of [sigma | kappa].  D = 128 (M would pass 128): Psi from the product, the vectors by column
// sums on the CUDA cores.
template <int D>
__global__ void __launch_bounds__(kThreads, BCfg<D>::G_CTAS)
    bwd_aggregate_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmPK, float *__restrict__ skg,
                         float *__restrict__ rec,
                         float *__restrict__ chunk_vec, int64_t n, int64_t seg_len, int64_t nseg,
                         int64_t nitems, int *err) {
  using G = BCfg<D>;
  constexpr int AT = G::AT;
  constexpr int KSC = C / 16;
  constexpr int OK = 0, OV = G::TILE;
  constexpr uint32_t LOAD = 2 * G::TILE;
  constexpr uint32_t I_S = make_idesc_bf16(D, D, true, true);
  constexpr bool XT = G::G_XT;
  constexpr uint32_t I_X = make_idesc_bf16(128, D + 16, true, true);  // the extended product
  const int64_t nck = (n + C - 1) / C;  // chunks per head
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  BwdShared &sh = *reinterpret_cast<BwdShared *>(sm + G::G_SH);
  const Lanes L = Lanes::make<D>();
  const int64_t it0 = blockIdx.x, istep = gridDim.x;

  uint8_t *sE = sm + G::G_E, *sOnes = sm + G::G_ONES;
  init_barriers(sh, 1);
  if (XT) {
    // E starts at zero (each chunk rewrites the first 16 bytes of its rows); the ones atom's
    // column 0 is 1 in every row (row r's column 0 sits in 16-byte chunk r & 7)
    uint32_t *e = reinterpret_cast<uint32_t *>(sE), *o = reinterpret_cast<uint32_t *>(sOnes);
    for (int i = threadIdx.x; i < kAtom / 4; i += kThreads) {
      const int row = i >> 5, word = i & 31;
      e[i] = 0u;
      o[i] = (word == 4 * (row & 7)) ? 0x00003F80u : 0u;
    }
    fence_proxy_async_smem();
  }
  if (L.warp == 0) {
    tmem_alloc(&sh.tmem_base, G::G_TCOLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint64_t pol = policy_evict_first();
  Sync S(sh, err, L.lane);

  int issued = 0, landed = 0;
  bool my_mma = false;  // thread 0 issued products
  auto issue = [&](const Item &I, int c) {
    uint64_t *fb = &sh.full[issued & 1];
    uint8_t *st = sm + (issued & 1) * G::G_STAGE;
    mbar_arrive_expect_tx(fb, LOAD);
    const int y = static_cast<int>(I.t_begin + (int64_t)c * C), z = static_cast<int>(I.head);
#pragma unroll
    for (int a = 0; a < AT; ++a) {
      tma_load_3d(st + OK + a * kAtom, &tmK, fb, 64 * a, y, z, pol);
      tma_load_3d(st + OV + a * kAtom, &tmV, fb, 64 * a, y, z, pol);
    }
    ++issued;
  };
  if (threadIdx.x == 0) issue(item_at<C>(it0, n, seg_len, nseg), 0);

  int g = 0;
  for (int64_t it = it0; it < nitems && S.wait.ok; it += istep) {
    const Item I = item_at<C>(it, n, seg_len, nseg);
    float kap = 0.f;  // thread 0: kappa of the item (its vectors gather in sh.acc)
    for (int c = 0; c < I.nchunks; ++c, ++g) {
      uint8_t *st = sm + (g & 1) * G::G_STAGE;
      const int64_t t0 = I.t_begin + (int64_t)c * C;
      const int valid = I.t_end - t0 < C ? static_cast<int>(I.t_end - t0) : C;
      if (S.wait(&sh.full[g & 1], (g >> 1) & 1)) {
        if (threadIdx.x == 0) landed = g + 1;
        psi_tile<D>(st + OK, valid, sh.sk);
        if (XT && (threadIdx.x & 7) == 0) {
          // E's rows for the two rows whose sums this thread made (psi_tile's mapping); rows
          // past the item's end are zero
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int r = 32 * h + (threadIdx.x >> 3);
            const float skr = sh.sk[r];
            const uint32_t w0 = pack_bf16x2(r < valid ? 1.f : 0.f, skr);
            *reinterpret_cast<uint4 *>(sE + sw128_offset(r, 0)) =
                make_uint4(w0, pack_bf16x2(skr - bf16_hi(w0), 0.f), 0u, 0u);
          }
        }
      }
      fence_proxy_async_smem();
      if (!S.barrier()) break;
      // psi(k) and its row sums to the workspace (rows past n are not stored)
      if (threadIdx.x < valid) skg[I.head * n + t0 + threadIdx.x] = sh.sk[threadIdx.x];
      if (threadIdx.x == 0) {
#pragma unroll
        for (int a = 0; a < AT; ++a)
          tma_store_3d(&tmPK, st + OK + a * kAtom, 64 * a, static_cast<int>(t0),
                       static_cast<int>(I.head), pol);
        tma_store_commit();
        // the other stage's tile has been read by its store before the next load lands there
        tma_store_wait_read<1>();
        if (c + 1 < I.nchunks)
          issue(I, c + 1);
        else if (it + istep < nitems)
          issue(item_at<C>(it + istep, n, seg_len, nseg), 0);
        const uint32_t k0 = smem_u32(st + OK), v0 = smem_u32(st + OV);
        if (XT) {
          // [Psi | zeta; vs | count; sigma | kappa] += [psi(K) | E]^T [V | 1]: the second
          // 64-wide block of each operand (E, ones) is one atom shared by both stages, reached
          // through the descriptor's block stride
          const uint64_t dA = mnmajor_base(k0, smem_u32(sE) - k0);
          const uint64_t dB = mnmajor_base(v0, smem_u32(sOnes) - v0);
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tmem, desc_add(dA, mnmajor_off(ks)), desc_add(dB, mnmajor_off(ks)), I_X,
                        (c > 0 || ks > 0));
        } else {
          // Psi += psi(K)^T V
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tmem, mdesc(k0, ks, kAtom), mdesc(v0, ks, kAtom), I_S, (c > 0 || ks > 0));
        }
        mma_commit(&sh.mma);
        my_mma = true;
      }
      // D = 128: zeta, vs, sigma of the chunk's keys (rows past the item's end: psi(K) zero, V
      // skipped)
      if (!XT) column_sums3<D>(sh.acc, [&](int i, int c, float (*t)[8]) {
        float kr[8], vr[8];
        tile_row8(st + OK, i, c, kr);
        tile_row8(st + OV, i, c, vr);
        const float w = i < valid ? 1.f : 0.f, ski = sh.sk[i];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          t[0][e] += kr[e];
          t[1][e] = fmaf(w, vr[e], t[1][e]);
          t[2][e] = fmaf(w * ski, vr[e], t[2][e]);
        }
      });
      if (!XT && L.warp == 0) {
        const float ks = warp_sum64([&](int i) { return sh.sk[i]; });
        if (threadIdx.x == 0) kap += ks;
      }
      S.wait_mma();
      if (XT && S.wait.ok) {
        // the item's vectors so far, from the accumulator: zeta (column D of rows 0..63:
        // warps 0, 1) into sh.racc[0]; rows 64..66 (warp 2, lanes 0..2), columns 0..D, into
        // sh.acc[0..2]
        tc_fence_after();
        if (L.warp < 2) {
          sh.racc[0][32 * L.warp + L.lane] = __uint_as_float(tmem_ld1(tmem + L.lane_off + D));
        } else if (L.warp == 2) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float f[32];
            tmem_row32(tmem + L.lane_off + c0, f);
            if (L.lane < 3) {
#pragma unroll
              for (int e = 0; e < 32; ++e) sh.acc[L.lane][c0 + e] = f[e];
            }
          }
          const float last = __uint_as_float(tmem_ld1(tmem + L.lane_off + D));
          if (L.lane < 3) sh.acc[L.lane][D] = last;
        }
      }
      if (!S.barrier()) break;
      // the item's vectors before its next chunk (exclusive within the item), for the walk
      if (c + 1 < I.nchunks) {
        float *cv = chunk_vec + (I.head * nck + I.t_begin / C + c + 1) * vec_floats<D>();
        if (XT) {
          if (threadIdx.x < D) {
            cv[threadIdx.x] = sh.racc[0][threadIdx.x];
            cv[D + threadIdx.x] = sh.acc[0][threadIdx.x];
            cv[2 * D + threadIdx.x] = sh.acc[1][threadIdx.x] + sh.acc[2][threadIdx.x];
          }
          if (threadIdx.x == 0) cv[3 * D] = sh.acc[1][D] + sh.acc[2][D];
        } else {
          if (threadIdx.x < D) {
#pragma unroll
            for (int k = 0; k < 3; ++k) cv[k * D + threadIdx.x] = sh.acc[k][threadIdx.x];
          }
          if (threadIdx.x == 0) cv[3 * D] = kap;
        }
      }
    }
    if (!S.wait.ok) break;
    float *dst = rec + (I.head * nseg + I.seg) * rec_floats<D>();
    if (XT) {
      // Psi: rows 0..63 are lanes 0..63 (warps 0, 1; 4, 5 take the other half of the columns);
      // the vectors from the last chunk's read-out
      if (L.sp < 2) {
        float f[32];
        tmem_row32(tmem + L.lane_off + L.hf * 32, f);
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4 *>(dst + (int64_t)(32 * L.sp + L.lane) * D + L.hf * 32 + e) =
              make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
      }
      if (threadIdx.x < D) {
        dst[(int64_t)D * D + threadIdx.x] = sh.racc[0][threadIdx.x];
        dst[(int64_t)D * D + D + threadIdx.x] = sh.acc[0][threadIdx.x];
        dst[(int64_t)D * D + 2 * D + threadIdx.x] = sh.acc[1][threadIdx.x] + sh.acc[2][threadIdx.x];
      }
      if (threadIdx.x == 0) kap = sh.acc[1][D] + sh.acc[2][D];
    } else {
      state_to_global<D>(tmem + L.lane_off, dst, L);
      drain_acc<D>(sh.acc, dst + (int64_t)D * D, D);
    }
    if (threadIdx.x == 0) {
      dst[(int64_t)D * D + 3 * D] = kap;
      dst[(int64_t)D * D + 3 * D + 1] = 0.f;
      dst[(int64_t)D * D + 3 * D + 2] = 0.f;
      dst[(int64_t)D * D + 3 * D + 3] = 0.f;
    }
    if (!S.barrier()) break;
  }
  if (threadIdx.x == 0) tma_store_wait_all<0>();  // the stores are done with shared memory
  finish(sh, landed, issued, tmem, G::G_TCOLS, err, 1, my_mma);
}

// ---------------------------------------------------------------- B1: the prefix walk
// q, dout: [heads][n][D] via tmQ, tmG; psi(k), v via tmK, tmV and skg (psi(k)'s row sums,
// [heads][n]) (causal only).  Causal: stores psi(q) via tmPQ with its row sums to sqg, for the
// suffix walk.  dq, and (causal) a as a bf16 pair, are stored through tile stores (tmDQ,
// tmAH, tmAL: [heads][n][D]).  start: each item's forward record (causal: exclusive prefix at start + head * start_hs + seg * start_ss;
// non-causal: the head's total).  Writes dq, a as a bf16 pair (a_hi, a_lo: [heads][n][D]),
// b ([heads][n]) and each item's reverse record to r_rec + (head * nseg + seg) * rec_floats.
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, BCfg<D>::CTAS)
    bwd_prefix_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmG,
                      const __grid_constant__ CUtensorMap tmPQ, float *__restrict__ sqg,
                      const float *__restrict__ skg, const __grid_constant__ CUtensorMap tmDQ,
                      const __grid_constant__ CUtensorMap tmAH,
                      const __grid_constant__ CUtensorMap tmAL,
                      float *__restrict__ b_out, const float *__restrict__ start,
                      int64_t start_hs, int64_t start_ss, const float *__restrict__ s_vec,
                      float *__restrict__ r_rec, float *__restrict__ r_vec, int64_t n,
                      int64_t seg_len, int64_t nseg, int64_t nitems, int *err) {
  using G = BCfg<D>;
  constexpr int AT = G::AT;
  constexpr int KSD = D / 16;  // K-steps over D
  constexpr int KSC = C / 16;  // K-steps over the chunk's tokens
  constexpr int HD = D / 2;    // columns per half of a D-wide accumulator
  constexpr int OQ = 0, OG = G::TILE, OK = 2 * G::TILE, OV = 3 * G::TILE;
  constexpr uint32_t LOAD = (CAUSAL ? 4 : 2) * G::TILE;
  constexpr uint32_t SA = G::S_ATOM;
  constexpr uint32_t I_P = make_idesc_bf16(64, 64, false, false);  // P', dW
  constexpr uint32_t I_S = make_idesc_bf16(D, D, true, true);      // Psi, Phi updates
  constexpr uint32_t I_O = make_idesc_bf16(64, D, false, true);    // psi(Q) Psi, M V, L V, W psi(K)
  constexpr uint32_t I_T = make_idesc_bf16(64, D, false, false);   // A Psi^T
  constexpr float kD = static_cast<float>(D);
  constexpr int64_t VF = vec_floats<D>();
  const int64_t nck = (n + C - 1) / C;  // chunks per head

  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  BwdShared &sh = *reinterpret_cast<BwdShared *>(sm + G::P_SH);
  uint8_t *sST = sm + G::P_ST;  // bf16 Psi (rows: features; 64-column blocks of values)
  uint8_t *sA = sm + G::P_A, *sAL = sm + G::P_AL, *sW = sm + G::P_W, *sL = sm + G::P_L;
  const Lanes L = Lanes::make<D>();
  const int64_t it0 = blockIdx.x, istep = gridDim.x;

  init_barriers(sh, kIssuers);
  // L: [64][64] lower triangle of ones (j <= i), the K-major operand of the prefix sums of V
  for (int i = threadIdx.x; i < kAtom / 16; i += kThreads) {
    const int row = i >> 3, c8 = 8 * (i & 7);
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[e] = (c8 + 2 * e <= row ? 0x3F80u : 0u) | (c8 + 2 * e + 1 <= row ? 0x3F800000u : 0u);
    *reinterpret_cast<uint4 *>(sL + sw128_offset(row, c8)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  fence_proxy_async_smem();
  if (L.warp == 0) {
    tmem_alloc(&sh.tmem_base, G::TCOLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmG);
    if (CAUSAL) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint32_t tX = tmem, tY = tmem + D, tR = tmem + 2 * D, tS = tmem + 3 * D;
  const uint32_t myX = tX + L.lane_off, myY = tY + L.lane_off, myR = tR + L.lane_off,
                 myS = tS + L.lane_off;
  const uint64_t pol = policy_evict_first();
  Sync S(sh, err, L.lane);

  int issued = 0, landed = 0;
  bool my_mma = false;  // this thread (an issuer) issued products
  auto issue = [&](const Item &I, int c) {
    uint64_t *fb = &sh.full[issued & 1];
    uint8_t *st = sm + (issued & 1) * G::P_STAGE;
    mbar_arrive_expect_tx(fb, LOAD);
    const int y = static_cast<int>(I.t_begin + (int64_t)c * C), z = static_cast<int>(I.head);
#pragma unroll
    for (int a = 0; a < AT; ++a) {
      tma_load_3d(st + OQ + a * kAtom, &tmQ, fb, 64 * a, y, z, pol);
      tma_load_3d(st + OG + a * kAtom, &tmG, fb, 64 * a, y, z, pol);
      if (CAUSAL) {
        tma_load_3d(st + OK + a * kAtom, &tmK, fb, 64 * a, y, z, pol);
        tma_load_3d(st + OV + a * kAtom, &tmV, fb, 64 * a, y, z, pol);
      }
    }
    ++issued;
  };
  if (threadIdx.x == 0) issue(item_at<C>(it0, n, seg_len, nseg), 0);

  const uint32_t uA = smem_u32(sA), uAL = smem_u32(sAL), uST = smem_u32(sST);
  const uint32_t uW = smem_u32(sW), uL = smem_u32(sL);
  int g = 0;  // steps of this CTA's walk
  for (int64_t it = it0; it < nitems && S.wait.ok; it += istep) {
    const Item I = item_at<C>(it, n, seg_len, nseg);
    // ---- the item's starting forward record: Psi (TMEM, causal) and its operand; vectors
    const float *rec0 = start + I.head * start_hs + I.seg * start_ss;
    load_record<D>(rec0, sST, myS, CAUSAL, L, sh);
    // the record's vectors (threads t < D, column t) and scalar (thread 0), to which each
    // chunk's exclusive sums within the item (from the aggregate kernel) are added
    float base[3] = {0.f, 0.f, 0.f}, base_s = 0.f;
    if (CAUSAL && threadIdx.x < D) {
#pragma unroll
      for (int k = 0; k < 3; ++k) base[k] = rec0[(int64_t)D * D + k * D + threadIdx.x];
    }
    if (CAUSAL && threadIdx.x == 0) base_s = rec0[(int64_t)D * D + 3 * D];
    float bs_acc = 0.f;  // thread 0: bs of the item (its vectors gather in sh.racc)
    for (int c = 0; c < I.nchunks; ++c, ++g) {
      uint8_t *st = sm + (g & 1) * G::P_STAGE;
      const uint32_t uQ = smem_u32(st + OQ), uK = smem_u32(st + OK), uV = smem_u32(st + OV);
      const int64_t t0 = I.t_begin + (int64_t)c * C;
      const int valid = I.t_end - t0 < C ? static_cast<int>(I.t_end - t0) : C;
      const bool more = CAUSAL && c + 1 < I.nchunks;  // the record after this chunk is needed
      // every lane takes two rows i (qa, qb) and a quarter of each group of 8 columns
      const bool la = L.qa < valid, lb = L.qb < valid;
      const int64_t rowa = I.head * n + t0 + L.qa, rowb = rowa + 8;  // global rows
      // keys row i sees: every key up to it (causal), all n (non-causal)
      const float Na = CAUSAL ? static_cast<float>(t0 + L.qa + 1) : static_cast<float>(n);
      const float Nb = CAUSAL ? static_cast<float>(t0 + L.qb + 1) : static_cast<float>(n);
      const int64_t slot = I.head * nck + t0 / C;  // this chunk's per-chunk vectors
      // causal: the forward record before this chunk = the item's record + the item's chunks
      // before this one; fetched now, stored once the stage has landed
      float fv[3] = {0.f, 0.f, 0.f}, fs = 0.f;
      if (CAUSAL && c > 0) {
        if (threadIdx.x < D) {
#pragma unroll
          for (int k = 0; k < 3; ++k) fv[k] = s_vec[slot * VF + k * D + threadIdx.x];
        }
        if (threadIdx.x == 0) fs = s_vec[slot * VF + 3 * D];
      }
      // causal: psi(k)'s row sums of the chunk (zero past the item's end, where the tile's
      // rows, past n, read as zero)
      const float skv = CAUSAL && threadIdx.x < valid ? skg[I.head * n + t0 + threadIdx.x] : 0.f;

      // ---- (a) psi on Q, with row sums (causal: psi(K) and its row sums come from K1)
      if (S.wait(&sh.full[g & 1], (g >> 1) & 1)) {
        if (threadIdx.x == 0) landed = g + 1;
        psi_tile<D>(st + OQ, C, sh.sq);
      }
      if (CAUSAL && threadIdx.x < C) sh.sk[threadIdx.x] = skv;
      if (CAUSAL && c > 0) {
        if (threadIdx.x < D) {
#pragma unroll
          for (int k = 0; k < 3; ++k) sh.vec[k][threadIdx.x] = base[k] + fv[k];
        }
        if (threadIdx.x == 0) sh.scal = base_s + fs;
      }
      fence_proxy_async_smem();
      if (!S.barrier()) break;
      // causal: psi(q) and its row sums to the workspace for the suffix walk (rows past n are
      // not stored)
      if (CAUSAL && threadIdx.x < valid) sqg[I.head * n + t0 + threadIdx.x] = sh.sq[threadIdx.x];
      if (threadIdx.x == 0) {
        if (CAUSAL) {
#pragma unroll
          for (int a = 0; a < AT; ++a)
            tma_store_3d(&tmPQ, st + OQ + a * kAtom, 64 * a, static_cast<int>(t0),
                         static_cast<int>(I.head), pol);
          tma_store_commit();
          // every earlier tile store (the other stage's psi(q), the last chunk's a pair and dq)
          // has read its tile before the next load, or this chunk's a pair, lands there
          tma_store_wait_read<1>();
        } else {
          tma_store_wait_read<0>();  // the last chunk's dq has been read from sA
        }
        // the next step's tiles into the other stage (its last reader, step g - 1, is done)
        if (c + 1 < I.nchunks)
          issue(I, c + 1);
        else if (it + istep < nitems)
          issue(item_at<C>(it + istep, n, seg_len, nseg), 0);
        if (CAUSAL) {
          // P' = psi(Q) psi(K)^T
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX, kdesc(uQ, ks, kAtom), kdesc(uK, ks, kAtom), I_P, ks > 0);
        } else {
          // O' = psi(Q) Psi
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX, kdesc(uQ, ks, kAtom), mdesc(uST, ks, SA), I_O, ks > 0);
        }
        mma_commit(&sh.mma);
        my_mma = true;
      } else if (threadIdx.x == 32) {
        if (CAUSAL) {
          // LV = L V
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tY, kdesc(uL, ks, kAtom), mdesc(uV, ks, kAtom), I_O, ks > 0);
        }
        phase_done(&sh.mma, CAUSAL);
        my_mma = my_mma || CAUSAL;
      } else if (threadIdx.x == 64) {
        if (more) {
          // Psi += psi(K)^T V
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tS, mdesc(uK, ks, kAtom), mdesc(uV, ks, kAtom), I_S, 1u);
        }
        phase_done(&sh.mma, more);
        my_mma = my_mma || more;
      }
      // psi(q_i) . zeta over this half's features (this lane's quarter of them)
      float dpa = 0.f, dpb = 0.f;
#pragma unroll
      for (int f = L.hf * HD + L.cq; f < L.hf * HD + HD; f += 8) {
        const float2 z = *reinterpret_cast<const float2 *>(&sh.vec[0][f]);
        const uint32_t ua = *reinterpret_cast<const uint32_t *>(st + OQ + tile_off(L.qa, f));
        const uint32_t ub = *reinterpret_cast<const uint32_t *>(st + OQ + tile_off(L.qb, f));
        dpa = fmaf(bf16_lo(ua), z.x, fmaf(bf16_hi(ua), z.y, dpa));
        dpb = fmaf(bf16_lo(ub), z.x, fmaf(bf16_hi(ub), z.y, dpb));
      }
      if (CAUSAL) {
        // ---- (c) M = mask(P' + sk) (j <= i) rounded into its operand; row sums of M
        S.wait_mma();
        if (S.wait.ok) {
          float p[16];
          tmem_quad32(myX + 32 * L.hf, p);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int j = 32 * L.hf + 8 * q + L.cq;  // columns j, j + 1
            const float2 skj = *reinterpret_cast<const float2 *>(&sh.sk[j]);
            const uint32_t ua = pack_bf16x2(j <= L.qa ? p[4 * q] + skj.x : 0.f,
                                            j + 1 <= L.qa ? p[4 * q + 1] + skj.y : 0.f);
            const uint32_t ub = pack_bf16x2(j <= L.qb ? p[4 * q + 2] + skj.x : 0.f,
                                            j + 1 <= L.qb ? p[4 * q + 3] + skj.y : 0.f);
            dpa += bf16_lo(ua) + bf16_hi(ua);
            dpb += bf16_lo(ub) + bf16_hi(ub);
            *reinterpret_cast<uint32_t *>(sW + sw128_offset(L.qa, j)) = ua;
            *reinterpret_cast<uint32_t *>(sW + sw128_offset(L.qb, j)) = ub;
          }
        }
      }
      // each row's partial denominator over the four lanes that hold it
      dpa += __shfl_xor_sync(0xffffffffu, dpa, 1);
      dpb += __shfl_xor_sync(0xffffffffu, dpb, 1);
      dpa += __shfl_xor_sync(0xffffffffu, dpa, 2);
      dpb += __shfl_xor_sync(0xffffffffu, dpb, 2);
      if ((L.lane & 3) == 0) {
        sh.part[L.hf][L.qa] = dpa;
        sh.part[L.hf][L.qb] = dpb;
      }
      if (CAUSAL) {
        fence_proxy_async_smem();
        if (!S.barrier()) break;
        if (threadIdx.x == 0) {
          // O' = psi(Q) Psi + M V
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX, kdesc(uQ, ks, kAtom), mdesc(uST, ks, SA), I_O, ks > 0);
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tX, kdesc(uW, ks, kAtom), mdesc(uV, ks, kAtom), I_O, 1u);
          mma_commit(&sh.mma);
        } else if (threadIdx.x == 32 || threadIdx.x == 64) {
          mbar_arrive(&sh.mma);
        }
      } else {
        S.wait_mma();
        if (!S.barrier()) break;
      }
      const float sqa = sh.sq[L.qa], sqb = sh.sq[L.qb];
      const float dena = Na * (kD + sqa) + sh.scal + sh.part[0][L.qa] + sh.part[1][L.qa];
      const float denb = Nb * (kD + sqb) + sh.scal + sh.part[0][L.qb] + sh.part[1][L.qb];

      // ---- (e) out_i, a_i = g_i / den_i (the bf16 pair into its operands and the
      //     workspace); partial a_i . out_i and a_i . (vs + LV_i)
      if (CAUSAL) S.wait_mma();
      float gda = 0.f, gdb = 0.f, cda = 0.f, cdb = 0.f;
      if (S.wait.ok) {
        const float inva = 1.f / dena, invb = 1.f / denb;
        const float wa = kD + sqa, wb = kD + sqb;
        // a_i, its bf16 pair and the partial dot products, for columns c, c + 1 of one row
        auto emit = [&](bool lv_ok, int row, int c, float o0, float o1, float l0,
                        float l1, float w, float inv, float g0, float g1, float &gd, float &cd) {
          const float2 vs = *reinterpret_cast<const float2 *>(&sh.vec[1][c]);
          const float2 sg = *reinterpret_cast<const float2 *>(&sh.vec[2][c]);
          const float v0 = vs.x + l0, v1 = vs.y + l1;
          const float a0 = lv_ok ? g0 * inv : 0.f, a1 = lv_ok ? g1 * inv : 0.f;
          gd = fmaf(a0, (w * v0 + sg.x + o0) * inv, fmaf(a1, (w * v1 + sg.y + o1) * inv, gd));
          cd = fmaf(a0, v0, fmaf(a1, v1, cd));
          const uint32_t hi = pack_bf16x2(a0, a1);
          const uint32_t lo = pack_bf16x2(a0 - bf16_lo(hi), a1 - bf16_hi(hi));
          *reinterpret_cast<uint32_t *>(sA + tile_off(row, c)) = hi;
          *reinterpret_cast<uint32_t *>(sAL + tile_off(row, c)) = lo;
        };
#pragma unroll 1
        for (int c0 = L.hf * HD; c0 < L.hf * HD + HD; c0 += 32) {
          float o[16], lv[16];
          tmem_quad32(myX + c0, o);
          if (CAUSAL) {
            tmem_quad32(myY + c0, lv);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) lv[e] = 0.f;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = c0 + 8 * q + L.cq;
            const uint32_t ga = *reinterpret_cast<const uint32_t *>(st + OG + tile_off(L.qa, c));
            const uint32_t gb = *reinterpret_cast<const uint32_t *>(st + OG + tile_off(L.qb, c));
            emit(la, L.qa, c, o[4 * q], o[4 * q + 1], lv[4 * q], lv[4 * q + 1], wa, inva,
                 bf16_lo(ga), bf16_hi(ga), gda, cda);
            emit(lb, L.qb, c, o[4 * q + 2], o[4 * q + 3], lv[4 * q + 2], lv[4 * q + 3], wb, invb,
                 bf16_lo(gb), bf16_hi(gb), gdb, cdb);
          }
        }
      }
      // each row's partial dot products over the four lanes that hold it
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        gda += __shfl_xor_sync(0xffffffffu, gda, o);
        gdb += __shfl_xor_sync(0xffffffffu, gdb, o);
        cda += __shfl_xor_sync(0xffffffffu, cda, o);
        cdb += __shfl_xor_sync(0xffffffffu, cdb, o);
      }
      if ((L.lane & 3) == 0) {
        sh.gd[L.hf][L.qa] = gda;
        sh.gd[L.hf][L.qb] = gdb;
        sh.cd[L.hf][L.qa] = cda;
        sh.cd[L.hf][L.qb] = cdb;
      }
      fence_proxy_async_smem();
      if (!S.barrier()) break;
      // b_i = -(a_i . out_i);  C_i = sum_{j seen} dW_ij = a_i . (vs + LV_i) + N_i b_i
      const float ba = la ? -(sh.gd[0][L.qa] + sh.gd[1][L.qa]) : 0.f;
      const float bb = lb ? -(sh.gd[0][L.qb] + sh.gd[1][L.qb]) : 0.f;
      const float Ca = la ? sh.cd[0][L.qa] + sh.cd[1][L.qa] + Na * ba : 0.f;
      const float Cb = lb ? sh.cd[0][L.qb] + sh.cd[1][L.qb] + Nb * bb : 0.f;
      if (L.hf == 0 && (L.lane & 3) == 0) {
        if (la) b_out[rowa] = ba;
        if (lb) b_out[rowb] = bb;
      }
      if (CAUSAL && threadIdx.x == 0) {
        // a as a bf16 pair to the workspace for the suffix walk (rows past n are not stored)
#pragma unroll
        for (int a = 0; a < AT; ++a) {
          tma_store_3d(&tmAH, sA + a * kAtom, 64 * a, static_cast<int>(t0),
                       static_cast<int>(I.head), pol);
          tma_store_3d(&tmAL, sAL + a * kAtom, 64 * a, static_cast<int>(t0),
                       static_cast<int>(I.head), pol);
        }
        tma_store_commit();
      }
      if (threadIdx.x == 0) {
        if (CAUSAL) {
          // dW = A V^T  (a_hi, then a_lo, along the contraction)
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX, kdesc(uA, ks, kAtom), kdesc(uV, ks, kAtom), I_P, ks > 0);
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX, kdesc(uAL, ks, kAtom), kdesc(uV, ks, kAtom), I_P, 1u);
        }
        phase_done(&sh.mma, CAUSAL);
      } else if (threadIdx.x == 32) {
        // dQ' = A Psi^T
#pragma unroll
        for (int ks = 0; ks < KSD; ++ks)
          mma_bf16_ss(tY, kdesc(uA, ks, kAtom), kdesc(uST, ks, SA), I_T, ks > 0);
#pragma unroll
        for (int ks = 0; ks < KSD; ++ks)
          mma_bf16_ss(tY, kdesc(uAL, ks, kAtom), kdesc(uST, ks, SA), I_T, 1u);
        mma_commit(&sh.mma);
        my_mma = true;
      } else if (threadIdx.x == 64) {
        // Phi += psi(Q)^T A
#pragma unroll
        for (int ks = 0; ks < KSC; ++ks)
          mma_bf16_ss(tR, mdesc(uQ, ks, kAtom), mdesc(uA, ks, kAtom), I_S, (c > 0 || ks > 0));
#pragma unroll
        for (int ks = 0; ks < KSC; ++ks)
          mma_bf16_ss(tR, mdesc(uQ, ks, kAtom), mdesc(uAL, ks, kAtom), I_S, 1u);
        mma_commit(&sh.mma);
        my_mma = true;
      }
      // this chunk's part of the item's reverse record: rho, as, tau (sh.racc), bs; b of each
      // row from the exchanged partial dot products, zero past the item's end (so is a)
      column_sums3<D>(sh.acc, [&](int i, int c, float (*t)[8]) {
        float qr[8], ar[8], lr[8];
        tile_row8(st + OQ, i, c, qr);
        tile_row8(sA, i, c, ar);
        tile_row8(sAL, i, c, lr);
        const float bi = i < valid ? -(sh.gd[0][i] + sh.gd[1][i]) : 0.f, sqi = sh.sq[i];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float aa = ar[e] + lr[e];
          t[0][e] = fmaf(qr[e], bi, t[0][e]);
          t[1][e] += aa;
          t[2][e] = fmaf(sqi, aa, t[2][e]);
        }
      });
      float bs_chunk = 0.f;  // thread 0: bs of this chunk's rows
      if (L.warp == 0) {
        const float bsum =
            warp_sum64([&](int i) { return i < valid ? -(sh.gd[0][i] + sh.gd[1][i]) : 0.f; });
        if (threadIdx.x == 0) bs_chunk = bsum;
      }
      S.wait_mma();
      if (CAUSAL) {
        // ---- (g) mask(dW + b) (j <= i) rounded into the M operand's buffer (M V is done);
        //     the record after this chunk: Psi (TMEM) -> operand (A Psi^T is done)
        if (S.wait.ok) {
          float w[16];
          tmem_quad32(myX + 32 * L.hf, w);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int j = 32 * L.hf + 8 * q + L.cq;  // columns j, j + 1
            *reinterpret_cast<uint32_t *>(sW + sw128_offset(L.qa, j)) =
                pack_bf16x2(j <= L.qa ? w[4 * q] + ba : 0.f, j + 1 <= L.qa ? w[4 * q + 1] + ba : 0.f);
            *reinterpret_cast<uint32_t *>(sW + sw128_offset(L.qb, j)) =
                pack_bf16x2(j <= L.qb ? w[4 * q + 2] + bb : 0.f,
                            j + 1 <= L.qb ? w[4 * q + 3] + bb : 0.f);
          }
          if (more) state_to_operand<D>(myS, sST, L);
        }
        // (i) stages dq in sA: the tile stores of the pair have read it by the barrier below
        if (threadIdx.x == 0) tma_store_wait_read<0>();
        fence_proxy_async_smem();
        if (!S.barrier()) break;
        if (threadIdx.x == 0) {
          // dQ' += mask(dW + b) psi(K)
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tY, kdesc(uW, ks, kAtom), mdesc(uK, ks, kAtom), I_O, 1u);
          mma_commit(&sh.mma);
        } else if (threadIdx.x == 32 || threadIdx.x == 64) {
          mbar_arrive(&sh.mma);
        }
        S.wait_mma();
      }
      // ---- (i) dq_i = (dQ'_i + zeta b_i + C_i) * phi'(q_i)
      if (S.wait.ok) {
#pragma unroll 1
        for (int c0 = L.hf * HD; c0 < L.hf * HD + HD; c0 += 32) {
          float f[16];
          tmem_quad32(myY + c0, f);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = c0 + 8 * q + L.cq;  // columns c, c + 1
            const float2 z = *reinterpret_cast<const float2 *>(&sh.vec[0][c]);
            const uint32_t pa = *reinterpret_cast<const uint32_t *>(st + OQ + tile_off(L.qa, c));
            const uint32_t pb = *reinterpret_cast<const uint32_t *>(st + OQ + tile_off(L.qb, c));
            *reinterpret_cast<uint32_t *>(sA + tile_off(L.qa, c)) =
                pack_bf16x2((f[4 * q] + fmaf(z.x, ba, Ca)) * dphi_from_psi(bf16_lo(pa)),
                            (f[4 * q + 1] + fmaf(z.y, ba, Ca)) * dphi_from_psi(bf16_hi(pa)));
            *reinterpret_cast<uint32_t *>(sA + tile_off(L.qb, c)) =
                pack_bf16x2((f[4 * q + 2] + fmaf(z.x, bb, Cb)) * dphi_from_psi(bf16_lo(pb)),
                            (f[4 * q + 3] + fmaf(z.y, bb, Cb)) * dphi_from_psi(bf16_hi(pb)));
          }
        }
      }
      fence_proxy_async_smem();
      if (!S.barrier()) break;
      if (threadIdx.x == 0) {
        // the chunk's dq rows, staged in sA (rows past n are not stored)
#pragma unroll
        for (int a = 0; a < AT; ++a)
          tma_store_3d(&tmDQ, sA + a * kAtom, 64 * a, static_cast<int>(t0),
                       static_cast<int>(I.head), pol);
        tma_store_commit();
      }
      // this chunk's reverse sums: into the item's record, and (causal) to the suffix walk
      if (threadIdx.x < D) {
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          const float x = sh.acc[k][threadIdx.x];
          sh.racc[k][threadIdx.x] += x;
          sh.acc[k][threadIdx.x] = 0.f;
          if (CAUSAL) r_vec[slot * VF + k * D + threadIdx.x] = x;
        }
      }
      if (threadIdx.x == 0) {
        bs_acc += bs_chunk;
        if (CAUSAL) r_vec[slot * VF + 3 * D] = bs_chunk;
      }
    }
    if (!S.wait.ok) break;
    // ---- the item's reverse record [Phi | rho | as | tau | bs]
    float *dst = r_rec + (I.head * nseg + I.seg) * rec_floats<D>();
    state_to_global<D>(myR, dst, L);
    drain_acc<D>(sh.racc, dst + (int64_t)D * D, D);
    if (threadIdx.x == 0) {
      dst[(int64_t)D * D + 3 * D] = bs_acc;
      dst[(int64_t)D * D + 3 * D + 1] = 0.f;
      dst[(int64_t)D * D + 3 * D + 2] = 0.f;
      dst[(int64_t)D * D + 3 * D + 3] = 0.f;
    }
    if (!S.barrier()) break;
  }
  if (threadIdx.x == 0) tma_store_wait_all<0>();  // the tile stores are done
  finish(sh, landed, issued, tmem, G::TCOLS, err, kIssuers, my_mma);
}

// ---------------------------------------------------------------- B3: the suffix walk
// psi(q), a_hi, a_lo: [heads][n][D] via tmQ, tmA, tmAL, and b_in: [heads][n] (causal only);
// psi(k), v via tmK, tmV; sqg, skg: the row sums of psi(q), psi(k) ([heads][n]).  dk, dv leave
// through tile stores (tmDK, tmDV: [heads][n][D]), staged in the stage's A slots.  start: each item's reverse record (causal: exclusive suffix at start +
// head * start_hs + seg * start_ss; non-causal: the head's total).  Writes dk, dv.
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, BCfg<D>::CTAS)
    bwd_suffix_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmAL,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const float *__restrict__ sqg,
                      const float *__restrict__ skg, const float *__restrict__ b_in,
                      const __grid_constant__ CUtensorMap tmDK,
                      const __grid_constant__ CUtensorMap tmDV,
                      const float *__restrict__ start, int64_t start_hs, int64_t start_ss,
                      const float *__restrict__ r_vec, int64_t n, int64_t seg_len, int64_t nseg,
                      int64_t nitems, int *err) {
  using G = BCfg<D>;
  constexpr int AT = G::AT;
  constexpr int KSD = D / 16;
  constexpr int KSC = C / 16;
  constexpr int HD = D / 2;
  constexpr int OQ = 0, OA = G::TILE, OAL = 2 * G::TILE, OK = 3 * G::TILE, OV = 4 * G::TILE;
  constexpr uint32_t LOAD = (CAUSAL ? 5 : 2) * G::TILE;
  constexpr uint32_t SA = G::S_ATOM;
  constexpr uint32_t I_P = make_idesc_bf16(64, 64, false, false);  // P'^T, dW^T
  constexpr uint32_t I_S = make_idesc_bf16(D, D, true, true);      // Phi update
  constexpr uint32_t I_O = make_idesc_bf16(64, D, false, true);    // psi(K) Phi, W A, W psi(Q)
  constexpr uint32_t I_T = make_idesc_bf16(64, D, false, false);   // V Phi^T
  constexpr float kD = static_cast<float>(D);
  constexpr int64_t VF = vec_floats<D>();
  const int64_t nck = (n + C - 1) / C;  // chunks per head

  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  BwdShared &sh = *reinterpret_cast<BwdShared *>(sm + G::S_SH);
  uint8_t *sFT = sm + G::S_ST;  // bf16 Phi (rows: features; 64-column blocks of values)
  uint8_t *sW0 = sm + G::S_W0;  // mask(w^T): the weights of the chunk's keys
  uint8_t *sW1 = sm + G::S_W1;  // mask(dW^T + b)
  const Lanes L = Lanes::make<D>();
  const int64_t it0 = blockIdx.x, istep = gridDim.x;

  init_barriers(sh, kIssuers);
  if (L.warp == 0) {
    tmem_alloc(&sh.tmem_base, G::TCOLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (CAUSAL) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmAL);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint32_t tX = tmem, tR = tmem + 2 * D;  // X: P'^T | dW^T, then dV' | dK'
  const uint32_t myX = tX + L.lane_off, myR = tR + L.lane_off;
  const uint64_t pol = policy_evict_first();
  Sync S(sh, err, L.lane);
  // walk step w of an item -> its chunk (the causal walk runs from the item's last chunk)
  auto chunk_of = [](int w, int nchunks) { return CAUSAL ? nchunks - 1 - w : w; };

  int issued = 0, landed = 0;
  bool my_mma = false;  // this thread (an issuer) issued products
  auto issue = [&](const Item &I, int w) {
    uint64_t *fb = &sh.full[issued & 1];
    uint8_t *st = sm + (issued & 1) * G::S_STAGE;
    mbar_arrive_expect_tx(fb, LOAD);
    const int y = static_cast<int>(I.t_begin + (int64_t)chunk_of(w, I.nchunks) * C);
    const int z = static_cast<int>(I.head);
#pragma unroll
    for (int a = 0; a < AT; ++a) {
      tma_load_3d(st + OK + a * kAtom, &tmK, fb, 64 * a, y, z, pol);
      tma_load_3d(st + OV + a * kAtom, &tmV, fb, 64 * a, y, z, pol);
      if (CAUSAL) {
        tma_load_3d(st + OQ + a * kAtom, &tmQ, fb, 64 * a, y, z, pol);
        tma_load_3d(st + OA + a * kAtom, &tmA, fb, 64 * a, y, z, pol);
        tma_load_3d(st + OAL + a * kAtom, &tmAL, fb, 64 * a, y, z, pol);
      }
    }
    ++issued;
  };
  if (threadIdx.x == 0) issue(item_at<C>(it0, n, seg_len, nseg), 0);

  const uint32_t uFT = smem_u32(sFT), uW0 = smem_u32(sW0), uW1 = smem_u32(sW1);
  int g = 0;
  for (int64_t it = it0; it < nitems && S.wait.ok; it += istep) {
    const Item I = item_at<C>(it, n, seg_len, nseg);
    // ---- the item's starting reverse record: Phi (TMEM, causal) and its operand; vectors
    load_record<D>(start + I.head * start_hs + I.seg * start_ss, sFT, myR, CAUSAL, L, sh);
    // b and the row sums of psi(k), psi(q) of a chunk's rows (zero past the item's end, where
    // the tiles' rows, past n, read as zero), fetched a chunk ahead of their use
    float nb = 0.f, nsk = 0.f, nsq = 0.f;
    auto fetch = [&](int ww) {
      const int64_t tt = I.t_begin + (int64_t)chunk_of(ww, I.nchunks) * C;
      if (threadIdx.x < I.t_end - tt && threadIdx.x < C) {
        const int64_t at = I.head * n + tt + threadIdx.x;
        nsk = skg[at];
        if (CAUSAL) {
          nb = b_in[at];
          nsq = sqg[at];
        }
      } else {
        nb = nsk = nsq = 0.f;
      }
    };
    fetch(0);
    for (int w = 0; w < I.nchunks; ++w, ++g) {
      uint8_t *st = sm + (g & 1) * G::S_STAGE;
      const uint32_t uQ = smem_u32(st + OQ), uA = smem_u32(st + OA), uAL = smem_u32(st + OAL);
      const uint32_t uK = smem_u32(st + OK), uV = smem_u32(st + OV);
      const int64_t t0 = I.t_begin + (int64_t)chunk_of(w, I.nchunks) * C;
      const int valid = I.t_end - t0 < C ? static_cast<int>(I.t_end - t0) : C;
      const bool more = CAUSAL && w + 1 < I.nchunks;  // the record before this chunk is needed

      const float bload = nb, skv = nsk, sqv = nsq;
      if (w + 1 < I.nchunks) fetch(w + 1);
      // this chunk's reverse sums (from the prefix walk), added to the record after it
      float rv[3] = {0.f, 0.f, 0.f}, rs = 0.f;
      if (more) {
        const float *src = r_vec + (I.head * nck + t0 / C) * VF;
        if (threadIdx.x < D) {
#pragma unroll
          for (int k = 0; k < 3; ++k) rv[k] = src[k * D + threadIdx.x];
        }
        if (threadIdx.x == 0) rs = src[3 * D];
      }
      // ---- (a) the stage (psi(K), V; causal psi(Q), a_hi, a_lo: the rows of A past the
      //     item's end zeroed) and the row sums
      if (S.wait(&sh.full[g & 1], (g >> 1) & 1)) {
        if (threadIdx.x == 0) landed = g + 1;
        if (CAUSAL) {
          zero_rows<D>(st + OA, valid);
          zero_rows<D>(st + OAL, valid);
        }
      }
      if (threadIdx.x < C) {
        sh.sk[threadIdx.x] = skv;
        sh.sq[threadIdx.x] = sqv;
        if (CAUSAL) sh.bv[threadIdx.x] = bload;
      }
      fence_proxy_async_smem();
      if (!S.barrier()) break;
      if (threadIdx.x == 0) {
        // the other stage's dk, dv (the last chunk's) have been read by their tile stores
        // before the next load lands there
        tma_store_wait_read<0>();
        if (w + 1 < I.nchunks)
          issue(I, w + 1);
        else if (it + istep < nitems)
          issue(item_at<C>(it + istep, n, seg_len, nseg), 0);
        if (CAUSAL) {
          // P'^T = psi(K) psi(Q)^T
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX, kdesc(uK, ks, kAtom), kdesc(uQ, ks, kAtom), I_P, ks > 0);
        } else {
          // dV' = psi(K) Phi  (Phi the head's total)
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX, kdesc(uK, ks, kAtom), mdesc(uFT, ks, SA), I_O, ks > 0);
        }
        mma_commit(&sh.mma);
        my_mma = true;
      } else if (threadIdx.x == 32) {
        if (CAUSAL) {
          // dW^T = V A^T (a_hi, then a_lo)
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX + 64, kdesc(uV, ks, kAtom), kdesc(uA, ks, kAtom), I_P, ks > 0);
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX + 64, kdesc(uV, ks, kAtom), kdesc(uAL, ks, kAtom), I_P, 1u);
        } else {
          // dK' = V Phi^T
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX + D, kdesc(uV, ks, kAtom), kdesc(uFT, ks, SA), I_T, ks > 0);
        }
        mma_commit(&sh.mma);
        my_mma = true;
      } else if (threadIdx.x == 64) {
        if (more) {
          // Phi += psi(Q)^T A
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tR, mdesc(uQ, ks, kAtom), mdesc(uA, ks, kAtom), I_S, 1u);
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tR, mdesc(uQ, ks, kAtom), mdesc(uAL, ks, kAtom), I_S, 1u);
        }
        phase_done(&sh.mma, more);
        my_mma = my_mma || more;
      }
      // v_j . as over this half's columns (as: the record after this chunk, read after the
      // barrier above, which orders it after the record's load or last update)
      if (L.v64) {
        float vdot = 0.f;
#pragma unroll 2
        for (int c0 = L.hf * HD; c0 < L.hf * HD + HD; c0 += 8) {
          float f[8];
          tile_row8(st + OV, L.r64, c0, f);
#pragma unroll
          for (int e = 0; e < 8; ++e) vdot = fmaf(f[e], sh.vec[1][c0 + e], vdot);
        }
        sh.gd[L.hf][L.r64] = vdot;
      }
      if (CAUSAL) {
        // ---- (c) row j: the weights w_ji = d + sq_i + sk_j + P'^T_ji and dW^T_ji + b_i, kept
        //     for i >= j and rounded into their operands; C'_j's part from this chunk
        S.wait_mma();
        // every lane takes two rows j (qa, qb) and 16 of this half's columns i (tmem_quad32)
        float cina = 0.f, cinb = 0.f;
        if (S.wait.ok) {
          float p[16];
          tmem_quad32(myX + 32 * L.hf, p);
          const float ska = kD + sh.sk[L.qa], skb = kD + sh.sk[L.qb];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = 32 * L.hf + 8 * q + L.cq;  // columns i, i + 1
            const float2 sqi = *reinterpret_cast<const float2 *>(&sh.sq[i]);
            const float a0 = i >= L.qa ? p[4 * q] + sqi.x + ska : 0.f;
            const float a1 = i + 1 >= L.qa ? p[4 * q + 1] + sqi.y + ska : 0.f;
            const float b0 = i >= L.qb ? p[4 * q + 2] + sqi.x + skb : 0.f;
            const float b1 = i + 1 >= L.qb ? p[4 * q + 3] + sqi.y + skb : 0.f;
            *reinterpret_cast<uint32_t *>(sW0 + sw128_offset(L.qa, i)) = pack_bf16x2(a0, a1);
            *reinterpret_cast<uint32_t *>(sW0 + sw128_offset(L.qb, i)) = pack_bf16x2(b0, b1);
          }
          tmem_quad32(myX + 64 + 32 * L.hf, p);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = 32 * L.hf + 8 * q + L.cq;
            const float2 bi = *reinterpret_cast<const float2 *>(&sh.bv[i]);
            const float a0 = i >= L.qa ? p[4 * q] + bi.x : 0.f;
            const float a1 = i + 1 >= L.qa ? p[4 * q + 1] + bi.y : 0.f;
            const float b0 = i >= L.qb ? p[4 * q + 2] + bi.x : 0.f;
            const float b1 = i + 1 >= L.qb ? p[4 * q + 3] + bi.y : 0.f;
            cina += a0 + a1;
            cinb += b0 + b1;
            *reinterpret_cast<uint32_t *>(sW1 + sw128_offset(L.qa, i)) = pack_bf16x2(a0, a1);
            *reinterpret_cast<uint32_t *>(sW1 + sw128_offset(L.qb, i)) = pack_bf16x2(b0, b1);
          }
        }
        // each row's sum over the four lanes that hold it
        cina += __shfl_xor_sync(0xffffffffu, cina, 1);
        cinb += __shfl_xor_sync(0xffffffffu, cinb, 1);
        cina += __shfl_xor_sync(0xffffffffu, cina, 2);
        cinb += __shfl_xor_sync(0xffffffffu, cinb, 2);
        if ((L.lane & 3) == 0) {
          sh.part[L.hf][L.qa] = cina;
          sh.part[L.hf][L.qb] = cinb;
        }
        fence_proxy_async_smem();
        if (!S.barrier()) break;
        if (threadIdx.x == 0) {
          // dV' = psi(K) Phi + mask(w^T) a_hi
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX, kdesc(uK, ks, kAtom), mdesc(uFT, ks, SA), I_O, ks > 0);
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tX, kdesc(uW0, ks, kAtom), mdesc(uA, ks, kAtom), I_O, 1u);
          mma_commit(&sh.mma);
        } else if (threadIdx.x == 32) {
          // dK' = V Phi^T + mask(dW^T + b) psi(Q)
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tX + D, kdesc(uV, ks, kAtom), kdesc(uFT, ks, SA), I_T, ks > 0);
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tX + D, kdesc(uW1, ks, kAtom), mdesc(uQ, ks, kAtom), I_O, 1u);
          mma_commit(&sh.mma);
        } else if (threadIdx.x == 64) {
          mbar_arrive(&sh.mma);
        }
      }
      // ---- (e) dv_j = (d + sk_j) as + tau + dV'_j;  dk_j = (dK'_j + rho + C'_j) phi'(k_j),
      //     C'_j = v_j . as + bs + (this chunk's sum_{i >= j} dW_ij);  Phi -> operand
      S.wait_mma();
      if (!CAUSAL && !S.barrier()) break;  // both halves of v_j . as are in sh.gd
      if (S.wait.ok) {
        // every lane takes two rows j (qa, qb) and 16 of each 32 columns (tmem_quad32); dv
        // and dk go to the stage's A and A-lo slots (the products that read them are done)
        uint8_t *sDV = st + OA, *sDK = st + OAL;
        const float ska = kD + sh.sk[L.qa], skb = kD + sh.sk[L.qb];
        const float cpa = sh.gd[0][L.qa] + sh.gd[1][L.qa] + sh.scal +
                          (CAUSAL ? sh.part[0][L.qa] + sh.part[1][L.qa] : 0.f);
        const float cpb = sh.gd[0][L.qb] + sh.gd[1][L.qb] + sh.scal +
                          (CAUSAL ? sh.part[0][L.qb] + sh.part[1][L.qb] : 0.f);
#pragma unroll 1
        for (int c0 = L.hf * HD; c0 < L.hf * HD + HD; c0 += 32) {
          float f[16];
          tmem_quad32(myX + c0, f);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = c0 + 8 * q + L.cq;  // columns c, c + 1
            const float2 as = *reinterpret_cast<const float2 *>(&sh.vec[1][c]);
            const float2 tau = *reinterpret_cast<const float2 *>(&sh.vec[2][c]);
            *reinterpret_cast<uint32_t *>(sDV + tile_off(L.qa, c)) =
                pack_bf16x2(fmaf(ska, as.x, tau.x + f[4 * q]), fmaf(ska, as.y, tau.y + f[4 * q + 1]));
            *reinterpret_cast<uint32_t *>(sDV + tile_off(L.qb, c)) =
                pack_bf16x2(fmaf(skb, as.x, tau.x + f[4 * q + 2]),
                            fmaf(skb, as.y, tau.y + f[4 * q + 3]));
          }
          tmem_quad32(myX + D + c0, f);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = c0 + 8 * q + L.cq;
            const float2 rho = *reinterpret_cast<const float2 *>(&sh.vec[0][c]);
            const uint32_t pa = *reinterpret_cast<const uint32_t *>(st + OK + tile_off(L.qa, c));
            const uint32_t pb = *reinterpret_cast<const uint32_t *>(st + OK + tile_off(L.qb, c));
            *reinterpret_cast<uint32_t *>(sDK + tile_off(L.qa, c)) =
                pack_bf16x2((f[4 * q] + rho.x + cpa) * dphi_from_psi(bf16_lo(pa)),
                            (f[4 * q + 1] + rho.y + cpa) * dphi_from_psi(bf16_hi(pa)));
            *reinterpret_cast<uint32_t *>(sDK + tile_off(L.qb, c)) =
                pack_bf16x2((f[4 * q + 2] + rho.x + cpb) * dphi_from_psi(bf16_lo(pb)),
                            (f[4 * q + 3] + rho.y + cpb) * dphi_from_psi(bf16_hi(pb)));
          }
        }
        if (more) state_to_operand<D>(myR, sFT, L);
      }
      fence_proxy_async_smem();
      if (!S.barrier()) break;
      if (threadIdx.x == 0) {
        // the chunk's dk, dv rows (rows past n are not stored)
#pragma unroll
        for (int a = 0; a < AT; ++a) {
          tma_store_3d(&tmDV, st + OA + a * kAtom, 64 * a, static_cast<int>(t0),
                       static_cast<int>(I.head), pol);
          tma_store_3d(&tmDK, st + OAL + a * kAtom, 64 * a, static_cast<int>(t0),
                       static_cast<int>(I.head), pol);
        }
        tma_store_commit();
      }
      if (more) {
        // the record before this chunk
        if (threadIdx.x < D) {
#pragma unroll
          for (int k = 0; k < 3; ++k) sh.vec[k][threadIdx.x] += rv[k];
        }
        if (threadIdx.x == 0) sh.scal += rs;
      }
    }
  }
  if (threadIdx.x == 0) tma_store_wait_all<0>();  // the tile stores are done
  finish(sh, landed, issued, tmem, G::TCOLS, err, kIssuers, my_mma);
}

// ------------------------------------------------------------------ host side
template <typename K>
cudaError_t prepare(K kern, int smem) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

template <int D, bool CAUSAL>
cudaError_t backward_dims(const void *q, const void *k, const void *v, const void *g, void *dq,
                          void *dk, void *dv, int64_t heads, int64_t n, int64_t seg,
                          const TcBackwardLayout &W, int *err, cudaStream_t st) {
  using G = BCfg<D>;
  const int64_t nseg = (n + seg - 1) / seg;
  const int64_t rec = rec_floats<D>();
  const int64_t nitems = heads * nseg;
  const int64_t sms = sm_count();
  const unsigned grid = static_cast<unsigned>(nitems < sms * G::CTAS ? nitems : sms * G::CTAS);
  const unsigned grid_agg =
      static_cast<unsigned>(nitems < sms * G::G_CTAS ? nitems : sms * G::G_CTAS);
  CUtensorMap tq, tk, tv, tg, ta, tal, tpq, tpk, tdq, tdk, tdv;
  cudaError_t e;
  if ((e = make_tmap_bf16(&tq, q, heads, n, D, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tk, k, heads, n, D, C)) != cudaSuccess) return e;
  // psi(q), psi(k) in the workspace: stored by B1 and K1, read by the walks
  if ((e = make_tmap_bf16(&tpq, W.psi_q, heads, n, D, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tpk, W.psi_k, heads, n, D, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, heads, n, D, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tg, g, heads, n, D, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&ta, W.a_hi, heads, n, D, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tal, W.a_lo, heads, n, D, C)) != cudaSuccess) return e;
  // the gradients leave through tile stores
  if ((e = make_tmap_bf16(&tdq, dq, heads, n, D, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tdk, dk, heads, n, D, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tdv, dv, heads, n, D, C)) != cudaSuccess) return e;
  // the scans treat a record as 4 x (rec / 4 - 1) + 4 floats: element by element
  const int sdk = 4, sdv = static_cast<int>(rec / 4 - 1);

  // K1 + K2: the forward record before every segment (causal) or of the head (non-causal)
  auto kg = bwd_aggregate_kernel<D>;
  if ((e = prepare(kg, G::G_SMEM)) != cudaSuccess) return e;
  kg<<<grid_agg, kThreads, G::G_SMEM, st>>>(tk, tv, tpk, W.sk, W.s_rec, W.s_vec, n, seg, nseg,
                                            nitems, err);
  count_launches(1);
  record_launch_event(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const float *s_start = W.s_rec;
  int64_t s_hs = nseg * rec, s_ss = rec;
  if (CAUSAL) {
    e = launch_scan_states(W.s_rec, heads, nseg, sdk, sdv, 0, nullptr, 0, nullptr, 0, nullptr,
                           nullptr, st);
  } else {
    e = launch_scan_states(W.s_rec, heads, nseg, sdk, sdv, 1, W.s_tot, rec, W.s_tot + rec - 4,
                           rec, nullptr, nullptr, st);
    s_start = W.s_tot;
    s_hs = rec;
    s_ss = 0;
  }
  if (e != cudaSuccess) return e;

  // B1: dq, a (hi, lo), b and the reverse record of every segment
  auto k1 = bwd_prefix_kernel<D, CAUSAL>;
  if ((e = prepare(k1, G::P_SMEM)) != cudaSuccess) return e;
  k1<<<grid, kThreads, G::P_SMEM, st>>>(tq, tpk, tv, tg, tpq, W.sq, W.sk, tdq, ta, tal,
                                        W.b, s_start, s_hs, s_ss, W.s_vec,
                                        W.r_rec, W.r_vec, n, seg, nseg, nitems, err);
  count_launches(1);
  record_launch_event(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // K2: the reverse record after every segment (causal) or of the head (non-causal)
  const float *r_start = W.r_rec;
  int64_t r_hs = nseg * rec, r_ss = rec;
  if (CAUSAL) {
    e = launch_scan_states(W.r_rec, heads, nseg, sdk, sdv, 2, nullptr, 0, nullptr, 0, nullptr,
                           nullptr, st);
  } else {
    e = launch_scan_states(W.r_rec, heads, nseg, sdk, sdv, 1, W.r_tot, rec, W.r_tot + rec - 4,
                           rec, nullptr, nullptr, st);
    r_start = W.r_tot;
    r_hs = rec;
    r_ss = 0;
  }
  if (e != cudaSuccess) return e;

  // B3: dk, dv
  auto k3 = bwd_suffix_kernel<D, CAUSAL>;
  if ((e = prepare(k3, G::S_SMEM)) != cudaSuccess) return e;
  k3<<<grid, kThreads, G::S_SMEM, st>>>(tpq, ta, tal, tpk, tv, W.sq, W.sk, W.b, tdk, tdv,
                                        r_start, r_hs, r_ss,
                                        W.r_vec, n, seg, nseg, nitems, err);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

}  // namespace

int64_t tc_backward_segment(int64_t heads, int64_t n, int d) {
  // the segment (a multiple of 256 tokens, at most 4096) with the smallest loss to partial
  // waves over every walk CTA slot of the device, preferring long segments (fewer records)
  const int64_t slots = (int64_t)sm_count() * (d == 64 ? BCfg<64>::CTAS : BCfg<128>::CTAS);
  int64_t best = 256, best_score = -1;
  for (int64_t seg = 4096; seg >= 256; seg -= 256) {
    const int64_t items = heads * ((n + seg - 1) / seg);
    const int64_t waves = (items + slots - 1) / slots;
    const int64_t eff = items * 1000 / (waves * slots);
    if (best_score < 0 || eff > best_score + 30) {
      best_score = eff;
      best = seg;
    }
  }
  const int64_t nrounded = (n + C - 1) / C * C;
  return best > nrounded ? nrounded : best;
}

TcBackwardLayout tc_backward_layout(void *ws, int64_t heads, int64_t n, int d, int64_t seg,
                                    size_t *bytes) {
  const int64_t nseg = (n + seg - 1) / seg;
  const int64_t rec = (int64_t)d * d + 3 * d + 4;
  size_t off = 0;
  char *base = static_cast<char *>(ws);
  auto take = [&](size_t nbytes) {
    char *p = base ? base + off : nullptr;
    off += (nbytes + 255) / 256 * 256;
    return p;
  };
  TcBackwardLayout W;
  W.s_rec = reinterpret_cast<float *>(take(heads * nseg * rec * sizeof(float)));
  W.r_rec = reinterpret_cast<float *>(take(heads * nseg * rec * sizeof(float)));
  W.s_tot = reinterpret_cast<float *>(take(heads * rec * sizeof(float)));
  W.r_tot = reinterpret_cast<float *>(take(heads * rec * sizeof(float)));
  W.a_hi = reinterpret_cast<__nv_bfloat16 *>(take(heads * n * d * sizeof(__nv_bfloat16)));
  W.a_lo = reinterpret_cast<__nv_bfloat16 *>(take(heads * n * d * sizeof(__nv_bfloat16)));
  W.b = reinterpret_cast<float *>(take(heads * n * sizeof(float)));
  const int64_t nck = (n + C - 1) / C;
  W.s_vec = reinterpret_cast<float *>(take(heads * nck * (3 * d + 4) * sizeof(float)));
  W.r_vec = reinterpret_cast<float *>(take(heads * nck * (3 * d + 4) * sizeof(float)));
  W.psi_q = reinterpret_cast<__nv_bfloat16 *>(take(heads * n * d * sizeof(__nv_bfloat16)));
  W.psi_k = reinterpret_cast<__nv_bfloat16 *>(take(heads * n * d * sizeof(__nv_bfloat16)));
  W.sq = reinterpret_cast<float *>(take(heads * n * sizeof(float)));
  W.sk = reinterpret_cast<float *>(take(heads * n * sizeof(float)));
  if (bytes) *bytes = off;
  return W;
}

cudaError_t tc_backward(const void *q, const void *k, const void *v, const void *g, void *dq,
                        void *dk, void *dv, int64_t heads, int64_t n, int d, int causal,
                        int64_t seg, void *ws, int *err, cudaStream_t st) {
  const TcBackwardLayout W = tc_backward_layout(ws, heads, n, d, seg, nullptr);
  if (d == 64)
    return causal ? backward_dims<64, true>(q, k, v, g, dq, dk, dv, heads, n, seg, W, err, st)
                  : backward_dims<64, false>(q, k, v, g, dq, dk, dv, heads, n, seg, W, err, st);
  if (d == 128)
    return causal ? backward_dims<128, true>(q, k, v, g, dq, dk, dv, heads, n, seg, W, err, st)
                  : backward_dims<128, false>(q, k, v, g, dq, dk, dv, heads, n, seg, W, err, st);
  return cudaErrorInvalidValue;
}

}  // namespace linattn
