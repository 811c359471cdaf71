// bf16-I/O forward pass on the 5th-generation tensor cores (tcgen05, TMEM, TMA): the segment
// aggregates and the non-causal outputs, and the host side of the whole tensor-core pass.
//
// The method (page "Efficient Transformers: Linear Attention and Flash Attention",
// sections "Linear attention: reordering the matmuls, not shrinking them" and "The
// recurrent view: attention as an RNN"):
//     out_i = phi(q_i) S / phi(q_i).z,  S = sum_j phi(k_j) v_j^T,  z = sum_j phi(k_j)
// with j <= i in the causal mode.  A head's tokens are split into segments, the work items of
// the CTAs, and segments into chunks of C = 64 tokens.  The pass runs as three kernels:
//   K1  this file, mode kState: each segment's aggregate (S_s, z_s) -> fp32 workspace;
//   K2  simt_forward.cu: exclusive prefix over the segments (causal) or the per-head total;
//   K3  causal: tc_causal.cu (128-token chunks from each segment's prefix);
//       non-causal: this file, mode kNoncausalOut, out = phi(Q) S / phi(Q).z.
//
// Products (tcgen05.mma kind::f16, bf16 operands, fp32 accumulators in TMEM):
//   [S | z] += phi(K_c)^T [V_c | 1]   M=DK N=DV+16 K=64   (A: K MN-major; a constant ones atom
//                                      after each V tile puts z in column DV)
//   [O | den] = phi(Q_c) [S | z]      M=64 N=DV+16 K=DK   (B: the bf16 total, MN-major, an
//                                      extra atom holds z, so column DV is the denominator)
// DK is the feature dimension of phi(q), phi(k) (the head dimension for phi = elu + 1, m for
// random features), DV the value dimension; each 64 or 128.
//
// Warp roles (one CTA per SM; 22 warps in the aggregate mode, 18 in the non-causal mode):
//   warp 0     TMA producer: 3-D tiled loads (128-byte swizzle) of the chunks into a ring of
//              stages; no multicast.
//   warp 1     TMEM allocation and the single MMA-issuing thread.
//   next 12/8  feature map: phi applied in place to the K (aggregate) or Q (non-causal) tiles
//              (packed bf16), K rows beyond the item's end zeroed.
//   next 4     state: the item's aggregate out of TMEM (aggregate); the head's total rounded
//              into the bf16 S operand (non-causal).
//   last 4     output: O / den -> bf16 rows stored straight to global memory (non-causal).
// Every wait is bounded (2 s); a wait that gives up records LINATTN_ERR_TIMEOUT and the
// CTA drains and exits without trapping.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace linattn {
namespace {

using namespace tc;

constexpr int C = kTcChunk;     // tokens per chunk (64)
constexpr int kAtom = C * 128;  // one [64 rows][64 bf16] 128B-swizzled atom: 8 KB

enum Mode : int { kState = 0, kNoncausalOut = 2 };

constexpr int kWarpTMA = 0;
constexpr int kWarpMMA = 1;
constexpr int kWarpXform0 = 2;
constexpr int kGroupThreads = 128;
// Warps per mode (measured on the benchmark shapes).  Aggregate: the feature map on K bounds
// the chunk rate, so 12 feature-map warps (22 warps, 80 registers).  Non-causal: 8 feature-map
// warps (18 warps, 96 registers).
template <int MODE>
struct Warps {
  static constexpr int XFORM = MODE == kState ? 12 : 8;
  static constexpr int XTHREADS = XFORM * 32;
  static constexpr int STATE0 = kWarpXform0 + XFORM;  // state group: 4 warps
  static constexpr int OUT0 = STATE0 + 4;             // output group: 4 warps
  static constexpr int THREADS = (OUT0 + 4) * 32;
};

template <int DK, int DV, int MODE>
struct Cfg {
  static constexpr int AK = DK / 64;        // 64-column atoms per [64][DK] tile (Q, K)
  static constexpr int AV = DV / 64;        // 64-column atoms per [64][DV] tile (V)
  static constexpr bool LQ = MODE != kState;
  static constexpr bool LKV = MODE == kState;
  // aggregate stage: K tile, V tile, then a constant atom whose column 0 is 1: the S MMA with
  // N = DV + 16 then also accumulates z = phi(K)^T 1 in its column DV.
  // non-causal stage: the Q tile.
  static constexpr int OFF_V = AK * kAtom;
  static constexpr int OFF_ONES = OFF_V + AV * kAtom;
  static constexpr int STAGE = LQ ? AK * kAtom : OFF_ONES + kAtom;
  static constexpr int LOAD_BYTES = LQ ? AK * kAtom : (AK + AV) * kAtom;
  // non-causal: bf16 S operand, MN-major [atoms][DK rows][128 B] with one more atom whose
  // column 0 is z, so O (N = DV + 16) carries phi(q_i).z in its column DV; two of them, so
  // the next item's total is rounded while this one runs
  static constexpr int S_ATOM = DK * 128;
  static constexpr int S_BUF = LQ ? (AV + 1) * S_ATOM : 0;
  static constexpr int S_BYTES = 2 * S_BUF;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int NS_FIT = (kMaxSmem - 1024 - BAR_BYTES - S_BYTES) / STAGE;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int OFF_S = NS * STAGE;
  static constexpr int OFF_BAR = OFF_S + S_BYTES;
  static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
  static_assert(NS >= 2, "at least two pipeline stages");
  static_assert(SMEM <= kMaxSmem, "shared memory budget");
  static_assert(OFF_S % 1024 == 0 && STAGE % 1024 == 0 && OFF_V % 1024 == 0 &&
                    OFF_ONES % 1024 == 0 && S_ATOM % 1024 == 0,
                "128B-swizzled operands need 1024-byte alignment");
};

// TMEM columns.  Aggregate: two [S | z] accumulators (DV + 16 columns each), one per item
// parity, so one item's aggregate is written out while the next one accumulates.
// Non-causal: two O buffers (DV + 16 columns, the denominator in column DV).
template <int DV, int MODE>
struct TmemMap {
  static constexpr uint32_t OW = (DV + 16 + 31) / 32 * 32;
  static constexpr uint32_t O0 = 0;
  static constexpr uint32_t O1 = OW;
  static constexpr uint32_t S = 0;
  static constexpr uint32_t S1 = kTmemCols / 2;
  static_assert((MODE == kNoncausalOut ? O1 + OW : S1 + DV + 16) <= kTmemCols, "TMEM budget");
};

struct Bars {
  uint64_t full[8], ready[8], empty[8];
  uint64_t o_full[2], o_empty[2], fin;
  // per item parity: aggregate mode, S accumulator complete (MMA -> state group) / written out
  // (state group -> MMA); non-causal, S operand rounded (state group -> MMA) / no longer read
  // (MMA -> state group)
  uint64_t item_full[2], item_empty[2];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

// CTA b takes the items b, b + gridDim.x, b + 2 gridDim.x, ... (one item when the grid
// covers them all; several on persistent CTAs).  Every role walks the same sequence of
// chunks, and g counts them across items, so the stage ring, the barrier phases and the O
// buffers run on from one item into the next: the loads of an item's first chunks overlap
// the previous item's last ones.
// PHI: apply phi = elu + 1 to Q and K (the method); false takes Q and K as given,
// non-negative features (FAVOR+ features computed by the feature kernels).
// init_state (non-causal): the head's total [DK][DV] then z [DK], at init_state +
// head * init_head_stride.  out_state (aggregate): [heads][nseg][DK*DV + DK].
template <int DK, int DV, int MODE, bool PHI>
__global__ void __launch_bounds__(Warps<MODE>::THREADS, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ out,
              const float *__restrict__ init_state, int64_t init_head_stride,
              float *__restrict__ out_state, int64_t n, int64_t seg_len, int64_t nseg,
              int64_t nitems, int *err) {
  using G = Cfg<DK, DV, MODE>;
  using TM = TmemMap<DV, MODE>;
  using W = Warps<MODE>;
  constexpr int NS = G::NS;
  constexpr int KSD = DK / 16;  // K-steps over the feature dimension
  constexpr int KSC = C / 16;   // K-steps over the chunk's tokens
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Bars &bar = *reinterpret_cast<Bars *>(smem + G::OFF_BAR);
  volatile int *abort = &bar.abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t it0 = blockIdx.x, istep = gridDim.x;

  // ---- set-up: barriers, constant operand blocks, TMEM
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.ready[s], W::XTHREADS);
      mbar_init(&bar.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.o_full[b], 1);
      mbar_init(&bar.o_empty[b], kGroupThreads);
      mbar_init(&bar.item_full[b], MODE == kNoncausalOut ? kGroupThreads : 1);
      mbar_init(&bar.item_empty[b], MODE == kState ? kGroupThreads : 1);
    }
    mbar_init(&bar.fin, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  if (G::LKV) {
    // ones atom of every stage: column 0 of every row is 1.0 (row r's column 0 sits in 16-byte
    // chunk r & 7)
    for (int s = 0; s < NS; ++s) {
      uint32_t *ones = reinterpret_cast<uint32_t *>(smem + s * G::STAGE + G::OFF_ONES);
      for (int i = threadIdx.x; i < kAtom / 4; i += W::THREADS) {
        const int row = i >> 5, word = i & 31;  // 32 words per 128-byte row
        ones[i] = (word == 4 * (row & 7)) ? 0x00003F80u : 0u;
      }
    }
  }
  if (MODE == kNoncausalOut) {
    // the z atoms of the two S operands: zero except column 0 (rewritten with z per item)
    for (int b = 0; b < 2; ++b) {
      uint32_t *za =
          reinterpret_cast<uint32_t *>(smem + G::OFF_S + b * G::S_BUF + G::AV * G::S_ATOM);
      for (int i = threadIdx.x; i < G::S_ATOM / 4; i += W::THREADS) za[i] = 0u;
    }
  }
  fence_proxy_async_smem();
  if (warp == kWarpMMA) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTMA && lane == 0) {
    if (G::LQ) prefetch_tmap(&tmQ);
    if (G::LKV) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp == kWarpTMA) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int g = 0;  // chunks issued
      bool ok = true;
      for (int64_t it = it0; ok && it < nitems; it += istep) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        const int zc = static_cast<int>(I.head);
        for (int c = 0; c < I.nchunks; ++c, ++g) {
          const int s = g % NS;
          const uint32_t ph = g / NS;
          if (g >= NS && !mbar_wait(&bar.empty[s], (ph - 1) & 1, abort, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar.full[s], G::LOAD_BYTES);
          uint8_t *st = smem + s * G::STAGE;
          const int y = static_cast<int>(I.t_begin + (int64_t)c * C);
          if (G::LQ) {
#pragma unroll
            for (int a = 0; a < G::AK; ++a)
              tma_load_3d(st + a * kAtom, &tmQ, &bar.full[s], a * 64, y, zc, pol);
          } else {
#pragma unroll
            for (int a = 0; a < G::AK; ++a)
              tma_load_3d(st + a * kAtom, &tmK, &bar.full[s], a * 64, y, zc, pol);
#pragma unroll
            for (int a = 0; a < G::AV; ++a)
              tma_load_3d(st + G::OFF_V + a * kAtom, &tmV, &bar.full[s], a * 64, y, zc, pol);
          }
        }
      }
      // drain: every issued load has landed before the CTA may exit
      for (int gg = (g > NS ? g - NS : 0); gg < g; ++gg)
        mbar_wait_drain(&bar.full[gg % NS], (gg / NS) & 1, err);
    }
  } else if (warp == kWarpMMA) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t I_O = make_idesc_bf16(64, DV + 16, false, true);
      constexpr uint32_t I_S = make_idesc_bf16(DK, DV + 16, true, true);
      const uint32_t st0 = smem_u32(smem);
      int g = 0;
      int j = 0;  // items of this CTA
      bool ok = true;
      for (int64_t it = it0; ok && it < nitems; it += istep, ++j) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        const int b = j & 1;
        const uint32_t tS = tmem + (b ? TM::S1 : TM::S);
        const uint64_t dS = mnmajor_base(smem_u32(smem + G::OFF_S + b * G::S_BUF), G::S_ATOM);
        // aggregate: this S accumulator written out (item j - 2); non-causal: the head's
        // total rounded into this S operand
        if (MODE == kState && j >= 2 &&
            !mbar_wait(&bar.item_empty[b], ((j >> 1) - 1) & 1, abort, err))
          break;
        if (MODE == kNoncausalOut && !mbar_wait(&bar.item_full[b], (j >> 1) & 1, abort, err))
          break;
        for (int c = 0; c < I.nchunks; ++c, ++g) {
          const int s = g % NS;
          if (!mbar_wait(&bar.ready[s], (g / NS) & 1, abort, err)) {
            ok = false;
            break;
          }
          const uint32_t st = st0 + s * G::STAGE;
          if (MODE == kState) {
            tc_fence_after();
            const uint64_t dKm = mnmajor_base(st, kAtom);               // K, MN-major
            const uint64_t dVm = mnmajor_base(st + G::OFF_V, kAtom);    // [V | ones], MN-major
#pragma unroll
            for (int ks = 0; ks < KSC; ++ks)
              mma_bf16_ss(tS, desc_add(dKm, mnmajor_off(ks)), desc_add(dVm, mnmajor_off(ks)),
                          I_S, (c > 0 || ks > 0) ? 1u : 0u);
            mma_commit(&bar.empty[s]);
            continue;
          }
          const int ob = g & 1;
          const uint32_t tO = tmem + (ob ? TM::O1 : TM::O0);
          // this O buffer drained
          if (g >= 2 && !mbar_wait(&bar.o_empty[ob], ((g >> 1) - 1) & 1, abort, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dQk = kmajor_base(st);
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tO, desc_add(dQk, kmajor_off(ks, kAtom)), desc_add(dS, mnmajor_off(ks)),
                        I_O, ks > 0 ? 1u : 0u);
          mma_commit(&bar.o_full[ob]);
          mma_commit(&bar.empty[s]);
        }
        if (!ok) break;
        if (MODE == kState) mma_commit(&bar.item_full[b]);        // aggregate complete
        if (MODE == kNoncausalOut) mma_commit(&bar.item_empty[b]);  // S operand no longer read
      }
      // every MMA this CTA issued has finished before TMEM is released
      mma_commit(&bar.fin);
      mbar_wait_drain(&bar.fin, 0, err);
    }
  } else if (warp < W::STATE0) {
    // ================================================================ feature map
    // phi in place on the Q tile (non-causal) or on the K tile (aggregate); K rows past the
    // item's end are zeroed (they must add nothing to S or z).
    const int xt = threadIdx.x - kWarpXform0 * 32;
    int g = 0;
    bool ok = true;
    for (int64_t it = it0; ok && it < nitems; it += istep) {
      const Item I = item_at<C>(it, n, seg_len, nseg);
      for (int c = 0; c < I.nchunks; ++c, ++g) {
        const int s = g % NS;
        if (!mbar_wait(&bar.full[s], (g / NS) & 1, abort, err)) {
          ok = false;
          break;
        }
        uint8_t *st = smem + s * G::STAGE;
        const int64_t left = I.t_end - (I.t_begin + (int64_t)c * C);
        const int valid = left < C ? static_cast<int>(left) : C;
#pragma unroll 2
        for (int i = xt; i < G::AK * kAtom / 16; i += W::XTHREADS) {
          uint4 *p = reinterpret_cast<uint4 *>(st) + i;
          if (G::LQ) {
            if (PHI) *p = phi_bf16x8(*p);
          } else {
            const int row = (i % (kAtom / 16)) >> 3;  // 8 x 16 B per 128-byte row
            uint4 x = make_uint4(0u, 0u, 0u, 0u);
            if (row < valid) {
              x = *p;
              if (PHI) x = phi_bf16x8(x);
            }
            *p = x;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bar.ready[s]);
      }
    }
  } else if (warp < W::OUT0) {
    // ================================================================ state group
    // Aggregate: each item's aggregate out of TMEM.  Non-causal: each item's head total ->
    // one of the two S operands.  Control flow is warp-uniform: lane 0 waits and the warp
    // shares the outcome.
    const int sp = warp & 3;  // TMEM sub-partition of this warp
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    // row rS of S (M = DK: lanes 0..127 at DK = 128; at DK = 64 rows 16 sp .. 16 sp + 15 sit
    // in lanes 0..15 of sub-partition sp)
    const int rS = DK == 128 ? 32 * sp + lane : 16 * sp + lane;
    const bool vS = DK == 128 || lane < 16;
    WarpWaiter wait{abort, err, lane};
    if (MODE == kNoncausalOut) {
      int j = 0;
      for (int64_t it = it0; it < nitems; it += istep, ++j) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        const int b = j & 1;
        uint8_t *sS = smem + G::OFF_S + b * G::S_BUF;
        // the MMAs of item j - 2 no longer read this S operand
        if (j < 2 || wait(&bar.item_empty[b], ((j >> 1) - 1) & 1)) {
          const float *src = init_state + I.head * init_head_stride;
          if (vS) {
            for (int c0 = 0; c0 < DV; c0 += 8) {
              const float4 lo = *reinterpret_cast<const float4 *>(src + (int64_t)rS * DV + c0);
              const float4 hi =
                  *reinterpret_cast<const float4 *>(src + (int64_t)rS * DV + c0 + 4);
              const float f[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
              *reinterpret_cast<uint4 *>(sS + (c0 >> 6) * G::S_ATOM +
                                         sw128_offset(rS, c0 & 63)) = pack8(f);
            }
            // z_r in column 0 of the z atom
            *reinterpret_cast<__nv_bfloat16 *>(sS + G::AV * G::S_ATOM + sw128_offset(rS, 0)) =
                __float2bfloat16_rn(src[(int64_t)DK * DV + rS]);
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(&bar.item_full[b]);
      }
    } else {
      // segment aggregates -> fp32 workspace [DK][DV] then z[DK]
      int j = 0;
      for (int64_t it = it0; it < nitems; it += istep, ++j) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        const int b = j & 1;
        const uint32_t tS = tmem + lane_off + (b ? TM::S1 : TM::S);
        if (wait(&bar.item_full[b], (j >> 1) & 1)) {
          tc_fence_after();
          float *dst = out_state + (I.head * nseg + I.seg) * ((int64_t)DK * DV + DK);
          for (int c0 = 0; c0 < DV; c0 += 32) {
            uint32_t r[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) tmem_ld16_async(tS + c0 + 16 * q, r + 16 * q);
            tmem_ld_wait();
            tmem_reg_fence<32>(r);
            if (vS) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4 *>(dst + (int64_t)rS * DV + c0 + e) =
                    make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
            }
          }
          const uint32_t zr = tmem_ld1(tS + DV);
          if (vS) dst[(int64_t)DK * DV + rS] = __uint_as_float(zr);
        }
        tc_fence_before();
        mbar_arrive(&bar.item_empty[b]);
      }
    }
  } else if (MODE == kNoncausalOut) {
    // ================================================================ output
    // O / den -> bf16 rows stored straight to global memory (32-byte stores; rows past the
    // item's end are not written).  Lanes < 16 of each warp hold rows of the M = 64 tile.
    const int sp = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const bool v64 = lane < 16;
    const int r64 = 16 * sp + lane;
    WarpWaiter wait{abort, err, lane};
    int g = 0;
    for (int64_t it = it0; it < nitems; it += istep) {
      const Item I = item_at<C>(it, n, seg_len, nseg);
      for (int c = 0; c < I.nchunks; ++c, ++g) {
        const int ob = g & 1;
        const uint32_t tO = tmem + lane_off + (ob ? TM::O1 : TM::O0);
        if (!wait(&bar.o_full[ob], (g >> 1) & 1)) continue;
        tc_fence_after();
        const float inv = 1.f / __uint_as_float(tmem_ld1(tO + DV));
        const int64_t t = I.t_begin + (int64_t)c * C + r64;
        const bool live = v64 && t < I.t_end;
        __nv_bfloat16 *orow = out + (I.head * n + (live ? t : 0)) * DV;
#pragma unroll 1
        for (int c0 = 0; c0 < DV; c0 += 32) {
          uint32_t r[32];
          tmem_ld16_async(tO + c0, r);
          tmem_ld16_async(tO + c0 + 16, r + 16);
          tmem_ld_wait();
          tmem_reg_fence<32>(r);
          if (live) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              float f[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) f[e] = __uint_as_float(r[16 * q + e]) * inv;
              st_global_32B(orow + c0 + 16 * q, pack8(f), pack8(f + 8));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bar.o_empty[ob]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMMA) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host side
template <int DK, int DV, int MODE, bool PHI>
cudaError_t launch_tc(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                      void *out, const float *init, int64_t ihs, float *out_state,
                      int64_t heads, int64_t n, int64_t seg, int64_t nseg, int *err,
                      cudaStream_t st) {
  using G = Cfg<DK, DV, MODE>;
  auto kern = tc_kernel<DK, DV, MODE, PHI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  // One CTA holds a whole SM's shared memory and TMEM; persistent CTAs (one per SM, items
  // dealt round-robin) save each item the CTA start-up and pipeline fill and drain.
  const int64_t nitems = heads * nseg;
  const int64_t sms = sm_count();
  const unsigned grid = static_cast<unsigned>(nitems < sms ? nitems : sms);
  kern<<<grid, Warps<MODE>::THREADS, G::SMEM, st>>>(q, k, v, static_cast<__nv_bfloat16 *>(out),
                                                    init, ihs, out_state, n, seg, nseg, nitems,
                                                    err);
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

// The whole pass: K1 aggregates, K2 scan, K3 outputs.  q, k: [heads][n][DK]; v, out: [heads]
// [n][DV].
template <int DK, int DV, bool PHI>
cudaError_t tc_forward_dims(const void *q, const void *k, const void *v, void *out,
                            int64_t heads, int64_t n, int causal, int64_t seg, void *ws, int *err,
                            const float *init_S, const float *init_z, cudaStream_t st) {
  const int64_t nseg = (n + seg - 1) / seg;
  const int64_t per = (int64_t)DK * DV + DK;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_tmap_bf16(&tk, k, heads, n, DK, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, heads, n, DV, C)) != cudaSuccess) return e;
  float *w = static_cast<float *>(ws);
  // causal: one kernel, each segment's prefix by a look-back over the published states
  if (causal) return tc_causal_fused(q, k, v, out, heads, n, DK, DV, seg, ws, init_S, init_z,
                                     PHI ? 0 : 1, err, st);
  e = launch_tc<DK, DV, kState, PHI>(tk, tk, tv, out, nullptr, 0, w, heads, n, seg, nseg, err,
                                     st);
  if (e != cudaSuccess) return e;
  // per-head totals, packed as [heads][DK*DV + DK] (S row-major, then z)
  float *tot = w + heads * nseg * per;
  e = launch_scan_states(w, heads, nseg, DK, DV, 1, tot, per, tot + (int64_t)DK * DV, per, init_S,
                         init_z, st);
  if (e != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tq, q, heads, n, DK, C)) != cudaSuccess) return e;
  return launch_tc<DK, DV, kNoncausalOut, PHI>(tq, tk, tv, out, tot, per, nullptr, heads, n, seg,
                                               nseg, err, st);
}

template <int DK, int DV>
cudaError_t tc_state_dims(const void *k, const void *v, float *S_out, float *z_out,
                          int64_t heads, int64_t n, int64_t seg, void *ws, int *err,
                          cudaStream_t st) {
  const int64_t nseg = (n + seg - 1) / seg;
  CUtensorMap tk, tv;
  cudaError_t e;
  if ((e = make_tmap_bf16(&tk, k, heads, n, DK, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, heads, n, DV, C)) != cudaSuccess) return e;
  float *w = static_cast<float *>(ws);
  e = launch_tc<DK, DV, kState, true>(tk, tk, tv, nullptr, nullptr, 0, w, heads, n, seg, nseg,
                                      err, st);
  if (e != cudaSuccess) return e;
  return launch_scan_states(w, heads, nseg, DK, DV, 1, S_out, (int64_t)DK * DV, z_out, DK,
                            nullptr, nullptr, st);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

cudaError_t make_tmap_bf16(CUtensorMap *m, const void *ptr, int64_t heads, int64_t n, int d,
                           int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int64_t tc_default_segment(int64_t heads, int64_t n, int d) {
  (void)d;
  // smallest tail loss over whole waves of the device's SMs (one CTA each), preferring long
  // segments
  const int64_t sms = sm_count();
  int64_t best = 64, best_score = -1;
  for (int64_t seg = 4096; seg >= 256; seg -= 256) {
    const int64_t nseg = (n + seg - 1) / seg;
    const int64_t ctas = heads * nseg;
    const int64_t waves = (ctas + sms - 1) / sms;
    // efficiency in 1/1000 units; prefer longer segments on ties
    const int64_t eff = ctas * 1000 / (waves * sms);
    if (eff > best_score + 30 || (best_score < 0)) {
      best_score = eff;
      best = seg;
    }
  }
  const int64_t nrounded = ((n + kTcCausalChunk - 1) / kTcCausalChunk) * kTcCausalChunk;
  return best > nrounded ? nrounded : best;
}

size_t tc_workspace_bytes(int64_t heads, int64_t n, int dk, int dv, int64_t seg, int causal) {
  if (causal) return tc_fused_workspace_bytes(heads, n, dk, dv, seg);
  const int64_t nseg = (n + seg - 1) / seg;
  const int64_t per = (int64_t)dk * dv + dk;
  return (size_t)(heads * nseg * per + (causal ? 0 : heads * per)) * sizeof(float);
}

cudaError_t tc_forward(const void *q, const void *k, const void *v, void *out, int64_t heads,
                       int64_t n, int dk, int dv, int causal, int64_t seg, void *ws, int *err,
                       const float *init_S, const float *init_z, int features,
                       cudaStream_t st) {
  if (!features) {  // phi = elu + 1 keeps the dimension
    if (dk == 64 && dv == 64)
      return tc_forward_dims<64, 64, true>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                           init_z, st);
    if (dk == 128 && dv == 128)
      return tc_forward_dims<128, 128, true>(q, k, v, out, heads, n, causal, seg, ws, err,
                                             init_S, init_z, st);
    return cudaErrorInvalidValue;
  }
  if (dk == 64 && dv == 64)
    return tc_forward_dims<64, 64, false>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                          init_z, st);
  if (dk == 128 && dv == 128)
    return tc_forward_dims<128, 128, false>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                            init_z, st);
  if (dk == 128 && dv == 64)
    return tc_forward_dims<128, 64, false>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                           init_z, st);
  if (dk == 64 && dv == 128)
    return tc_forward_dims<64, 128, false>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                           init_z, st);
  return cudaErrorInvalidValue;
}

cudaError_t tc_forward_state(const void *k, const void *v, float *S_out, float *z_out,
                             int64_t heads, int64_t n, int d, int64_t seg, void *ws, int *err,
                             cudaStream_t st) {
  return d == 64 ? tc_state_dims<64, 64>(k, v, S_out, z_out, heads, n, seg, ws, err, st)
                 : tc_state_dims<128, 128>(k, v, S_out, z_out, heads, n, seg, ws, err, st);
}

}  // namespace linattn
