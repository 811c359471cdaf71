// Causal outputs of the bf16-I/O forward pass on caller-given features (Performer's FAVOR+
// random features, named on the page "Efficient Transformers: Linear Attention and Flash
// Attention"), whose dimension m may differ from the value dimension d, on the tensor cores in
// chunks of 128 tokens.  (Features with m = d, and phi = elu + 1, run tc_forward.cu's causal
// kernel.)
//
// The method (same page, sections "Linear attention: reordering the matmuls, not shrinking
// them" and "The recurrent view: attention as an RNN"): out_i = f(q_i) S_i / f(q_i).z_i with
// S_i = sum_{j<=i} f(k_j) v_j^T (m x d) and z_i = sum_{j<=i} f(k_j), f the given features.  A work
// item is one segment of one head; it starts from the exclusive prefix state (S_<s, z_<s) of
// the earlier segments (the aggregates of tc_forward.cu and their scan in simt_forward.cu) and
// walks its chunks of C = 128 tokens with the running state:
//     num_c = F(Q_c) S_<c + mask(F(Q_c) F(K_c)^T) V_c
//     den_c = F(Q_c).z_<c + mask(F(Q_c) F(K_c)^T) 1
//     S_<c+1 = S_<c + F(K_c)^T V_c,   z_<c+1 = z_<c + F(K_c)^T 1
// where mask keeps the keys j <= i (the current token included).
//
// Tensor-core products of one chunk (tcgen05.mma kind::f16: bf16 operands, fp32 accumulators in
// tensor memory; DK = m, DV = d):
//   P   = F(Q_c) F(K_c)^T       M=128 N=128 K=DK   A: Q, B: K (both K-major, shared memory)
//   O   = F(Q_c) S_<c           M=128 N=DV  K=DK   B: the bf16 copy of S_<c (MN-major)
//   S  += F(K_c)^T V_c          M=DK  N=DV  K=128  A: K (MN-major), B: V (MN-major)
//   O  += mask(P) V_c           M=128 N=DV  K=128  A: the masked bf16 scores, in tensor memory
// The scores never go through shared memory: the score warps mask and round them in place
// (fp32 columns 0..127 become packed bf16 columns 0..63), and the P V product reads them from
// tensor memory.  The normaliser z is summed on the CUDA cores: the feature warps add up the
// columns of F(K) (z_<c+1) and take F(q_i).z_<c per row.
//
// Warp roles (18 warps, one CTA per SM):
//   warp 0       TMA producer: Q, K, V tiles of a chunk (64-column boxes, 128-byte swizzle)
//                into a ring of stages; no multicast.
//   warp 1       tensor-memory allocation and the single thread that issues every MMA.
//   warps 2-9    features: K rows past the item's end zeroed; F(q_i).z_<c per row; column
//                sums of F(K) into z.
//   warps 10-13  state: each item's starting state into tensor memory and the bf16 S operand;
//                after each chunk's update, S_<c+1 rounded into that operand.
//   warps 14-17  scores and output: mask and round P, the row sums and denominators; O / den
//                -> bf16 rows, stored straight to global memory (32-byte stores).
// Every wait is bounded (2 s); a wait that gives up records LINATTN_ERR_TIMEOUT and the CTA
// drains its copies and products and exits without trapping.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace linattn {
namespace {

using namespace tc;

constexpr int C = kTcFeatureChunk;  // tokens per chunk (128)
constexpr int kAtom = C * 128;     // one [128 rows][64 bf16] 128B-swizzled atom: 16 KB

constexpr int kWarpTMA = 0;
constexpr int kWarpMMA = 1;
constexpr int kWarpPhi0 = 2;
constexpr int kPhiWarps = 8;
constexpr int kPhiThreads = kPhiWarps * 32;
constexpr int kWarpState0 = kWarpPhi0 + kPhiWarps;  // 10
constexpr int kWarpOut0 = kWarpState0 + 4;          // 14
constexpr int kThreads = (kWarpOut0 + 4) * 32;      // 576
constexpr int kZBufs = 3;  // column-sum buffers of the feature-map warps, by chunk mod 3
// items of at most this many tokens run on persistent CTAs
constexpr int64_t kPersistentTokens = 2048;

// Shared memory of a CTA: NS stages (Q, K, V tiles of one chunk), the bf16 S operand, the
// column-sum buffers, phi(q).z per stage, and the barriers.
constexpr int kBarBytes = 256;
template <int DK, int DV>
constexpr int smem_bytes(int ns) {
  return ns * (2 * (DK / 64) + DV / 64) * kAtom + (DV / 64) * DK * 128 + kZBufs * DK * 4 +
         ns * C * 4 + kBarBytes;
}
template <int DK, int DV>
constexpr int stages_that_fit() {
  return smem_bytes<DK, DV>(4) <= kMaxSmem ? 4
         : smem_bytes<DK, DV>(3) <= kMaxSmem ? 3
                                             : 2;
}

// DK: feature dimension of phi(q), phi(k) (the head dimension d for phi = elu + 1; m for
// random features); DV: value dimension d.  Both 64 or 128.
template <int DK, int DV>
struct Cfg {
  static constexpr int AK = DK / 64;         // 64-column atoms per [128][DK] tile (Q, K)
  static constexpr int AV = DV / 64;         // 64-column atoms per [128][DV] tile (V)
  static constexpr int QTILE = AK * kAtom;   // bytes of a bf16 [128][DK] tile
  static constexpr int OFF_K = QTILE;
  static constexpr int OFF_V = 2 * QTILE;
  static constexpr int STAGE = 2 * QTILE + AV * kAtom;
  static constexpr int NS = stages_that_fit<DK, DV>();
  static constexpr int S_ATOM = DK * 128;    // one 64-column atom of the [DK][DV] S operand
  static constexpr int S_BYTES = AV * S_ATOM;
  static constexpr int OFF_S = NS * STAGE;
  static constexpr int OFF_ZACC = OFF_S + S_BYTES;            // float [kZBufs][DK]
  static constexpr int OFF_QZ = OFF_ZACC + kZBufs * DK * 4;  // float [NS][C]
  static constexpr int OFF_BAR = OFF_QZ + NS * C * 4;
  static constexpr int SMEM = OFF_BAR + kBarBytes;
  static_assert(SMEM == smem_bytes<DK, DV>(NS) && SMEM <= kMaxSmem, "shared memory budget");
  static_assert(STAGE % 1024 == 0 && OFF_S % 1024 == 0, "128B-swizzled operands need 1024 B");
};

// Tensor-memory columns: P (128), two O buffers (DV each), S (DV; rows in lanes, M = DK).
template <int DV>
struct TmemMap {
  static constexpr uint32_t P = 0;
  static constexpr uint32_t O0 = 128;
  static constexpr uint32_t O1 = O0 + DV;
  static constexpr uint32_t S = O1 + DV;
  static_assert(S + DV <= kTmemCols, "tensor memory budget");
};

template <int NS>
struct Bars {
  uint64_t full[NS], ready[NS], empty[NS];
  uint64_t p_full, p_ready, s_full, s_ready, o_full[2], o_empty[2], zsync, fin;
  uint32_t tmem_base;
  int abort;
};

// Byte offset of (row, column) in a 128B-swizzled tile of 64-column rows.
__device__ __forceinline__ uint32_t sw_off(int row, int col) {  // 128B-swizzled [rows][64]
  return sw128_offset(static_cast<uint32_t>(row), static_cast<uint32_t>(col));
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f16: A is read from tensor memory (K-major, two bf16
// per 32-bit column), B from a shared-memory descriptor.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void red_add_shared(float *p, float v) {
  asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(smem_u32(p)), "f"(v) : "memory");
}

// CTA b takes the items b, b + gridDim.x, ... (one item when the grid covers them all).  Every
// role walks the same sequence of chunks, and g counts them across items, so the stage ring,
// the barrier phases and the O buffers run on from one item into the next.
// init_state: per item, the fp32 state [DK][DV] then z [DK] before the item's first token, at
// init_state + head * init_head_stride + seg * init_seg_stride.
// q and k are the features F(q), F(k) themselves (non-negative; no feature map applied).
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    tc_causal_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ out,
                     const float *__restrict__ init_state, int64_t init_head_stride,
                     int64_t init_seg_stride, int64_t n, int64_t seg_len, int64_t nseg,
                     int64_t nitems, int *err) {
  using G = Cfg<DK, DV>;
  using TM = TmemMap<DV>;
  constexpr int NS = G::NS;
  constexpr int KSD = DK / 16;  // K-steps over the feature dimension
  constexpr int KSC = C / 16;  // K-steps over the chunk's tokens
  extern __shared__ __align__(1024) uint8_t smem[];
  // Every stage and operand offset is a multiple of 1024 from the base; a base that is not
  // (never seen) is reported instead of used.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(err, kErrLayout);
    return;
  }
  Bars<NS> &bar = *reinterpret_cast<Bars<NS> *>(smem + G::OFF_BAR);
  float *zacc = reinterpret_cast<float *>(smem + G::OFF_ZACC);
  float *qz = reinterpret_cast<float *>(smem + G::OFF_QZ);
  volatile int *abort = &bar.abort;
  const int warp = threadIdx.x >> 5;
  const bool a32 = aligned32(out);  // output rows take full-sector stores
  const int lane = threadIdx.x & 31;
  const int64_t it0 = blockIdx.x, istep = gridDim.x;

  // ---- set-up: barriers, the column-sum buffers, tensor memory
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.ready[s], kPhiThreads);
      mbar_init(&bar.empty[s], 1);
    }
    mbar_init(&bar.p_full, 1);
    mbar_init(&bar.p_ready, 128);
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.s_ready, 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.o_full[b], 1);
      mbar_init(&bar.o_empty[b], 128);
    }
    mbar_init(&bar.zsync, kPhiThreads);
    mbar_init(&bar.fin, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < kZBufs * DK; i += kThreads) zacc[i] = 0.f;
  if (warp == kWarpMMA) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTMA && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
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
          if (g >= NS && !mbar_wait(&bar.empty[s], ((g / NS) - 1) & 1, abort, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar.full[s], G::STAGE);
          uint8_t *st = smem + s * G::STAGE;
          const int y = static_cast<int>(I.t_begin + (int64_t)c * C);
#pragma unroll
          for (int a = 0; a < G::AK; ++a) {
            tma_load_3d(st + a * kAtom, &tmQ, &bar.full[s], a * 64, y, zc, pol);
            tma_load_3d(st + G::OFF_K + a * kAtom, &tmK, &bar.full[s], a * 64, y, zc, pol);
          }
#pragma unroll
          for (int a = 0; a < G::AV; ++a)
            tma_load_3d(st + G::OFF_V + a * kAtom, &tmV, &bar.full[s], a * 64, y, zc, pol);
        }
      }
      // every issued load has landed before the CTA may exit
      for (int gg = (g > NS ? g - NS : 0); gg < g; ++gg)
        mbar_wait_drain(&bar.full[gg % NS], (gg / NS) & 1, err);
    }
  } else if (warp == kWarpMMA) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t I_P = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t I_O = make_idesc_bf16(128, DV, false, true);
      constexpr uint32_t I_S = make_idesc_bf16(DK, DV, true, true);
      constexpr uint32_t I_PV = make_idesc_bf16(128, DV, false, true);
      const uint32_t tP = tmem + TM::P;
      const uint32_t tS = tmem + TM::S;
      const uint64_t dS = mnmajor_base(smem_u32(smem + G::OFF_S), G::S_ATOM);
      const uint32_t st0 = smem_u32(smem);
      int g = 0;
      bool ok = true;
      for (int64_t it = it0; ok && it < nitems; it += istep) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        for (int c = 0; c < I.nchunks; ++c, ++g) {
          const int s = g % NS;
          // this chunk's tiles transformed; S_<c in the S operand and TMEM S free to update;
          // this O buffer emitted (chunk g - 2)
          if (!mbar_wait(&bar.ready[s], (g / NS) & 1, abort, err) ||
              !mbar_wait(&bar.s_ready, g & 1, abort, err) ||
              (g >= 2 && !mbar_wait(&bar.o_empty[g & 1], ((g >> 1) - 1) & 1, abort, err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = st0 + s * G::STAGE;
          const uint64_t dQ = kmajor_base(st);
          const uint64_t dK = kmajor_base(st + G::OFF_K);
          const uint64_t dKm = mnmajor_base(st + G::OFF_K, kAtom);
          const uint64_t dVm = mnmajor_base(st + G::OFF_V, kAtom);
          const uint32_t tO = tmem + ((g & 1) ? TM::O1 : TM::O0);
          // The scores first, so that their rounding overlaps the next products; then
          // F(Q_c) S_<c and S += F(K_c)^T V_c (not after the item's last chunk: nothing reads
          // it), independent accumulators issued K-step by K-step.
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tP, desc_add(dQ, kmajor_off(ks, kAtom)),
                        desc_add(dK, kmajor_off(ks, kAtom)), I_P, ks > 0 ? 1u : 0u);
          mma_commit(&bar.p_full);
#pragma unroll
          for (int ks = 0; ks < (KSD > KSC ? KSD : KSC); ++ks) {
            if (ks < KSD)
              mma_bf16_ss(tO, desc_add(dQ, kmajor_off(ks, kAtom)), desc_add(dS, mnmajor_off(ks)),
                          I_O, ks > 0 ? 1u : 0u);
            if (c + 1 < I.nchunks && ks < KSC)
              mma_bf16_ss(tS, desc_add(dKm, mnmajor_off(ks)), desc_add(dVm, mnmajor_off(ks)), I_S,
                          1u);
          }
          mma_commit(&bar.s_full);
          // O += mask(P) V_c, the rounded scores read from tensor memory
          if (!mbar_wait(&bar.p_ready, g & 1, abort, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ts(tO, tP + 8 * ks, desc_add(dVm, mnmajor_off(ks)), I_PV, 1u);
          mma_commit(&bar.o_full[g & 1]);
          mma_commit(&bar.empty[s]);
        }
      }
      // every MMA this CTA issued has finished before tensor memory is released
      mma_commit(&bar.fin);
      mbar_wait_drain(&bar.fin, 0, err);
    }
  } else if (warp < kWarpState0) {
    // ================================================================ feature map
    // Thread t holds the 16-byte vectors t + 256 k of a tile: rows r0 + 32 m (m = 0..3) of
    // every atom, always in the same logical 8-column group cg of the atom (the swizzle XOR
    // is r0 & 7 for all four rows).  It keeps z_<c for its columns in registers.
    const int t = threadIdx.x - kWarpPhi0 * 32;
    const int r0 = t >> 3;
    const int cg = (t & 7) ^ (r0 & 7);
    const int vec_off = r0 * 128 + (t & 7) * 16;  // byte offset of row r0's vector in an atom
    WarpWaiter wait{abort, err, lane};
    grid_dependency_wait();  // the prefix states come from the scan before this kernel
    float zr[G::AK][8];
    int g = 0;
    for (int64_t it = it0; it < nitems; it += istep) {
      const Item I = item_at<C>(it, n, seg_len, nseg);
      const float *z0 = init_state + I.head * init_head_stride + I.seg * init_seg_stride +
                        (int64_t)DK * DV + cg * 8;
#pragma unroll
      for (int a = 0; a < G::AK; ++a) {
        const float4 lo = *reinterpret_cast<const float4 *>(z0 + a * 64);
        const float4 hi = *reinterpret_cast<const float4 *>(z0 + a * 64 + 4);
        zr[a][0] = lo.x; zr[a][1] = lo.y; zr[a][2] = lo.z; zr[a][3] = lo.w;
        zr[a][4] = hi.x; zr[a][5] = hi.y; zr[a][6] = hi.z; zr[a][7] = hi.w;
      }
      for (int c = 0; c < I.nchunks; ++c, ++g) {
        const int s = g % NS;
        float *zbuf = zacc + (g % kZBufs) * DK;
        if (wait(&bar.full[s], (g / NS) & 1)) {
          uint8_t *st = smem + s * G::STAGE;
          const int64_t left = I.t_end - (I.t_begin + (int64_t)c * C);
          const int valid = left < C ? static_cast<int>(left) : C;
          // K: rows past the item's end zeroed; column sums of F(K).  One atom at a time:
          // its four vectors are loaded together (the shared-memory latency is paid once per
          // atom, not once per vector).
          float cs[G::AK][8];
#pragma unroll
          for (int a = 0; a < G::AK; ++a)
#pragma unroll
            for (int e = 0; e < 8; ++e) cs[a][e] = 0.f;
#pragma unroll
          for (int a = 0; a < G::AK; ++a) {
            uint4 *p = reinterpret_cast<uint4 *>(st + G::OFF_K + a * kAtom + vec_off);
            uint4 x[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) x[m] = p[m * 256];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              if (r0 + 32 * m >= valid) {
                x[m] = make_uint4(0u, 0u, 0u, 0u);
                p[m * 256] = x[m];
              }
              const uint32_t w[4] = {x[m].x, x[m].y, x[m].z, x[m].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                cs[a][2 * e] += bf16_lo(w[e]);
                cs[a][2 * e + 1] += bf16_hi(w[e]);
              }
            }
          }
          // Q: F(q_i).z_<c for rows r0 + 32 m (this thread's 8 columns per atom)
          float qp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int a = 0; a < G::AK; ++a) {
            const uint4 *p = reinterpret_cast<const uint4 *>(st + a * kAtom + vec_off);
            uint4 x[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) x[m] = p[m * 256];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const uint32_t w[4] = {x[m].x, x[m].y, x[m].z, x[m].w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                qp[m] += bf16_lo(w[e]) * zr[a][2 * e] + bf16_hi(w[e]) * zr[a][2 * e + 1];
            }
          }
          // a row's 8 column groups sit in the 8 lanes that share t >> 3
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            qp[m] += __shfl_xor_sync(0xffffffffu, qp[m], 1);
            qp[m] += __shfl_xor_sync(0xffffffffu, qp[m], 2);
            qp[m] += __shfl_xor_sync(0xffffffffu, qp[m], 4);
          }
          if ((t & 7) == 0) {
#pragma unroll
            for (int m = 0; m < 4; ++m) qz[s * C + r0 + 32 * m] = qp[m];
          }
          // the lanes l, l^9, l^18, l^27 of a warp hold the same column group (rows differ)
#pragma unroll
          for (int a = 0; a < G::AK; ++a)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              cs[a][e] += __shfl_xor_sync(0xffffffffu, cs[a][e], 9);
              cs[a][e] += __shfl_xor_sync(0xffffffffu, cs[a][e], 18);
            }
          if (lane < 8) {
#pragma unroll
            for (int a = 0; a < G::AK; ++a)
#pragma unroll
              for (int e = 0; e < 8; ++e) red_add_shared(zbuf + a * 64 + cg * 8 + e, cs[a][e]);
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(&bar.ready[s]);
        // every warp's column sums are in: z_<c+1 = z_<c + phi(K_c)^T 1
        mbar_arrive(&bar.zsync);
        if (wait(&bar.zsync, g & 1)) {
#pragma unroll
          for (int a = 0; a < G::AK; ++a)
#pragma unroll
            for (int e = 0; e < 8; ++e) zr[a][e] += zbuf[a * 64 + cg * 8 + e];
          // the buffer of chunk g - 1 (read by every thread before this barrier) is zeroed
          // for chunk g + 2 (whose sums start after the next barrier)
          if (t < DK) zacc[((g + kZBufs - 1) % kZBufs) * DK + t] = 0.f;
        }
      }
    }
  } else if (warp < kWarpOut0) {
    // ================================================================ state group
    // Row rS of the S accumulator (M = DK: lanes 0..127 at DK = 128; at DK = 64 the M = 64
    // layout puts rows 16 sp .. 16 sp + 15 in lanes 0..15 of sub-partition sp).
    const int sp = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const int rS = DK == 128 ? 32 * sp + lane : 16 * sp + lane;
    const bool vS = DK == 128 || lane < 16;
    uint8_t *sS = smem + G::OFF_S;
    WarpWaiter wait{abort, err, lane};
    grid_dependency_wait();  // the prefix states come from the scan before this kernel
    // 32 consecutive columns [c0, c0 + 32) of row rS (fp32 bits) -> the bf16 S operand
    auto store_S32 = [&](const uint32_t *r, int c0) {
      if (!vS) return;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * j + e]);
        *reinterpret_cast<uint4 *>(sS + (c0 >> 6) * G::S_ATOM + sw_off(rS, (c0 & 63) + 8 * j)) =
            pack8(f);
      }
    };
    int g = 0;
    for (int64_t it = it0; it < nitems; it += istep) {
      const Item I = item_at<C>(it, n, seg_len, nseg);
      // the item's starting state, once the previous item's last products are done with
      // TMEM S and the S operand
      if (g == 0 || wait(&bar.s_full, (g - 1) & 1)) {
        tc_fence_after();
        const float *src = init_state + I.head * init_head_stride + I.seg * init_seg_stride;
        for (int c0 = 0; c0 < DV; c0 += 32) {
          uint32_t r[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
            if (vS) f = *reinterpret_cast<const float4 *>(src + (int64_t)rS * DV + c0 + 4 * j);
            r[4 * j + 0] = __float_as_uint(f.x);
            r[4 * j + 1] = __float_as_uint(f.y);
            r[4 * j + 2] = __float_as_uint(f.z);
            r[4 * j + 3] = __float_as_uint(f.w);
          }
          tmem_st16(tmem + lane_off + TM::S + c0, *reinterpret_cast<const uint32_t(*)[16]>(r));
          tmem_st16(tmem + lane_off + TM::S + c0 + 16,
                    *reinterpret_cast<const uint32_t(*)[16]>(r + 16));
          store_S32(r, c0);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(&bar.s_ready);
      // after each chunk but the last: S_<c+1 -> the S operand of the next chunk
      for (int c = 0; c < I.nchunks; ++c, ++g) {
        if (c + 1 == I.nchunks) continue;
        if (wait(&bar.s_full, g & 1)) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < DV; c0 += 32) {
            uint32_t r[32];
            tmem_ld16_async(tmem + lane_off + TM::S + c0, r);
            tmem_ld16_async(tmem + lane_off + TM::S + c0 + 16, r + 16);
            tmem_ld_wait();
            tmem_reg_fence<32>(r);
            store_S32(r, c0);
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&bar.s_ready);
      }
    }
  } else {
    // ================================================================ scores and output
    // Thread = row i of the chunk (tensor-memory lane i).  P(c): mask keys j > i, round to
    // bf16 in place (packed two per column), row sum; den = phi(q_i).z_<c + row sum.  O(c) /
    // den -> bf16 row of the output (32-byte stores; rows past the item's end not written).
    const int sp = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const int i = 32 * sp + lane;
    WarpWaiter wait{abort, err, lane};

    auto convert_P = [&](int gg) -> float {
      const int s = gg % NS;
      // qz of this stage is complete once the feature-map warps released it
      if (!wait(&bar.ready[s], (gg / NS) & 1) || !wait(&bar.p_full, gg & 1)) return 1.f;
      tc_fence_after();
      const uint32_t tp = tmem + lane_off + TM::P;
      float sum = 0.f;
#pragma unroll
      for (int b = 0; b < 4; ++b) {  // keys [32 b, 32 b + 32) -> packed columns [16 b, 16 b + 16)
        uint32_t w[16];
        if (b <= sp) {  // warp-uniform: later keys are masked for every row of this warp
          uint32_t p[32];
          tmem_ld16_async(tp + 32 * b, p);
          tmem_ld16_async(tp + 32 * b + 16, p + 16);
          tmem_ld_wait();
          tmem_reg_fence<32>(p);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int j = 32 * b + 2 * e;
            const float x0 = j <= i ? __uint_as_float(p[2 * e]) : 0.f;
            const float x1 = j + 1 <= i ? __uint_as_float(p[2 * e + 1]) : 0.f;
            sum += x0 + x1;
            w[e] = pack_bf16x2(x0, x1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = 0u;
        }
        tmem_st16(tp + 16 * b, *reinterpret_cast<const uint32_t(*)[16]>(w));
      }
      tmem_st_wait();
      const float d = qz[s * C + i] + sum;
      tc_fence_before();
      mbar_arrive(&bar.p_ready);
      return d;
    };

    auto emit_O = [&](int gg, const Item &I, int c, float den) {
      const int ob = gg & 1;
      const uint32_t tO = tmem + lane_off + (ob ? TM::O1 : TM::O0);
      if (!wait(&bar.o_full[ob], (gg >> 1) & 1)) return;
      tc_fence_after();
      const float inv = 1.f / den;
      const int64_t t = I.t_begin + (int64_t)c * C + i;
      const bool live = t < I.t_end;
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
            st_global_32B(orow + c0 + 16 * q, pack8(f), pack8(f + 8), a32);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.o_empty[ob]);
    };

    int g = 0;
    Item prev{};
    int prev_c = 0;
    float prev_den = 1.f;
    for (int64_t it = it0; it < nitems; it += istep) {
      const Item I = item_at<C>(it, n, seg_len, nseg);
      for (int c = 0; c < I.nchunks; ++c, ++g) {
        if (g >= 1) emit_O(g - 1, prev, prev_c, prev_den);
        prev_den = convert_P(g);
        prev = I;
        prev_c = c;
      }
    }
    if (g > 0) emit_O(g - 1, prev, prev_c, prev_den);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMMA) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

namespace {

template <int DK, int DV>
cudaError_t launch_causal(const void *q, const void *k, const void *v, void *out, int64_t heads,
                          int64_t n, int64_t seg, const float *prefix, int *err,
                          cudaStream_t st) {
  using G = Cfg<DK, DV>;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_tmap_bf16(&tq, q, heads, n, DK, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tk, k, heads, n, DK, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, heads, n, DV, C)) != cudaSuccess) return e;
  auto kern = tc_causal_kernel<DK, DV>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t nseg = (n + seg - 1) / seg;
  const int64_t per = (int64_t)DK * DV + DK;
  const int64_t nitems = heads * nseg;
  // Short items run on persistent CTAs (one per SM, items dealt round-robin), which saves
  // each item the CTA start-up and pipeline fill; long items run one CTA each, so that the
  // hardware's placement of CTAs evens out the SMs' speed differences.
  const int64_t want = seg <= kPersistentTokens ? (int64_t)sm_count() : nitems;
  const unsigned grid = static_cast<unsigned>(nitems < want ? nitems : want);
  // follows the scan: launched so that its set-up and first loads overlap the scan's tail
  e = launch_programmatic(kern, dim3(grid), dim3(kThreads), G::SMEM, st, tq, tk, tv,
                          static_cast<__nv_bfloat16 *>(out), prefix, nseg * per, per, n, seg,
                          nseg, nitems, err);
  if (e != cudaSuccess) return e;
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t tc_causal_features(const void *q, const void *k, const void *v, void *out,
                               int64_t heads, int64_t n, int dk, int dv, int64_t seg,
                               const float *prefix, int *err, cudaStream_t st) {
  if (seg % C != 0) return cudaErrorInvalidValue;
  if (dk == 128 && dv == 64)
    return launch_causal<128, 64>(q, k, v, out, heads, n, seg, prefix, err, st);
  if (dk == 64 && dv == 128)
    return launch_causal<64, 128>(q, k, v, out, heads, n, seg, prefix, err, st);
  return cudaErrorInvalidValue;
}

}  // namespace linattn
