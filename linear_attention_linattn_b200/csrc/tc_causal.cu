// Causal outputs of the bf16-I/O forward pass on the tensor cores, in chunks of 128 tokens.
//
// The method (page "Efficient Transformers: Linear Attention and Flash Attention", sections
// "Linear attention: reordering the matmuls, not shrinking them" and "The recurrent view:
// attention as an RNN"): out_i = phi(q_i) S_i / phi(q_i).z_i with S_i = sum_{j<=i} phi(k_j) v_j^T
// and z_i = sum_{j<=i} phi(k_j).  A work item is one segment of one head; it starts from the
// exclusive prefix state (S_<s, z_<s) of the earlier segments and walks its chunks of C = 128
// tokens with the running state:
//     num_c = phi(Q_c) S_<c + mask(phi(Q_c) phi(K_c)^T) V_c
//     den_c = phi(Q_c).z_<c + mask(phi(Q_c) phi(K_c)^T) 1
//     S_<c+1 = S_<c + phi(K_c)^T V_c,   z_<c+1 = z_<c + phi(K_c)^T 1
// where mask keeps the keys j <= i (the current token included).
//
// Where the prefix comes from:
//   three-kernel pass   the segment aggregates (tc_forward.cu) and their exclusive scan
//                       (simt_forward.cu) are computed first; this kernel reads the prefix.
//   single pass (FUSED) each item first streams its own K, V and forms its aggregate A_s in
//                       tensor memory, publishes it, then looks back over the items before it
//                       in its head: an item that has published its inclusive state I_j ends
//                       the walk, one that has only published A_j adds it and the walk goes on
//                       (a decoupled look-back).  The item publishes I_s = P_s + A_s and runs its
//                       outputs from P_s, re-reading its K, V (from L2: items are dealt so that
//                       the K, V a CTA just read are still there).  K and V cross HBM once.
//                       Items are ordered segment-major, so every item an item waits for has a
//                       smaller index; all CTAs are resident (cooperative launch), so the
//                       smallest unfinished item can always proceed.
//
// Tensor-core products of one chunk (tcgen05.mma kind::f16: bf16 operands, fp32 accumulators in
// tensor memory; every product has M = 128 rows except the state update at DK = 64):
//   P   = phi(Q_c) phi(K_c)^T   M=128 N=128 K=DK   A: Q, B: K (both K-major, shared memory)
//   O   = phi(Q_c) S_<c         M=128 N=DV  K=DK   B: the bf16 copy of S_<c (MN-major)
//   S  += phi(K_c)^T V_c        M=DK  N=DV  K=128  A: K (MN-major), B: V (MN-major)
//   O  += mask(P) V_c           M=128 N=DV  K=128  A: the masked bf16 scores, in tensor memory
// DK/8 + 16 instructions per 128 tokens.  The scores never go through shared memory: the score
// warps mask and round them in place (fp32 columns 0..127 become packed bf16 columns 0..63),
// and the P V product reads them from tensor memory.  The normaliser z is summed on the CUDA
// cores: the feature-map warps, which touch every phi(k), add up its columns (z_<c+1), and
// take phi(q_i).z_<c while they apply phi to q_i.
//
// DK is the feature dimension of phi(q), phi(k) (the head dimension for phi = elu + 1, m for
// random features), DV the value dimension; each 64 or 128.
//
// Warp roles (22 warps, one CTA per SM):
//   warp 0       TMA producer: Q, K, V tiles of a chunk (64-column boxes, 128-byte swizzle)
//                into a ring of stages; no multicast.
//   warp 1       tensor-memory allocation and the single thread that issues every MMA.
//   warps 2-9    feature map: phi in place on the Q and K tiles (packed bf16), K rows past the
//                item's end zeroed; phi(q_i).z_<c per row; column sums of phi(K) into z.
//   warps 10-13  state: each item's starting state into tensor memory and the bf16 S operand
//                (single pass: its aggregate published, the look-back, its inclusive state);
//                after each chunk's update, S_<c+1 rounded into that operand.
//   warps 14-17  scores: mask and round P in tensor memory, the row sums and denominators.
//   warps 18-21  output: O / den -> bf16 rows, stored straight to global memory (32-byte
//                stores).  Separate from the score warps, so that rounding the next chunk's
//                scores never waits behind the previous chunk's stores.
// Every wait is bounded (2 s); a wait that gives up records LINATTN_ERR_TIMEOUT and the CTA
// drains its copies and products and exits without trapping.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace linattn {
namespace {

using namespace tc;

constexpr int C = kTcCausalChunk;  // tokens per chunk (128)
constexpr int kAtom = C * 128;     // one [128 rows][64 bf16] 128B-swizzled atom: 16 KB

constexpr int kWarpTMA = 0;
constexpr int kWarpMMA = 1;
constexpr int kWarpPhi0 = 2;
constexpr int kPhiWarps = 8;
constexpr int kPhiThreads = kPhiWarps * 32;
constexpr int kWarpState0 = kWarpPhi0 + kPhiWarps;  // 10
constexpr int kWarpConv0 = kWarpState0 + 4;         // 14
constexpr int kWarpEmit0 = kWarpConv0 + 4;          // 18
constexpr int kThreads = (kWarpEmit0 + 4) * 32;     // 704
constexpr int kZBufs = 3;  // column-sum buffers of the feature-map warps, by chunk mod 3
// items of at most this many tokens run on persistent CTAs
constexpr int64_t kPersistentTokens = 2048;

// Shared memory of a CTA: NS stages (Q, K, V tiles of one chunk), the bf16 S operand, the
// column-sum buffers, phi(q).z per stage, and the barriers.
// the barrier block: 3 per stage and 14 more mbarriers, then four 32-bit words; 64-byte units
constexpr int bar_bytes(int ns) { return ((3 * ns + 14) * 8 + 16 + 63) / 64 * 64; }
template <int DK, int DV>
constexpr int smem_bytes(int ns) {
  return ns * (2 * (DK / 64) + DV / 64) * kAtom + (DV / 64) * DK * 128 + kZBufs * DK * 4 +
         ns * C * 4 + bar_bytes(ns);
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
  static constexpr int SMEM = OFF_BAR + bar_bytes(NS);
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
  // the denominators of an output chunk, by O buffer (score group -> output group)
  uint64_t den_ready[2];
  // single pass: the item's z aggregate written (feature map -> state group); its inclusive
  // state written (state group -> feature map)
  uint64_t zpub, zready;
  uint32_t tmem_base;
  int abort;
  int flag;  // single pass: the look-back's current flag, shared by the state group
};

// Arguments of the causal kernel.  Three-kernel pass: prefix[item] is the state before the
// item, at prefix + head * prefix_head_stride + seg * prefix_seg_stride ([DK][DV] then [DK]).
// Single pass: agg and incl [heads][nseg][DK*DV + DK] receive each item's aggregate and
// inclusive state, flags [heads][nseg] (zero at launch) their publication (1: aggregate,
// 2: inclusive); init_S [heads][DK][DV] / init_z [heads][DK] (nullable) is the state before
// each head's first token.
struct CausalArgs {
  __nv_bfloat16 *out;
  const float *prefix;
  int64_t prefix_head_stride, prefix_seg_stride;
  float *agg, *incl;
  int *flags;
  const float *init_S, *init_z;
  int64_t n, seg_len, nseg, heads, nitems;
  int *err;
};

// Item it: head-major in the three-kernel pass, segment-major in the single pass (so that the
// items a look-back waits for always have smaller indices).
template <bool FUSED>
__device__ __forceinline__ Item causal_item(int64_t it, const CausalArgs &a) {
  const int64_t head = FUSED ? it % a.heads : it / a.nseg;
  const int64_t seg = FUSED ? it / a.heads : it % a.nseg;
  return item_at<C>(head * a.nseg + seg, a.n, a.seg_len, a.nseg);
}

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
// role walks the same sequence of chunks, and g counts them across items (in the single pass,
// an item's aggregate chunks and then its output chunks), so the stage ring and the barrier
// phases run on from one item into the next.
// PHI: apply phi = elu + 1 to Q and K; false takes them as given non-negative features.
// FUSED: the single pass (the item's aggregate, publication and look-back in this kernel).
template <int DK, int DV, bool PHI, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
    tc_causal_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CausalArgs A) {
  using G = Cfg<DK, DV>;
  using TM = TmemMap<DV>;
  constexpr int NS = G::NS;
  constexpr int KSD = DK / 16;  // K-steps over the feature dimension
  constexpr int KSC = C / 16;   // K-steps over the chunk's tokens
  constexpr int64_t PER = (int64_t)DK * DV + DK;  // floats of one state
  static_assert(sizeof(Bars<NS>) <= bar_bytes(NS), "barrier block");
  extern __shared__ __align__(1024) uint8_t smem[];
  int *err = A.err;
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
  const int lane = threadIdx.x & 31;
  const int64_t it0 = blockIdx.x, istep = gridDim.x;
  const int64_t nitems = A.nitems;
  // chunks an item streams: its aggregate chunks (single pass), then its output chunks
  auto chunks_before_out = [](const Item &I) { return FUSED ? I.nchunks : 0; };

  // ---- set-up: barriers, the column-sum buffers, tensor memory
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.ready[s], kPhiThreads);
      // the MMA commit after the chunk's last product, and the output group once it has read
      // the chunk's denominators (which sit in the stage's phi(q).z slot)
      mbar_init(&bar.empty[s], 1 + 128);
    }
    mbar_init(&bar.p_full, 1);
    mbar_init(&bar.p_ready, 128);
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.s_ready, 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.o_full[b], 1);
      mbar_init(&bar.o_empty[b], 128);
      mbar_init(&bar.den_ready[b], 128);
    }
    mbar_init(&bar.zsync, kPhiThreads);
    mbar_init(&bar.fin, 1);
    mbar_init(&bar.zpub, kPhiThreads);
    mbar_init(&bar.zready, 128);
    bar.abort = 0;
    bar.flag = 0;
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
      // single pass: an item's first read of K, V is kept in L2 for its output chunks
      const uint64_t pol_keep = policy_evict_last();
      const uint64_t pol = policy_evict_first();
      int g = 0;  // chunks issued
      bool ok = true;
      for (int64_t it = it0; ok && it < nitems; it += istep) {
        const Item I = causal_item<FUSED>(it, A);
        const int zc = static_cast<int>(I.head);
        const int na = chunks_before_out(I);
        for (int c = 0; ok && c < na + I.nchunks; ++c, ++g) {
          const int s = g % NS;
          if (g >= NS && !mbar_wait(&bar.empty[s], ((g / NS) - 1) & 1, abort, err)) {
            ok = false;
            break;
          }
          const bool agg = c < na;  // an aggregate chunk: K and V only
          uint8_t *st = smem + s * G::STAGE;
          const int y = static_cast<int>(I.t_begin + (int64_t)(agg ? c : c - na) * C);
          mbar_arrive_expect_tx(&bar.full[s], agg ? G::STAGE - G::QTILE : G::STAGE);
#pragma unroll
          for (int a = 0; a < G::AK; ++a) {
            if (!agg) tma_load_3d(st + a * kAtom, &tmQ, &bar.full[s], a * 64, y, zc, pol);
            tma_load_3d(st + G::OFF_K + a * kAtom, &tmK, &bar.full[s], a * 64, y, zc,
                        agg ? pol_keep : pol);
          }
#pragma unroll
          for (int a = 0; a < G::AV; ++a)
            tma_load_3d(st + G::OFF_V + a * kAtom, &tmV, &bar.full[s], a * 64, y, zc,
                        agg ? pol_keep : pol);
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
      int g = 0;   // chunks (the stage ring)
      int go = 0;  // output chunks
      bool ok = true;
      for (int64_t it = it0; ok && it < nitems; it += istep) {
        const Item I = causal_item<FUSED>(it, A);
        // single pass: the item's aggregate A_s = phi(K)^T V over its chunks, into TMEM S
        for (int c = 0; c < chunks_before_out(I); ++c, ++g) {
          const int s = g % NS;
          if (!mbar_wait(&bar.ready[s], (g / NS) & 1, abort, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = st0 + s * G::STAGE;
          const uint64_t dKm = mnmajor_base(st + G::OFF_K, kAtom);
          const uint64_t dVm = mnmajor_base(st + G::OFF_V, kAtom);
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tS, desc_add(dKm, mnmajor_off(ks)), desc_add(dVm, mnmajor_off(ks)), I_S,
                        (c > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&bar.empty[s]);
          mbar_arrive_cnt(&bar.empty[s], 128);  // no output group reads this stage
        }
        if (!ok) break;
        if (FUSED) mma_commit(&bar.s_full);  // the aggregate is complete
        for (int c = 0; c < I.nchunks; ++c, ++g, ++go) {
          const int s = g % NS;
          const bool last = c + 1 == I.nchunks;
          // this chunk's tiles transformed; S_<c in the S operand and TMEM S free to update;
          // this O buffer emitted (output chunk go - 2)
          if (!mbar_wait(&bar.ready[s], (g / NS) & 1, abort, err) ||
              !mbar_wait(&bar.s_ready, go & 1, abort, err) ||
              (go >= 2 && !mbar_wait(&bar.o_empty[go & 1], ((go >> 1) - 1) & 1, abort, err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = st0 + s * G::STAGE;
          const uint64_t dQ = kmajor_base(st);
          const uint64_t dK = kmajor_base(st + G::OFF_K);
          const uint64_t dKm = mnmajor_base(st + G::OFF_K, kAtom);
          const uint64_t dVm = mnmajor_base(st + G::OFF_V, kAtom);
          const uint32_t tO = tmem + ((go & 1) ? TM::O1 : TM::O0);
          // Three independent accumulators, issued K-step by K-step so that the tensor pipe
          // overlaps them: the scores and phi(Q_c) S_<c (sharing the A operand), and
          // S += phi(K_c)^T V_c (not after the item's last chunk: nothing reads it).
#pragma unroll
          for (int ks = 0; ks < (KSD > KSC ? KSD : KSC); ++ks) {
            if (ks < KSD) {
              const uint64_t a = desc_add(dQ, kmajor_off(ks, kAtom));
              mma_bf16_ss(tP, a, desc_add(dK, kmajor_off(ks, kAtom)), I_P, ks > 0 ? 1u : 0u);
              mma_bf16_ss(tO, a, desc_add(dS, mnmajor_off(ks)), I_O, ks > 0 ? 1u : 0u);
            }
            if (!last && ks < KSC)
              mma_bf16_ss(tS, desc_add(dKm, mnmajor_off(ks)), desc_add(dVm, mnmajor_off(ks)), I_S,
                          1u);
          }
          mma_commit(&bar.p_full);
          // the state group waits for this after every chunk but the last (single pass), or
          // after every chunk (three-kernel pass: the next item's start state follows it)
          if (!FUSED || !last) mma_commit(&bar.s_full);
          // O += mask(P) V_c, the rounded scores read from tensor memory
          if (!mbar_wait(&bar.p_ready, go & 1, abort, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ts(tO, tP + 8 * ks, desc_add(dVm, mnmajor_off(ks)), I_PV, 1u);
          mma_commit(&bar.o_full[go & 1]);
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
    // is r0 & 7 for all four rows).  It keeps z for its columns in registers: z_<c of the
    // output chunks, and in the single pass first the item's aggregate.
    const int t = threadIdx.x - kWarpPhi0 * 32;
    const int r0 = t >> 3;
    const int cg = (t & 7) ^ (r0 & 7);
    const int vec_off = r0 * 128 + (t & 7) * 16;  // byte offset of row r0's vector in an atom
    WarpWaiter wait{abort, err, lane};
    float zr[G::AK][8];
    auto load_z = [&](const float *src) {  // src: the z part of a state
#pragma unroll
      for (int a = 0; a < G::AK; ++a) {
        const float4 lo = __ldcg(reinterpret_cast<const float4 *>(src + a * 64 + cg * 8));
        const float4 hi = __ldcg(reinterpret_cast<const float4 *>(src + a * 64 + cg * 8 + 4));
        zr[a][0] = lo.x; zr[a][1] = lo.y; zr[a][2] = lo.z; zr[a][3] = lo.w;
        zr[a][4] = hi.x; zr[a][5] = hi.y; zr[a][6] = hi.z; zr[a][7] = hi.w;
      }
    };
    int g = 0;
    int j = 0;  // items of this CTA
    for (int64_t it = it0; it < nitems; it += istep, ++j) {
      const Item I = causal_item<FUSED>(it, A);
      const int64_t slot = I.head * A.nseg + I.seg;
      const int na = chunks_before_out(I);
      if (FUSED) {
#pragma unroll
        for (int a = 0; a < G::AK; ++a)
#pragma unroll
          for (int e = 0; e < 8; ++e) zr[a][e] = 0.f;
      } else {
        load_z(A.prefix + I.head * A.prefix_head_stride + I.seg * A.prefix_seg_stride +
               (int64_t)DK * DV);
      }
      for (int c = 0; c < na + I.nchunks; ++c, ++g) {
        const int s = g % NS;
        const bool agg = c < na;
        float *zbuf = zacc + (g % kZBufs) * DK;
        if (wait(&bar.full[s], (g / NS) & 1)) {
          uint8_t *st = smem + s * G::STAGE;
          const int64_t left = I.t_end - (I.t_begin + (int64_t)(agg ? c : c - na) * C);
          const int valid = left < C ? static_cast<int>(left) : C;
          // K: phi in place, rows past the item's end zeroed; column sums of phi(K)
          float cs[G::AK][8];
#pragma unroll
          for (int a = 0; a < G::AK; ++a)
#pragma unroll
            for (int e = 0; e < 8; ++e) cs[a][e] = 0.f;
#pragma unroll
          for (int k = 0; k < 4 * G::AK; ++k) {
            const int a = k >> 2, m = k & 3;
            uint4 *p = reinterpret_cast<uint4 *>(st + G::OFF_K + a * kAtom + vec_off + m * 4096);
            uint4 x = make_uint4(0u, 0u, 0u, 0u);
            if (r0 + 32 * m < valid) {
              x = *p;
              if (PHI) x = phi_bf16x8(x);
            }
            *p = x;
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              cs[a][2 * e] += bf16_lo(w[e]);
              cs[a][2 * e + 1] += bf16_hi(w[e]);
            }
          }
          if (!agg) {
            // Q: phi in place; phi(q_i).z_<c for rows r0 + 32 m (this thread's columns)
            float qp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 4 * G::AK; ++k) {
              const int a = k >> 2, m = k & 3;
              uint4 *p = reinterpret_cast<uint4 *>(st + a * kAtom + vec_off + m * 4096);
              uint4 x = *p;
              if (PHI) {
                x = phi_bf16x8(x);
                *p = x;
              }
              const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                qp[m] += bf16_lo(w[e]) * zr[a][2 * e] + bf16_hi(w[e]) * zr[a][2 * e + 1];
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
        // every warp's column sums are in: z += phi(K_c)^T 1
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
        if (FUSED && c + 1 == na) {
          // the item's aggregate z -> its published state (threads 0..7 hold every column
          // group); then z_<s of its output chunks = its inclusive z - its aggregate z
          if (t < 8) {
            float *dst = A.agg + slot * PER + (int64_t)DK * DV;
#pragma unroll
            for (int a = 0; a < G::AK; ++a) {
              *reinterpret_cast<float4 *>(dst + a * 64 + cg * 8) =
                  make_float4(zr[a][0], zr[a][1], zr[a][2], zr[a][3]);
              *reinterpret_cast<float4 *>(dst + a * 64 + cg * 8 + 4) =
                  make_float4(zr[a][4], zr[a][5], zr[a][6], zr[a][7]);
            }
            __threadfence();
          }
          mbar_arrive(&bar.zpub);
          if (wait(&bar.zready, j & 1)) {
            const float *inc = A.incl + slot * PER + (int64_t)DK * DV;
#pragma unroll
            for (int a = 0; a < G::AK; ++a) {
              const float4 lo = __ldcg(reinterpret_cast<const float4 *>(inc + a * 64 + cg * 8));
              const float4 hi = __ldcg(reinterpret_cast<const float4 *>(inc + a * 64 + cg * 8 + 4));
              zr[a][0] = lo.x - zr[a][0]; zr[a][1] = lo.y - zr[a][1];
              zr[a][2] = lo.z - zr[a][2]; zr[a][3] = lo.w - zr[a][3];
              zr[a][4] = hi.x - zr[a][4]; zr[a][5] = hi.y - zr[a][5];
              zr[a][6] = hi.z - zr[a][6]; zr[a][7] = hi.w - zr[a][7];
            }
          }
        }
      }
    }
  } else if (warp < kWarpConv0) {
    // ================================================================ state group
    // Row rS of the S accumulator (M = DK: lanes 0..127 at DK = 128; at DK = 64 the M = 64
    // layout puts rows 16 sp .. 16 sp + 15 in lanes 0..15 of sub-partition sp).
    const int sp = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const int rS = DK == 128 ? 32 * sp + lane : 16 * sp + lane;
    const bool vS = DK == 128 || lane < 16;
    const uint32_t tSrow = tmem + lane_off + TM::S;
    const int st_tid = threadIdx.x - kWarpState0 * 32;  // 0..127
    uint8_t *sS = smem + G::OFF_S;
    WarpWaiter wait{abort, err, lane};
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
    // TMEM S row rS (+)= src row rS (src: a [DK][DV] fp32 state in global memory, or null for
    // zero), 32 columns at a time; with to_operand, the result also into the S operand
    auto tmem_row_add = [&](const float *src, bool overwrite, bool to_operand) {
#pragma unroll 1
      for (int c0 = 0; c0 < DV; c0 += 32) {
        uint32_t r[32];
        if (!overwrite) {
          tmem_ld16_async(tSrow + c0, r);
          tmem_ld16_async(tSrow + c0 + 16, r + 16);
          tmem_ld_wait();
          tmem_reg_fence<32>(r);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        if (src && vS) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 f = __ldcg(reinterpret_cast<const float4 *>(src + (int64_t)rS * DV + c0 + e));
            r[e] = __float_as_uint(__uint_as_float(r[e]) + f.x);
            r[e + 1] = __float_as_uint(__uint_as_float(r[e + 1]) + f.y);
            r[e + 2] = __float_as_uint(__uint_as_float(r[e + 2]) + f.z);
            r[e + 3] = __float_as_uint(__uint_as_float(r[e + 3]) + f.w);
          }
        }
        tmem_st16(tSrow + c0, *reinterpret_cast<const uint32_t(*)[16]>(r));
        tmem_st16(tSrow + c0 + 16, *reinterpret_cast<const uint32_t(*)[16]>(r + 16));
        if (to_operand) store_S32(r, c0);
      }
      tmem_st_wait();
    };
    int g = 0;  // chunks ahead of the current item's output chunks whose s_full was waited
    int gs = 0;  // phases of s_full waited
    int j = 0;
    for (int64_t it = it0; it < nitems; it += istep, ++j) {
      const Item I = causal_item<FUSED>(it, A);
      if (FUSED) {
        // ---- the item's aggregate A_s: TMEM S -> agg (its z: the feature-map warps)
        const int64_t slot = I.head * A.nseg + I.seg;
        float *aggS = A.agg + slot * PER;
        if (wait(&bar.s_full, gs & 1)) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < DV; c0 += 32) {
            uint32_t r[32];
            tmem_ld16_async(tSrow + c0, r);
            tmem_ld16_async(tSrow + c0 + 16, r + 16);
            tmem_ld_wait();
            tmem_reg_fence<32>(r);
            if (vS) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4 *>(aggS + (int64_t)rS * DV + c0 + e) =
                    make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
            }
          }
        }
        ++gs;
        wait(&bar.zpub, j & 1);
        __threadfence();
        named_barrier_sync(1, 128);
        if (st_tid == 0) st_release_gpu(A.flags + slot, 1);
        // ---- look back: P = the sum of the earlier items' states, up to an inclusive one
        float pz = 0.f;  // z_<s of row rS
        bool first = true;
        for (int64_t sj = I.seg - 1;; --sj) {
          if (sj < 0) {  // the start of the head: the caller's initial state, if any
            if (A.init_S) {
              tmem_row_add(A.init_S + I.head * (int64_t)DK * DV, first, false);
              if (vS) pz += __ldcg(A.init_z + I.head * DK + rS);
              first = false;
            }
            break;
          }
          const int64_t pslot = I.head * A.nseg + sj;
          if (st_tid == 0) bar.flag = spin_flag(A.flags + pslot, abort, err);
          named_barrier_sync(1, 128);
          const int f = bar.flag;
          named_barrier_sync(1, 128);  // everyone has read the flag before the next spin
          if (f == 0) break;           // gave up (recorded): nothing more to wait for
          const float *src = (f == 2 ? A.incl : A.agg) + pslot * PER;
          tmem_row_add(src, first, false);
          if (vS) pz += __ldcg(src + (int64_t)DK * DV + rS);
          first = false;
          if (f == 2) break;
        }
        if (first) tmem_row_add(nullptr, true, false);  // P = 0
        // ---- the inclusive state I_s = P + A_s -> incl; P -> the S operand
        float *inclS = A.incl + slot * PER;
#pragma unroll 1
        for (int c0 = 0; c0 < DV; c0 += 32) {
          uint32_t r[32];
          tmem_ld16_async(tSrow + c0, r);
          tmem_ld16_async(tSrow + c0 + 16, r + 16);
          tmem_ld_wait();
          tmem_reg_fence<32>(r);
          if (vS) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 a4 = *reinterpret_cast<const float4 *>(aggS + (int64_t)rS * DV + c0 + e);
              *reinterpret_cast<float4 *>(inclS + (int64_t)rS * DV + c0 + e) =
                  make_float4(__uint_as_float(r[e]) + a4.x, __uint_as_float(r[e + 1]) + a4.y,
                              __uint_as_float(r[e + 2]) + a4.z, __uint_as_float(r[e + 3]) + a4.w);
            }
          }
          store_S32(r, c0);
        }
        if (vS)
          inclS[(int64_t)DK * DV + rS] = pz + __ldcg(aggS + (int64_t)DK * DV + rS);
        __threadfence();
        named_barrier_sync(1, 128);
        if (st_tid == 0) st_release_gpu(A.flags + slot, 2);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar.zready);
        mbar_arrive(&bar.s_ready);
      } else {
        // ---- the item's starting state, once the previous item's last products are done
        // with TMEM S and the S operand
        if (g == 0 || wait(&bar.s_full, gs & 1)) {
          tc_fence_after();
          tmem_row_add(A.prefix + I.head * A.prefix_head_stride + I.seg * A.prefix_seg_stride,
                       true, true);
          fence_proxy_async_smem();
        }
        if (g > 0) ++gs;
        tc_fence_before();
        mbar_arrive(&bar.s_ready);
      }
      // after each output chunk but the last: S_<c+1 -> the S operand of the next chunk
      for (int c = 0; c < I.nchunks; ++c, ++g) {
        if (c + 1 == I.nchunks) continue;
        if (wait(&bar.s_full, gs & 1)) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < DV; c0 += 32) {
            uint32_t r[32];
            tmem_ld16_async(tSrow + c0, r);
            tmem_ld16_async(tSrow + c0 + 16, r + 16);
            tmem_ld_wait();
            tmem_reg_fence<32>(r);
            store_S32(r, c0);
          }
          fence_proxy_async_smem();
        }
        ++gs;
        tc_fence_before();
        mbar_arrive(&bar.s_ready);
      }
    }
  } else if (warp < kWarpEmit0) {
    // ================================================================ scores
    // Thread = row i of the chunk (tensor-memory lane i).  P(c): mask keys j > i, round to
    // bf16 in place (packed two per column), row sum; den = phi(q_i).z_<c + row sum, written
    // over phi(q_i).z_<c in the stage's slot for the output group.
    const int sp = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const int i = 32 * sp + lane;
    const uint32_t tp = tmem + lane_off + TM::P;
    WarpWaiter wait{abort, err, lane};
    int g = 0, go = 0;
    for (int64_t it = it0; it < nitems; it += istep) {
      const Item I = causal_item<FUSED>(it, A);
      g += chunks_before_out(I);
      for (int c = 0; c < I.nchunks; ++c, ++g, ++go) {
        const int s = g % NS;
        // phi(q).z of this stage is complete once the feature-map warps released it
        if (!wait(&bar.ready[s], (g / NS) & 1) || !wait(&bar.p_full, go & 1)) continue;
        tc_fence_after();
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
              const int jj = 32 * b + 2 * e;
              const float x0 = jj <= i ? __uint_as_float(p[2 * e]) : 0.f;
              const float x1 = jj + 1 <= i ? __uint_as_float(p[2 * e + 1]) : 0.f;
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
        qz[s * C + i] += sum;
        tc_fence_before();
        mbar_arrive(&bar.p_ready);
        mbar_arrive(&bar.den_ready[go & 1]);
      }
    }
  } else {
    // ================================================================ output
    // Thread = row i of the chunk.  O(c) / den -> bf16 row of the output (32-byte stores; rows
    // past the item's end not written).
    const int sp = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const int i = 32 * sp + lane;
    WarpWaiter wait{abort, err, lane};
    int g = 0, go = 0;
    for (int64_t it = it0; it < nitems; it += istep) {
      const Item I = causal_item<FUSED>(it, A);
      g += chunks_before_out(I);
      for (int c = 0; c < I.nchunks; ++c, ++g, ++go) {
        const int s = g % NS, ob = go & 1;
        if (!wait(&bar.o_full[ob], (go >> 1) & 1) || !wait(&bar.den_ready[ob], (go >> 1) & 1))
          continue;
        tc_fence_after();
        const float inv = 1.f / qz[s * C + i];
        mbar_arrive(&bar.empty[s]);  // the stage's last reader
        const uint32_t tO = tmem + lane_off + (ob ? TM::O1 : TM::O0);
        const int64_t t = I.t_begin + (int64_t)c * C + i;
        const bool live = t < I.t_end;
        __nv_bfloat16 *orow = A.out + (I.head * A.n + (live ? t : 0)) * DV;
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

}  // namespace

namespace {

template <int DK, int DV, bool PHI, bool FUSED>
cudaError_t launch_causal(const void *q, const void *k, const void *v, const CausalArgs &args,
                          cudaStream_t st) {
  using G = Cfg<DK, DV>;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  const int64_t heads = args.heads, n = args.n;
  if ((e = make_tmap_bf16(&tq, q, heads, n, DK, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tk, k, heads, n, DK, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, heads, n, DV, C)) != cudaSuccess) return e;
  auto kern = tc_causal_kernel<DK, DV, PHI, FUSED>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t sms = sm_count();
  if (!FUSED) {
    // Short items run on persistent CTAs (one per SM, items dealt round-robin), which saves
    // each item the CTA start-up and pipeline fill; long items run one CTA each, so that the
    // hardware's placement of CTAs evens out the SMs' speed differences.
    const int64_t want = args.seg_len <= kPersistentTokens ? sms : args.nitems;
    const unsigned grid = static_cast<unsigned>(args.nitems < want ? args.nitems : want);
    kern<<<grid, kThreads, G::SMEM, st>>>(tq, tk, tv, args);
  } else {
    // Single pass: persistent CTAs, all resident at once (a cooperative launch), since an
    // item's look-back waits for items that other CTAs hold.  The publication flags start at 0.
    e = cudaMemsetAsync(args.flags, 0, (size_t)args.nitems * sizeof(int), st);
    if (e != cudaSuccess) return e;
    count_launches(1);
    record_launch_event(st);
    const unsigned grid = static_cast<unsigned>(args.nitems < sms ? args.nitems : sms);
    void *params[] = {const_cast<CUtensorMap *>(&tq), const_cast<CUtensorMap *>(&tk),
                      const_cast<CUtensorMap *>(&tv), const_cast<CausalArgs *>(&args)};
    e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), dim3(grid),
                                    dim3(kThreads), params, G::SMEM, st);
    if (e != cudaSuccess) return e;
  }
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

template <bool FUSED>
cudaError_t causal_dispatch(const void *q, const void *k, const void *v, int dk, int dv,
                            int features, const CausalArgs &args, cudaStream_t st) {
  // phi = elu + 1 keeps the dimension (dk = dv); random features may change it
  if (!features) {
    if (dk == 64 && dv == 64) return launch_causal<64, 64, true, FUSED>(q, k, v, args, st);
    if (dk == 128 && dv == 128) return launch_causal<128, 128, true, FUSED>(q, k, v, args, st);
    return cudaErrorInvalidValue;
  }
  if (dk == 64 && dv == 64) return launch_causal<64, 64, false, FUSED>(q, k, v, args, st);
  if (dk == 128 && dv == 128) return launch_causal<128, 128, false, FUSED>(q, k, v, args, st);
  if (dk == 128 && dv == 64) return launch_causal<128, 64, false, FUSED>(q, k, v, args, st);
  if (dk == 64 && dv == 128) return launch_causal<64, 128, false, FUSED>(q, k, v, args, st);
  return cudaErrorInvalidValue;
}

CausalArgs base_args(void *out, int64_t heads, int64_t n, int64_t seg, int *err) {
  CausalArgs a{};
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.n = n;
  a.seg_len = seg;
  a.nseg = (n + seg - 1) / seg;
  a.heads = heads;
  a.nitems = heads * a.nseg;
  a.err = err;
  return a;
}

}  // namespace

cudaError_t tc_causal_out(const void *q, const void *k, const void *v, void *out, int64_t heads,
                          int64_t n, int dk, int dv, int64_t seg, const float *prefix,
                          int features, int *err, cudaStream_t st) {
  if (seg % C != 0) return cudaErrorInvalidValue;
  CausalArgs a = base_args(out, heads, n, seg, err);
  const int64_t per = (int64_t)dk * dv + dk;
  a.prefix = prefix;
  a.prefix_head_stride = a.nseg * per;
  a.prefix_seg_stride = per;
  return causal_dispatch<false>(q, k, v, dk, dv, features, a, st);
}

int64_t tc_fused_segment(int64_t heads, int64_t n, int dk, int dv) {
  // The K, V an item reads first should still be in L2 when it reads them again: about
  // 64 MB of them in flight over all SMs (one item per SM).  Then no shorter than 256 tokens
  // (the published states cost 2 (dk dv + dk) floats per item) and no longer than the head.
  const int64_t sms = sm_count();
  int64_t seg = (int64_t(64) << 20) / (sms * (int64_t)(dk + dv) * 2);
  seg = seg / C * C;
  if (seg < 256) seg = 256;
  if (seg > 4096) seg = 4096;
  // enough items for every SM when the heads are few
  while (seg > 256 && heads * ((n + seg - 1) / seg) < sms) seg -= C;
  const int64_t nrounded = (n + C - 1) / C * C;
  return seg > nrounded ? nrounded : seg;
}

size_t tc_fused_workspace_bytes(int64_t heads, int64_t n, int dk, int dv, int64_t seg) {
  const int64_t nitems = heads * ((n + seg - 1) / seg);
  const int64_t per = (int64_t)dk * dv + dk;
  // aggregate and inclusive states, then the flags (16-byte aligned)
  return (size_t)(2 * nitems * per) * sizeof(float) + (size_t)((nitems + 3) / 4 * 4) * sizeof(int);
}

cudaError_t tc_causal_fused(const void *q, const void *k, const void *v, void *out,
                            int64_t heads, int64_t n, int dk, int dv, int64_t seg, void *ws,
                            const float *init_S, const float *init_z, int features, int *err,
                            cudaStream_t st) {
  if (seg % C != 0) return cudaErrorInvalidValue;
  CausalArgs a = base_args(out, heads, n, seg, err);
  const int64_t per = (int64_t)dk * dv + dk;
  a.agg = static_cast<float *>(ws);
  a.incl = a.agg + a.nitems * per;
  a.flags = reinterpret_cast<int *>(a.incl + a.nitems * per);
  a.init_S = init_S;
  a.init_z = init_z;
  return causal_dispatch<true>(q, k, v, dk, dv, features, a, st);
}

}  // namespace linattn
