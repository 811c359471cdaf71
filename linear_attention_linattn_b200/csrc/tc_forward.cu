// bf16-I/O forward pass on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// The method (page "Efficient Transformers: Linear Attention and Flash Attention",
// sections "Linear attention: reordering the matmuls, not shrinking them" and "The
// recurrent view: attention as an RNN"):
//     out_i = phi(q_i) S / phi(q_i).z,  S = sum_j phi(k_j) v_j^T,  z = sum_j phi(k_j)
// with j <= i in the causal mode.  Causal work is split into chunks of C = 64 tokens:
//     num_c = phi(Q_c) S_<c + mask(phi(Q_c) phi(K_c)^T) V_c
//     den_c = phi(Q_c) z_<c + mask(phi(Q_c) phi(K_c)^T) 1
//     S_<c+1 = S_<c + phi(K_c)^T V_c,   z_<c+1 = z_<c + phi(K_c)^T 1
// and chunks are grouped into segments, the work items of the CTAs.  The pass is three
// kernels: K1 the segment aggregates (mode kState), K2 their exclusive prefix or per-head total
// (the scan in simt_forward.cu), K3 the outputs (mode kCausalOut or kNoncausalOut).  On
// caller-given features (FAVOR+) the causal K3 is tc_causal.cu's, which also handles a feature
// dimension DK different from the value dimension DV.
//
// Every product is a tcgen05.mma (kind::f16, bf16 operands, fp32 accumulator in TMEM):
//   [P | phi(Q_c).z_<c] = phi(Q_c) [phi(K_c); z_<c]^T   M=64 N=80     K=D   (causal; A: Q, B: K,
//                          both K-major; the K tile carries 16 more rows, row 64 = z_<c)
//   O  = phi(Q_c) S_<c                                   M=64 N=DV    K=DK  (B: S bf16 MN-major;
//                          non-causal N=DV+16: an extra atom holds z, column DV = denominator)
//   O += mask(P) V_c                                     M=64 N=D     K=64  (A: P bf16 K-major,
//                          B: V MN-major)
//   [S | z] += phi(K_c)^T [V_c | 1]                      M=DK N=DV+16 K=64  (A: K MN-major; a
//                          constant ones atom after each V tile puts z in column DV)
// The causal denominator is column 64 of the score block plus the masked row sum of the
// scores (taken while they are rounded), so numerator and denominator weigh the same keys.
// DK is the feature dimension of phi(q), phi(k), DV the value dimension; the causal mode here
// keeps DK = DV = D.
//
// Warp roles (one CTA per SM; 16 or 15 warps in the causal mode at d = 128 or 64, 22 in the
// aggregate mode, 18 in the non-causal mode):
//   warp 0     TMA producer: 3-D tiled loads (128-byte swizzle) of Q/K/V chunks into a
//              ring of stages; no multicast.
//   warp 1     TMEM allocation and the MMA-issuing thread (warp 2 holds a second one in the
//              causal mode at d = 64).
//   next 4-12  feature map: phi applied in place to the Q and K tiles (bf16), K rows beyond
//              the item's end zeroed, then handed to the tensor cores.
//   next 4     state: round S_<c+1 and z into the next chunk's operands; the starting
//              state; the segment aggregate.
//   last 4     scores and output: mask and round P; divide O by its denominator and
//              store the bf16 rows.  P and S are drained by different warps, so the two
//              conversions on each chunk's critical path run side by side.
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

enum Mode : int { kState = 0, kCausalOut = 1, kNoncausalOut = 2 };

constexpr int kWarpTMA = 0;
constexpr int kWarpMMA = 1;
constexpr int kGroupThreads = 128;
// Warps per mode and feature width (measured on the benchmark shapes).  Causal: 16 or 15
// warps, so each SM sub-partition holds about 4 and a thread may use 128 registers (the score,
// state and output drains keep 64-column batches in registers).  At d = 64 two warps issue the MMAs (one
// thread issues a tcgen05.mma about every 55 cycles, slower than the tensor pipe runs these
// small products; issuers in different warps proceed in parallel), with 4 feature-map warps,
// one per SM sub-partition (0.167 ms with 5, 0.156 with 4, 0.194 with 3 on the batched
// workload); at d = 128 the feature map is the tighter bound, so one issuer and 6 feature-map
// warps (1.00 ms; 1.05 with 4).
// Aggregate: the feature map on K bounds the chunk rate, so 12 feature-map warps (22 warps,
// 80 registers), in two teams of 6 taking alternate stages where the stage count is even (at
// d = 64: 0.069 -> 0.060 ms on the batched workload).  Non-causal: 8 feature-map warps (18
// warps, 96 registers).
template <int MODE, int DK>
struct Warps {
  static constexpr bool TWO_ISSUERS = MODE == kCausalOut && DK == 64;
  static constexpr int MMA2 = 2;                      // the second issuer
  static constexpr int XFORM0 = TWO_ISSUERS ? 3 : 2;  // first feature-map warp
  static constexpr int XFORM =
      MODE == kCausalOut ? (TWO_ISSUERS ? 4 : 6) : (MODE == kState ? 12 : 8);
  static constexpr int XTHREADS = XFORM * 32;
  // feature-map teams wanted: the warps split into groups that take alternate chunks, so
  // several chunks are in flight instead of all warps waiting on one (the kernel keeps one
  // team unless the stage count is a multiple: a team must own whole stages and wait for
  // every phase of their barriers, since a wait may target only the pending phase)
  static constexpr int XTEAMS = MODE == kState ? 2 : 1;
  static_assert(XFORM % XTEAMS == 0, "equal teams");
  static constexpr int STATE0 = XFORM0 + XFORM;  // state group: 4 warps
  static constexpr int OUT0 = STATE0 + 4;             // scores and output group: 4 warps
  static constexpr int THREADS = (OUT0 + 4) * 32;
};
constexpr int kZRows = 16;  // extra key rows carrying z (row 0) in the causal K tile
// causal items of at most this many chunks run on persistent CTAs
constexpr int kPersistentCausalChunks = 32;

template <int DK, int DV, int MODE>
struct Cfg {
  static_assert(MODE != kCausalOut || DK == DV, "the causal mode keeps one dimension");
  static constexpr int AK = DK / 64;        // 64-column atoms per [64][DK] tile (Q, K)
  static constexpr int AV = DV / 64;        // 64-column atoms per [64][DV] tile (V)
  static constexpr bool LQ = MODE != kState;
  static constexpr bool LKV = MODE != kNoncausalOut;
  // causal: each K atom carries 16 more rows after the 64 keys; row 64 holds z_<c, so the
  // score MMA (N = 80) also yields phi(q_i).z_<c in its column 64.
  static constexpr int KROWS = MODE == kCausalOut ? 64 + kZRows : 64;
  static constexpr int KATOM = KROWS * 128;
  // a constant atom after each V tile whose column 0 is 1: the S MMA with N = DV + 16 then
  // also accumulates z = phi(K)^T 1 in its column DV.
  static constexpr int OFF_K = LQ ? AK * kAtom : 0;
  static constexpr int OFF_V = OFF_K + (LKV ? AK * KATOM : 0);
  static constexpr int OFF_ONES = OFF_V + (LKV ? AV * kAtom : 0);
  static constexpr int STAGE = OFF_ONES + (LKV ? kAtom : 0);
  static constexpr int LOAD_BYTES = (LQ ? AK * kAtom : 0) + (LKV ? (AK + AV) * kAtom : 0);
  // bf16 S operand, MN-major [atoms of 64 value columns][DK rows][128 B]; non-causal adds an
  // atom whose column 0 is z, so O (N = DV + 16) carries phi(q_i).z in its column DV
  static constexpr int S_ATOM = DK * 128;
  static constexpr int S_ATOMS = MODE == kState ? 0 : (MODE == kNoncausalOut ? AV + 1 : AV);
  static constexpr int S_BUF = S_ATOMS * S_ATOM;  // one S operand
  // non-causal: two S operands, so the next item's total is rounded while this one runs
  static constexpr int S_BYTES = (MODE == kNoncausalOut ? 2 : 1) * S_BUF;
  static constexpr int P_BYTES = MODE == kCausalOut ? kAtom : 0;  // bf16 [64][64], K-major
  static constexpr int FIXED = S_BYTES + P_BYTES;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int NS_FIT = (kMaxSmem - 1024 - BAR_BYTES - FIXED) / STAGE;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int OFF_S = NS * STAGE;
  static constexpr int OFF_P = OFF_S + S_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
  static_assert(NS >= 2, "at least two pipeline stages");
  static_assert(SMEM <= kMaxSmem, "shared memory budget");
  static_assert(OFF_S % 1024 == 0 && OFF_P % 1024 == 0 && STAGE % 1024 == 0 &&
                    OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_ONES % 1024 == 0 &&
                    KATOM % 1024 == 0 && S_ATOM % 1024 == 0,
                "128B-swizzled operands need 1024-byte alignment");
};

// TMEM column map (32-column aligned): P (80 columns, causal), two O buffers (DV columns,
// plus the 16-column denominator block in the non-causal mode), S (DV + 16 columns, z in
// column DV).  The aggregate mode keeps two S accumulators, one per item parity, so one
// item's aggregate is written out while the next one accumulates.
template <int DV, int MODE>
struct TmemMap {
  static constexpr uint32_t P = 0;
  static constexpr uint32_t OW = ((MODE == kNoncausalOut ? DV + 16 : DV) + 31) / 32 * 32;
  static constexpr uint32_t O0 = MODE == kCausalOut ? 96 : 0;
  static constexpr uint32_t O1 = O0 + OW;
  static constexpr uint32_t S = MODE == kCausalOut ? O1 + OW : 0;  // unused when non-causal
  static constexpr uint32_t S1 = MODE == kState ? kTmemCols / 2 : S;
  static_assert((MODE == kNoncausalOut ? O1 + OW : S1 + DV + 16) <= kTmemCols, "TMEM budget");
};

struct Bars {
  uint64_t full[8], ready[8], empty[8];
  uint64_t p_full, p_ready, s_full, s_ready, z_ready, rs_ready, o_full[2], o_empty[2], fin, fin2;
  // per item parity: aggregate mode, S accumulator complete (MMA -> state group) / written out
  // (state group -> MMA); non-causal, S operand rounded (state group -> MMA) / no longer read
  // (MMA -> state group)
  uint64_t item_full[2], item_empty[2];
  float rowsum[2][64];  // the state group's half of P's row sums, by chunk parity
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

// Columns [c0, c0 + 32) of the causal score row r64 (lanes < 16 of each warp hold rows of the
// M = 64 accumulator): mask keys after the query (j > i), round to bf16 into the K-major
// operand of P V, and return the row's partial sum (of the unrounded fp32 scores; it differs
// from the sum of the rounded ones by at most 2^-9 relative).
__device__ __forceinline__ float convert_P32(uint32_t taddr, uint8_t *sP, int r64, bool v64,
                                             int c0) {
  uint32_t p[32];
  tmem_ld16_async(taddr + c0, p);
  tmem_ld16_async(taddr + c0 + 16, p + 16);
  tmem_ld_wait();
  tmem_reg_fence<32>(p);
  float sum = 0.f;
  if (v64) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int g = c0 + 8 * j;  // first key of this group of 8
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x = __uint_as_float(p[8 * j + e]);
        f[e] = (g + 7 <= r64 || g + e <= r64) ? x : 0.f;
        sum += f[e];
      }
      *reinterpret_cast<uint4 *>(sP + sw128_offset(r64, g)) =
          g > r64 ? make_uint4(0u, 0u, 0u, 0u) : pack8(f);
    }
  }
  return sum;
}

// CTA b takes the items b, b + gridDim.x, b + 2 gridDim.x, ... (one item when the grid
// covers them all; several on persistent CTAs).  Every role walks the same sequence of
// chunks, and g counts them across items, so the stage ring, the barrier phases and the O
// buffers run on from one item into the next: the loads of an item's first chunks overlap
// the previous item's last ones.
// PHI: apply phi = elu + 1 to Q and K (the method); false takes Q and K as given,
// non-negative features (FAVOR+ features computed by the feature kernels).
// init_state: per item, the fp32 state [DK][DV] then z [DK] it starts from (causal: the
// exclusive prefix, at init_state + head * init_head_stride + seg * init_seg_stride;
// non-causal: the head's total).  out_state (aggregate): [heads][nseg][DK*DV + DK].
template <int DK, int DV, int MODE, bool PHI>
__global__ void __launch_bounds__(Warps<MODE, DK>::THREADS, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ out,
              const float *__restrict__ init_state, int64_t init_head_stride,
              int64_t init_seg_stride, float *__restrict__ out_state, int64_t n, int64_t seg_len,
              int64_t nseg, int64_t nitems, int *err) {
  using G = Cfg<DK, DV, MODE>;
  using TM = TmemMap<DV, MODE>;
  using W = Warps<MODE, DK>;
  constexpr int NS = G::NS;
  constexpr int TEAMS = NS % W::XTEAMS == 0 ? W::XTEAMS : 1;
  constexpr int TEAM_THREADS = W::XTHREADS / TEAMS;
  constexpr int KSD = DK / 16;  // K-steps over the feature dimension
  constexpr int KSC = C / 16;   // K-steps over the chunk's tokens
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Bars &bar = *reinterpret_cast<Bars *>(smem + G::OFF_BAR);
  volatile int *abort = &bar.abort;

  const int warp = threadIdx.x >> 5;
  const bool a32 = aligned32(out);  // output rows take full-sector stores
  const int lane = threadIdx.x & 31;
  const int64_t it0 = blockIdx.x, istep = gridDim.x;

  // ---- set-up: barriers, constant operand blocks, TMEM
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.ready[s], TEAM_THREADS);
      mbar_init(&bar.empty[s], 1);
    }
    mbar_init(&bar.p_full, 1);
    // the score drains: both groups, or (two issuers) the output group alone
    mbar_init(&bar.p_ready, W::TWO_ISSUERS ? kGroupThreads : 2 * kGroupThreads);
    mbar_init(&bar.rs_ready, kGroupThreads);
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.s_ready, kGroupThreads);
    mbar_init(&bar.z_ready, kGroupThreads);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.o_full[b], 1);
      mbar_init(&bar.o_empty[b], kGroupThreads);
      mbar_init(&bar.item_full[b], MODE == kNoncausalOut ? kGroupThreads : 1);
      mbar_init(&bar.item_empty[b], MODE == kState ? kGroupThreads : 1);
    }
    mbar_init(&bar.fin, 1);
    mbar_init(&bar.fin2, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  for (int s = 0; s < NS; ++s) {
    uint8_t *st = smem + s * G::STAGE;
    if (G::LKV) {
      // ones atom: column 0 of every row is 1.0 (row r's column 0 sits in 16-byte chunk r & 7)
      uint32_t *ones = reinterpret_cast<uint32_t *>(st + G::OFF_ONES);
      for (int i = threadIdx.x; i < kAtom / 4; i += W::THREADS) {
        const int row = i >> 5, word = i & 31;  // 32 words per 128-byte row
        ones[i] = (word == 4 * (row & 7)) ? 0x00003F80u : 0u;
      }
    }
    if (MODE == kCausalOut) {
      // z rows of the K tile start at zero (row 64 is rewritten before every chunk)
      for (int a = 0; a < G::AK; ++a) {
        uint32_t *zr = reinterpret_cast<uint32_t *>(st + G::OFF_K + a * G::KATOM + 64 * 128);
        for (int i = threadIdx.x; i < kZRows * 128 / 4; i += W::THREADS) zr[i] = 0u;
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

  // O of chunk gg (chunk c of item I) over its denominator -> bf16 rows of out, by the four
  // output warps (one per TMEM sub-partition; lanes < 16 hold the rows of the M = 64 product).
  // den: the causal denominator; the non-causal one is column DV of the accumulator.
  auto emit_O = [&](auto &wait, int gg, const Item &I, int c, float den) {
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const bool v64 = lane < 16;
    const int r64 = 16 * (warp & 3) + lane;
    const int ob = gg & 1;
    const uint32_t tO = tmem + lane_off + (ob ? TM::O1 : TM::O0);
    if (!wait(&bar.o_full[ob], (gg >> 1) & 1)) return;
    tc_fence_after();
    const float dd = MODE == kCausalOut ? den : __uint_as_float(tmem_ld1(tO + DV));
    const float inv = 1.f / dd;
    const int64_t t = I.t_begin + (int64_t)c * C + r64;
    const bool live = v64 && t < I.t_end;
    __nv_bfloat16 *orow = out + (I.head * n + (live ? t : 0)) * DV;
#pragma unroll 1
    for (int c0 = 0; c0 < DV; c0 += 64) {
      uint32_t r[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld16_async(tO + c0 + 16 * q, r + 16 * q);
      tmem_ld_wait();
      tmem_reg_fence<64>(r);
      if (live) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
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
          }
          if (G::LKV) {
#pragma unroll
            for (int a = 0; a < G::AK; ++a)
              tma_load_3d(st + G::OFF_K + a * G::KATOM, &tmK, &bar.full[s], a * 64, y, zc, pol);
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
      constexpr uint32_t I_P = make_idesc_bf16(64, 64 + kZRows, false, false);
      constexpr uint32_t I_O =
          make_idesc_bf16(64, MODE == kNoncausalOut ? DV + 16 : DV, false, true);
      constexpr uint32_t I_S = make_idesc_bf16(DK, DV + 16, true, true);
      constexpr uint32_t I_OV = make_idesc_bf16(64, DV, false, true);
      uint64_t dVprev = 0;  // causal: [V | ones] of the previous chunk (its P V is still due)
      int sprev = 0;        // and that chunk's stage
      const uint32_t tP = tmem + TM::P;
      const uint64_t dP = kmajor_base(smem_u32(smem + G::OFF_P));
      const uint32_t st0 = smem_u32(smem);
      int g = 0;
      int j = 0;  // items of this CTA
      bool ok = true;
      for (int64_t it = it0; ok && it < nitems; it += istep, ++j) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        const int b = j & 1;
        const uint32_t tS = tmem + (b ? TM::S1 : TM::S);
        const uint64_t dS = mnmajor_base(
            smem_u32(smem + G::OFF_S + (MODE == kNoncausalOut ? b * G::S_BUF : 0)), G::S_ATOM);
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
          const uint64_t dQk = kmajor_base(st);                        // Q, K-major
          const uint64_t dKk = kmajor_base(st + G::OFF_K);             // K (+z rows), K-major
          const uint64_t dKm = mnmajor_base(st + G::OFF_K, G::KATOM);  // K, MN-major
          const uint64_t dVm = mnmajor_base(st + G::OFF_V, kAtom);     // [V | ones], MN-major
          tc_fence_after();
          if (MODE == kState) {
#pragma unroll
            for (int ks = 0; ks < KSC; ++ks)
              mma_bf16_ss(tS, desc_add(dKm, mnmajor_off(ks)), desc_add(dVm, mnmajor_off(ks)),
                          I_S, (c > 0 || ks > 0) ? 1u : 0u);
            mma_commit(&bar.empty[s]);
            continue;
          }
          const int ob = g & 1;
          const uint32_t tO = tmem + (ob ? TM::O1 : TM::O0);
          if (MODE == kCausalOut) {
            // The previous chunk's P V (its scores rounded by now) interleaved with this
            // chunk's [scores | phi(q).z_<c]: different accumulators, so the tensor pipe
            // overlaps the two chains instead of running them back to back.  With a second
            // issuer, its products of the previous chunk (phi(Q) S_<c onto which P V adds, and
            // the S update, both reading its stage) are done by z_ready: the state group
            // reads z after their commit.
            if (!mbar_wait(&bar.z_ready, g & 1, abort, err)) {
              ok = false;
              break;
            }
            if (g >= 1 && !mbar_wait(&bar.p_ready, (g - 1) & 1, abort, err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t tOp = tmem + (((g - 1) & 1) ? TM::O1 : TM::O0);  // O of chunk g - 1
#pragma unroll
            for (int ks = 0; ks < KSD; ++ks) {
              if (g >= 1 && ks < KSC)
                mma_bf16_ss(tOp, desc_add(dP, kmajor_off(ks, kAtom)),
                            desc_add(dVprev, mnmajor_off(ks)), I_OV, 1u);
              mma_bf16_ss(tP, desc_add(dQk, kmajor_off(ks, kAtom)),
                          desc_add(dKk, kmajor_off(ks, G::KATOM)), I_P, ks > 0 ? 1u : 0u);
              if (g >= 1 && ks == KSC - 1) {
                mma_commit(&bar.o_full[(g - 1) & 1]);
                mma_commit(&bar.empty[sprev]);
              }
            }
            mma_commit(&bar.p_full);
            if (!W::TWO_ISSUERS) {
              // S_<c in the S operand; this O buffer drained
              if (!mbar_wait(&bar.s_ready, g & 1, abort, err)) {
                ok = false;
                break;
              }
              if (g >= 2 && !mbar_wait(&bar.o_empty[ob], ((g >> 1) - 1) & 1, abort, err)) {
                ok = false;
                break;
              }
              tc_fence_after();
              // phi(Q_c) S_<c, then S += phi(K_c)^T [V_c | 1] (interleaving these two
              // measured no faster)
#pragma unroll
              for (int ks = 0; ks < KSD; ++ks)
                mma_bf16_ss(tO, desc_add(dQk, kmajor_off(ks, kAtom)),
                            desc_add(dS, mnmajor_off(ks)), I_O, ks > 0 ? 1u : 0u);
#pragma unroll
              for (int ks = 0; ks < KSC; ++ks)
                mma_bf16_ss(tS, desc_add(dKm, mnmajor_off(ks)), desc_add(dVm, mnmajor_off(ks)),
                            I_S, 1u);
              mma_commit(&bar.s_full);
            }
            dVprev = dVm;  // P V of this chunk goes with the next chunk's scores
            sprev = s;
            continue;
          }
          // non-causal: this O buffer drained
          if (g >= 2 && !mbar_wait(&bar.o_empty[ob], ((g >> 1) - 1) & 1, abort, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
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
      if (MODE == kCausalOut && ok && g > 0) {
        // the last chunk's P V, once a second issuer's products of that chunk are done
        // (nothing else waits for that s_full phase)
        if ((!W::TWO_ISSUERS || mbar_wait(&bar.s_full, (g - 1) & 1, abort, err)) &&
            mbar_wait(&bar.p_ready, (g - 1) & 1, abort, err)) {
          tc_fence_after();
          const uint32_t tOp = tmem + (((g - 1) & 1) ? TM::O1 : TM::O0);
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tOp, desc_add(dP, kmajor_off(ks, kAtom)), desc_add(dVprev, mnmajor_off(ks)),
                        I_OV, 1u);
          mma_commit(&bar.o_full[(g - 1) & 1]);
          mma_commit(&bar.empty[sprev]);
        }
      }
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(&bar.fin);
      mbar_wait_drain(&bar.fin, 0, err);
    }
  } else if (W::TWO_ISSUERS && warp == W::MMA2) {
    // ================================================================ second MMA issuer
    // Causal, per chunk c: O = phi(Q_c) S_<c into the chunk's O buffer, then
    // [S | z] += phi(K_c)^T [V_c | 1] (interleaving these two measured no faster).  These are
    // issued as soon as their inputs are ready, not after the first issuer's scores of the
    // chunk: holding them back for the scores measured 10% slower (the S update ends the
    // chain that gives the next chunk its z).
    if (lane == 0) {
      constexpr uint32_t I_O = make_idesc_bf16(64, DV, false, true);
      constexpr uint32_t I_S = make_idesc_bf16(DK, DV + 16, true, true);
      const uint32_t tS = tmem + TM::S;
      const uint64_t dS = mnmajor_base(smem_u32(smem + G::OFF_S), G::S_ATOM);
      const uint32_t st0 = smem_u32(smem);
      int g = 0;
      bool ok = true;
      for (int64_t it = it0; ok && it < nitems; it += istep) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        for (int c = 0; c < I.nchunks; ++c, ++g) {
          const int s = g % NS;
          const int ob = g & 1;
          // the chunk's features; S_<c in the S operand (and TMEM S read out); this O
          // buffer drained
          if (!mbar_wait(&bar.ready[s], (g / NS) & 1, abort, err) ||
              !mbar_wait(&bar.s_ready, g & 1, abort, err) ||
              (g >= 2 && !mbar_wait(&bar.o_empty[ob], ((g >> 1) - 1) & 1, abort, err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = st0 + s * G::STAGE;
          const uint32_t tO = tmem + (ob ? TM::O1 : TM::O0);
          const uint64_t dQk = kmajor_base(st);                        // Q, K-major
          const uint64_t dKm = mnmajor_base(st + G::OFF_K, G::KATOM);  // K, MN-major
          const uint64_t dVm = mnmajor_base(st + G::OFF_V, kAtom);     // [V | ones], MN-major
#pragma unroll
          for (int ks = 0; ks < KSD; ++ks)
            mma_bf16_ss(tO, desc_add(dQk, kmajor_off(ks, kAtom)), desc_add(dS, mnmajor_off(ks)),
                        I_O, ks > 0 ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < KSC; ++ks)
            mma_bf16_ss(tS, desc_add(dKm, mnmajor_off(ks)), desc_add(dVm, mnmajor_off(ks)), I_S,
                        1u);
          mma_commit(&bar.s_full);
        }
      }
      mma_commit(&bar.fin2);
      mbar_wait_drain(&bar.fin2, 0, err);
    }
  } else if (warp < W::STATE0) {
    // ================================================================ feature map
    // phi in place on the Q tile and on the 64 key rows of each K atom; K rows past the
    // item's end are zeroed (they must add nothing to S, z or the scores).
    const int team = (threadIdx.x - W::XFORM0 * 32) / TEAM_THREADS;
    const int xt = (threadIdx.x - W::XFORM0 * 32) % TEAM_THREADS;
    int g = 0;
    bool ok = true;
    for (int64_t it = it0; ok && it < nitems; it += istep) {
      const Item I = item_at<C>(it, n, seg_len, nseg);
      for (int c = 0; c < I.nchunks; ++c, ++g) {
        if (g % TEAMS != team) continue;  // another team's stage
        const int s = g % NS;
        if (!mbar_wait(&bar.full[s], (g / NS) & 1, abort, err)) {
          ok = false;
          break;
        }
        uint8_t *st = smem + s * G::STAGE;
        const int64_t left = I.t_end - (I.t_begin + (int64_t)c * C);
        const int valid = left < C ? static_cast<int>(left) : C;
        if (G::LQ && PHI) {
          uint4 *p = reinterpret_cast<uint4 *>(st);
#pragma unroll 2
          for (int i = xt; i < G::AK * kAtom / 16; i += TEAM_THREADS) p[i] = phi_bf16x8(p[i]);
        }
        if (G::LKV) {
#pragma unroll 2
          for (int i = xt; i < G::AK * kAtom / 16; i += TEAM_THREADS) {
            const int a = i / (kAtom / 16), within = i % (kAtom / 16);
            const int row = within >> 3;  // 8 x 16 B per 128-byte row
            uint4 *p = reinterpret_cast<uint4 *>(st + G::OFF_K + a * G::KATOM) + within;
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
    // Causal: half of each chunk's scores (columns 0..31) and their row sums; S_<c+1, z_<c+1
    // -> bf16 operands of the next chunk (z into that chunk's K tile row 64); each item's
    // starting state.  Non-causal: each item's head total -> one of the two S operands.
    // Aggregate: each item's aggregate.  Control flow is warp-uniform: lane 0 waits and the
    // warp shares the outcome.
    const int sp = warp & 3;  // TMEM sub-partition of this warp
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const bool v64 = lane < 16;                       // lanes holding rows of an M=64 tile
    const int r64 = 16 * sp + lane;                   // row of an M=64 tile
    const int rS = DK == 128 ? 32 * sp + lane : r64;  // row of the S accumulator (M = DK)
    const bool vS = DK == 128 ? true : v64;
    WarpWaiterT<(DV >= 128)> wait{abort, err, lane};  // measured per value width
    // the output kernels start while the scan before them finishes (a programmatic launch):
    // the starting states it writes are read only once it is done
    if (MODE != kState) grid_dependency_wait();

    // 32 consecutive S columns [c0, c0+32) of row rS (fp32 in registers) -> bf16 operand sS
    auto store_S32 = [&](uint8_t *sS, const uint32_t *r, int c0) {
      if (!vS) return;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * q + e]);
        *reinterpret_cast<uint4 *>(sS + (c0 >> 6) * G::S_ATOM +
                                   sw128_offset(rS, (c0 & 63) + 8 * q)) = pack8(f);
      }
    };
    // z_< for chunk gg: causal -> row 64 of that chunk's K atoms; non-causal -> column 0 of
    // the z atom of the S operand sS
    auto store_z = [&](uint8_t *sS, uint32_t zbits, int gg) {
      if (!vS) return;
      const __nv_bfloat16 zb = __float2bfloat16_rn(__uint_as_float(zbits));
      if (MODE == kCausalOut) {
        uint8_t *kt = smem + (gg % NS) * G::STAGE + G::OFF_K;
        *reinterpret_cast<__nv_bfloat16 *>(kt + (rS >> 6) * G::KATOM +
                                           sw128_offset(64, rS & 63)) = zb;
      } else {
        *reinterpret_cast<__nv_bfloat16 *>(sS + G::AV * G::S_ATOM + sw128_offset(rS, 0)) = zb;
      }
    };
    // an item's starting state (exclusive prefix, causal; the head's total, non-causal) ->
    // TMEM S (causal) and the bf16 operand sS; z for the item's first chunk gg
    auto load_start = [&](const Item &I, uint8_t *sS, int gg) {
      const float *src = init_state + I.head * init_head_stride + I.seg * init_seg_stride;
      for (int c0 = 0; c0 < DV; c0 += 32) {
        uint32_t r[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (vS) f = *reinterpret_cast<const float4 *>(src + (int64_t)rS * DV + c0 + 4 * q);
          r[4 * q + 0] = __float_as_uint(f.x);
          r[4 * q + 1] = __float_as_uint(f.y);
          r[4 * q + 2] = __float_as_uint(f.z);
          r[4 * q + 3] = __float_as_uint(f.w);
        }
        if (MODE == kCausalOut) {
#pragma unroll
          for (int q = 0; q < 2; ++q)
            tmem_st16(tmem + lane_off + TM::S + c0 + 16 * q,
                      *reinterpret_cast<const uint32_t(*)[16]>(r + 16 * q));
        }
        store_S32(sS, r, c0);
      }
      const uint32_t zb = vS ? __float_as_uint(src[(int64_t)DK * DV + rS]) : 0u;
      if (MODE == kCausalOut) {
        tmem_st1(tmem + lane_off + TM::S + DV, zb);
        tmem_st_wait();
      }
      store_z(sS, zb, gg);
      fence_proxy_async_smem();
    };

    if (MODE == kCausalOut) {
      // One flat loop over this CTA's chunks; only the chunk counter, the chunks left in
      // the current item and the next item's index stay live across it.
      uint8_t *sS = smem + G::OFF_S;
      int64_t it = it0;
      int left = 0;
#pragma unroll 1
      for (int g = 0;; ++g) {
        if (left == 0) {
          // ---- an item's starting state, once the previous item's last S and O products
          // are done with TMEM S and the S operand
          if (it >= nitems) break;
          const Item I = item_at<C>(it, n, seg_len, nseg);
          it += istep;
          left = I.nchunks;
          if (g == 0 || wait(&bar.s_full, (g - 1) & 1)) {
            tc_fence_after();
            load_start(I, sS, g);
            tc_fence_before();
          }
          mbar_arrive(&bar.z_ready);
          mbar_arrive(&bar.s_ready);
        }
        // ---- this chunk's scores, columns 0..31 (the output group takes 32..63; with two
        // issuers it takes all 64, measured 2% faster than sharing them, and this group only
        // waits for the scores: that keeps its z_ready at most one phase ahead of the first
        // issuer's wait, which the second issuer alone would not)
        if (W::TWO_ISSUERS) {
          wait(&bar.p_full, g & 1);
        } else if (wait(&bar.p_full, g & 1)) {
          tc_fence_after();
          const float rs = convert_P32(tmem + lane_off + TM::P, smem + G::OFF_P, r64, v64, 0);
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&bar.p_ready);
          if (v64) bar.rowsum[g & 1][r64] = rs;
          mbar_arrive(&bar.rs_ready);
        }
        // ---- S_<c+1, z_<c+1: the operands of the item's next chunk
        if (--left > 0 && wait(&bar.s_full, g & 1)) {
          tc_fence_after();
          // z_<c+1 first: the next chunk's score MMA needs only that
          store_z(sS, tmem_ld1(tmem + lane_off + TM::S + DV), g + 1);
          fence_proxy_async_smem();
          mbar_arrive(&bar.z_ready);
#pragma unroll 1
          for (int c0 = 0; c0 < DV; c0 += 64) {
            uint32_t r[64];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              tmem_ld16_async(tmem + lane_off + TM::S + c0 + 16 * q, r + 16 * q);
            tmem_ld_wait();
            tmem_reg_fence<64>(r);
            store_S32(sS, r, c0);
            store_S32(sS, r + 32, c0 + 32);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&bar.s_ready);
        }
      }
    } else if (MODE == kNoncausalOut) {
      int j = 0;
      for (int64_t it = it0; it < nitems; it += istep, ++j) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        const int b = j & 1;
        uint8_t *sS = smem + G::OFF_S + b * G::S_BUF;
        // the MMAs of item j - 2 no longer read this S operand
        if (j < 2 || wait(&bar.item_empty[b], ((j >> 1) - 1) & 1)) load_start(I, sS, 0);
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
              for (int e = 0; e < 32; e += 8)
                st_global_32B(dst + (int64_t)rS * DV + c0 + e,
                              make_uint4(r[e], r[e + 1], r[e + 2], r[e + 3]),
                              make_uint4(r[e + 4], r[e + 5], r[e + 6], r[e + 7]), true);
            }
          }
          const uint32_t zr = tmem_ld1(tS + DV);
          if (vS) dst[(int64_t)DK * DV + rS] = __uint_as_float(zr);
        }
        tc_fence_before();
        mbar_arrive(&bar.item_empty[b]);
      }
    }
  } else {
    // ================================================================ scores and output
    // P(c) columns 32..63 -> masked bf16 operand of P V (the state group takes 0..31; with two
    // issuers this group takes all 64), with
    // phi(q).z_<c (column 64) and both groups' row sums -> the denominator of chunk c; then
    // O(c-1) / den -> bf16 rows stored straight to global memory (32-byte stores; rows past
    // the item's end are not written).
    const int sp = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * sp) << 16;
    const bool v64 = lane < 16;
    const int r64 = 16 * sp + lane;
    WarpWaiterT<(DV >= 128)> wait{abort, err, lane};  // measured per value width

    // Denominators of the chunks in flight, by parity.  The state group's half of the row sum
    // is read BEFORE this group releases p_ready: the state group's next sums need this
    // chunk's p_ready, so it never completes rs_ready's next phase (or rewrites that slot)
    // before this wait has seen the current one.
    float den0 = 1.f, den1 = 1.f;
    auto convert_P = [&](int gg) {
      if (!wait(&bar.p_full, gg & 1)) return;
      tc_fence_after();
      float rs = convert_P32(tmem + lane_off + TM::P, smem + G::OFF_P, r64, v64, 32);
      const float dz = __uint_as_float(tmem_ld1(tmem + lane_off + TM::P + 64));
      float d;
      if (W::TWO_ISSUERS) {
        // this group converts both halves: the row sums are all its own
        rs += convert_P32(tmem + lane_off + TM::P, smem + G::OFF_P, r64, v64, 0);
        d = dz + rs;
      } else {
        const bool got = wait(&bar.rs_ready, gg & 1);
        d = dz + rs + (got ? bar.rowsum[gg & 1][v64 ? r64 : 0] : 0.f);
      }
      if (gg & 1) den1 = d; else den0 = d;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar.p_ready);
    };


    if (MODE == kCausalOut) {
      int g = 0;
      Item prev{};
      int prev_c = 0;
      for (int64_t it = it0; it < nitems; it += istep) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        for (int c = 0; c < I.nchunks; ++c, ++g) {
          convert_P(g);
          if (g >= 1) emit_O(wait, g - 1, prev, prev_c, ((g - 1) & 1) ? den1 : den0);
          prev = I;
          prev_c = c;
        }
      }
      if (g > 0) emit_O(wait, g - 1, prev, prev_c, ((g - 1) & 1) ? den1 : den0);
    } else if (MODE == kNoncausalOut) {
      int g = 0;
      for (int64_t it = it0; it < nitems; it += istep) {
        const Item I = item_at<C>(it, n, seg_len, nseg);
        for (int c = 0; c < I.nchunks; ++c, ++g) emit_O(wait, g, I, c, 0.f);
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
                      void *out, const float *init, int64_t ihs, int64_t iss, float *out_state,
                      int64_t heads, int64_t n, int64_t seg, int64_t nseg, int *err,
                      cudaStream_t st) {
  using G = Cfg<DK, DV, MODE>;
  auto kern = tc_kernel<DK, DV, MODE, PHI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  // One CTA holds a whole SM's shared memory and TMEM.  Persistent CTAs (one per SM, items
  // dealt round-robin) save each item the CTA start-up and pipeline fill and drain; they
  // pay off for the aggregate and non-causal kernels and for short causal items.  Long
  // causal items run one CTA each: there the hardware's dynamic placement of CTAs on SMs
  // evens out the few per cent by which SMs differ in speed, and a fresh CTA hides the load
  // of its starting state behind its first TMA loads.
  const int64_t nitems = heads * nseg;
  const int64_t sms = sm_count();
  const bool persistent = MODE != kCausalOut || seg <= kPersistentCausalChunks * C;
  const int64_t want = persistent ? sms : nitems;
  const unsigned grid = static_cast<unsigned>(nitems < want ? nitems : want);
  if (MODE == kState) {
    kern<<<grid, Warps<MODE, DK>::THREADS, G::SMEM, st>>>(q, k, v, static_cast<__nv_bfloat16 *>(out),
                                                      init, ihs, iss, out_state, n, seg, nseg,
                                                      nitems, err);
  } else {
    // the output kernels follow the scan: launched so that their set-up and first loads of
    // q, k, v overlap the scan's tail (the state group waits for the scan's results)
    e = launch_programmatic(kern, dim3(grid), dim3(Warps<MODE, DK>::THREADS), G::SMEM, st, q, k, v,
                            static_cast<__nv_bfloat16 *>(out), init, ihs, iss, out_state, n, seg,
                            nseg, nitems, err);
    if (e != cudaSuccess) return e;
  }
  count_launches(1);
  record_launch_event(st);
  return cudaGetLastError();
}

// The whole pass: K1 aggregates, K2 scan, K3 outputs.  q, k: [heads][n][DK]; v, out: [heads]
// [n][DV].
template <int DK, int DV, bool PHI>
cudaError_t tc_forward_dims(const void *q, const void *k, const void *v, void *out,
                            int64_t heads, int64_t n, int causal, int64_t seg, void *ws, int *err,
                            const float *init_S, const float *init_z, cudaStream_t st,
                            float *aggregates) {
  const int64_t nseg = (n + seg - 1) / seg;
  const int64_t per = (int64_t)DK * DV + DK;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_tmap_bf16(&tq, q, heads, n, DK, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tk, k, heads, n, DK, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, heads, n, DV, C)) != cudaSuccess) return e;
  // the segment aggregates: computed here (K1), or given
  float *w = aggregates ? aggregates : static_cast<float *>(ws);
  if (!aggregates) {
    e = launch_tc<DK, DV, kState, PHI>(tk, tk, tv, out, nullptr, 0, 0, w, heads, n, seg, nseg,
                                       err, st);
    if (e != cudaSuccess) return e;
  }
  if (causal) {
    e = launch_scan_states(w, heads, nseg, DK, DV, 0, nullptr, 0, nullptr, 0, init_S, init_z, st);
    if (e != cudaSuccess) return e;
    // one dimension: the 64-token causal kernel here; features of their own dimension:
    // tc_causal.cu's
    if constexpr (DK == DV)
      return launch_tc<DK, DV, kCausalOut, PHI>(tq, tk, tv, out, w, nseg * per, per, nullptr,
                                                heads, n, seg, nseg, err, st);
    else
      return tc_causal_features(q, k, v, out, heads, n, DK, DV, seg, w, err, st);
  }
  // per-head totals, packed as [heads][DK*DV + DK] (S row-major, then z)
  float *tot = aggregates ? static_cast<float *>(ws) : w + heads * nseg * per;
  e = launch_scan_states(w, heads, nseg, DK, DV, 1, tot, per, tot + (int64_t)DK * DV, per, init_S,
                         init_z, st);
  if (e != cudaSuccess) return e;
  return launch_tc<DK, DV, kNoncausalOut, PHI>(tq, tk, tv, out, tot, per, 0, nullptr, heads, n,
                                               seg, nseg, err, st);
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
  e = launch_tc<DK, DV, kState, true>(tk, tk, tv, nullptr, nullptr, 0, 0, w, heads, n, seg, nseg,
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
  int64_t best = 256, best_score = -1;
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
  const int64_t nrounded = ((n + kTcFeatureChunk - 1) / kTcFeatureChunk) * kTcFeatureChunk;
  return best > nrounded ? nrounded : best;
}

size_t tc_workspace_bytes(int64_t heads, int64_t n, int dk, int dv, int64_t seg, int causal) {
  const int64_t nseg = (n + seg - 1) / seg;
  const int64_t per = (int64_t)dk * dv + dk;
  return (size_t)(heads * nseg * per + (causal ? 0 : heads * per)) * sizeof(float);
}

cudaError_t tc_forward(const void *q, const void *k, const void *v, void *out, int64_t heads,
                       int64_t n, int dk, int dv, int causal, int64_t seg, void *ws, int *err,
                       const float *init_S, const float *init_z, int features,
                       cudaStream_t st, float *aggregates) {
  if (!features) {  // phi = elu + 1 keeps the dimension
    if (dk == 64 && dv == 64)
      return tc_forward_dims<64, 64, true>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                           init_z, st, aggregates);
    if (dk == 128 && dv == 128)
      return tc_forward_dims<128, 128, true>(q, k, v, out, heads, n, causal, seg, ws, err,
                                             init_S, init_z, st, aggregates);
    return cudaErrorInvalidValue;
  }
  if (dk == 64 && dv == 64)
    return tc_forward_dims<64, 64, false>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                          init_z, st, aggregates);
  if (dk == 128 && dv == 128)
    return tc_forward_dims<128, 128, false>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                            init_z, st, aggregates);
  if (dk == 128 && dv == 64)
    return tc_forward_dims<128, 64, false>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                           init_z, st, aggregates);
  if (dk == 64 && dv == 128)
    return tc_forward_dims<64, 128, false>(q, k, v, out, heads, n, causal, seg, ws, err, init_S,
                                           init_z, st, aggregates);
  return cudaErrorInvalidValue;
}

cudaError_t tc_segment_aggregates(const void *k, const void *v, int64_t heads, int64_t n, int d,
                                  int64_t seg, float *out, int *err, cudaStream_t st) {
  const int64_t nseg = (n + seg - 1) / seg;
  CUtensorMap tk, tv;
  cudaError_t e;
  if ((e = make_tmap_bf16(&tk, k, heads, n, d, C)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, heads, n, d, C)) != cudaSuccess) return e;
  if (d == 64)
    return launch_tc<64, 64, kState, true>(tk, tk, tv, nullptr, nullptr, 0, 0, out, heads, n, seg,
                                           nseg, err, st);
  if (d == 128)
    return launch_tc<128, 128, kState, true>(tk, tk, tv, nullptr, nullptr, 0, 0, out, heads, n,
                                             seg, nseg, err, st);
  return cudaErrorInvalidValue;
}

cudaError_t tc_forward_state(const void *k, const void *v, float *S_out, float *z_out,
                             int64_t heads, int64_t n, int d, int64_t seg, void *ws, int *err,
                             cudaStream_t st) {
  return d == 64 ? tc_state_dims<64, 64>(k, v, S_out, z_out, heads, n, seg, ws, err, st)
                 : tc_state_dims<128, 128>(k, v, S_out, z_out, heads, n, seg, ws, err, st);
}

}  // namespace linattn
