// prefill_sm100.cuh -- causal differential attention prefill on tcgen05.
//
// One CTA computes 128 query rows of one output head, for both maps:
//   S_m = Q_m K_m^T          (tcgen05.mma, A and B from shared memory, D in TMEM)
//   P_m = exp(S_m/sqrt(d) - rowmax_m), l_m = rowsum(P_m)   (online, per map)
//   O_m += P_m V             (tcgen05.mma, A = P_m from TMEM, B = V from smem)
//   out = O_1 / l_1 - lambda * O_2 / l_2  [then RMSNorm]     (epilogue)
// ("差分注意力" tutorial, section 差分思路 and Step 2; V1/V2 layouts from
// its section V1 到 V2 的 diff.)  Each K/V tile is loaded once by TMA and
// serves both maps: in V2 both maps share K and V; in V1 the tile holds K1,
// K2 and the shared V.
//
// Warp roles (352 threads):
//   warps 0-3  softmax of map 1 (thread i <-> query row i <-> TMEM lane i)
//   warps 4-7  softmax of map 2
//   warp  8    TMA producer; allocates / frees TMEM
//   warp  9    PV issuer (one thread)
//   warp 10    QK issuer (one thread)
// Keys are processed in tiles of 64.  TMEM (512 columns) holds two S buffers
// per map -- S1[0] [0,64) S1[1] [64,128) S2[0] [128,192) S2[1] [192,256) --
// and the accumulators O1 [256,384) O2 [384,512).  While a map's softmax works
// on tile j in one buffer, the tensor pipe computes S for tile j+1 into the
// other, so each map's softmax runs back to back.  P_m(j) is written over
// S_m(j) as bf16 P_hi in the buffer's columns [0,32) and, for heads that need
// it, the bf16 residual P_lo = P - P_hi in [32,64); both accumulate into O_m.
// The tensor pipe takes MMAs from a very shallow queue, so a single issuing
// thread that stops to test a barrier leaves it idle.  Two issuers keep it
// fed: one issues PV_m(j) when P_m(j) is stored, the other issues S_m(j+2)
// into the buffer PV_m(j) read, once that PV has completed (s_free); each
// one's waits overlap the other's MMAs.
// Shared memory: Q1, Q2 tiles (128 rows), then NS stages of {K tile(s), V
// tile} of 64 keys; every tile is a set of boxes of 128-byte rows in the TMA
// 128-byte swizzle, which is the canonical K-major (Q, K) / MN-major (V) UMMA
// layout.
#pragma once

#include "common.cuh"

namespace da {

constexpr int PF_BM = 128;         // query rows per CTA
constexpr int PF_BN = 64;          // keys per tile
constexpr int PF_DV = 128;         // value width
constexpr int PF_NS = 4;           // K/V pipeline stages
constexpr int PF_THREADS = 352;
constexpr int PF_QBOX = 128 * 128; // bytes of one 128-row x 64-element bf16 box (Q)
constexpr int PF_KBOX = 64 * 128;  // bytes of one 64-row x 64-element bf16 box (K, V)
constexpr float PF_RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

struct PrefillArgs {
  const float* lambda;
  __nv_bfloat16* out;   // [B, Hout, Lq, 128]
  int B, Hout, Hq, Hkv, Lq, Lk;
  int v1;               // layout: 1 = V1 (q1/q2, k1/k2 tensors), 0 = V2 (pairs of Q heads)
  int causal, rms;
  float eps, scale_log2;
  int n_rb;             // row blocks per head
  int rb_group;         // launch order: groups of rb_group row blocks of one head are adjacent (>= 1)
  // Precision policy: P is stored as bf16 P_hi plus a bf16 residual P_lo (a
  // second PV MMA) for heads with |1 - lambda| < resid_tau.  The difference
  // O1/l1 - lambda*O2/l2 amplifies P's bf16 rounding (2^-9) by about
  // (1+|lambda|)/|1-lambda| when the two maps are alike; below resid_tau that
  // factor would exceed ~12 and the residual restores ~2^-17.
  float resid_tau;
  Watch watch;
  // Training outputs (null for inference): per row and map the log-sum-exp of
  // the scaled scores in log2 units, lse[B, Hout, 2, Lq] (+inf for a row that
  // sees no key), and the normalised map outputs O_m / l_m, o_maps[B, Hout, 2,
  // Lq, 128] bf16; with RMSNorm also the row's 1/rms, rstd[B, Hout, Lq] (0 for
  // a row that sees no key).
  float* lse;
  __nv_bfloat16* o_maps;
  float* rstd;
  // With RMSNorm the backward's dlambda = -sum dX . O_2 is a small remainder
  // of large terms: dX is orthogonal to the difference output X, and O_2 is
  // nearly parallel to X when the maps are alike.  The training forward
  // therefore stores map 2's normalised output as its component orthogonal to
  // X, O_2 - c X with c = <O_2, X> / <X, X> formed in f32 (o_maps[.., 1, ..]),
  // and per row o2c[B, Hout, Lq] = c eps r^2 (0 for a row that sees no key).
  // Then dX . O_2 = dX . (O_2 - c X) + c dX . X with dX . X = <y, dY> eps r^2,
  // so D_2 = dX . (O_2 - c X) + o2c <y, dY>, and the bf16 rounding of the
  // stored operand scales with the orthogonal part only.
  float* o2c;
  // Single-map mode (PF_SINGLE): output heads are pairs of independent
  // heads (2h, 2h+1) over one KV head, each with its own lambda[2h + m] (which
  // sets only its residual choice); the kernel writes each head's normalised
  // map output O_m / l_m in f32, o_f32[B, Hout, 2, Lq, 128] = [B, 2 Hout, Lq,
  // 128], and nothing else.
  float* o_f32;
};

// What a launch writes (template argument of prefill_kernel).
constexpr int PF_INFER = 0;    // out
constexpr int PF_TRAIN = 1;    // out, lse, o_maps [, rstd]
constexpr int PF_SINGLE = 2;   // o_f32 only

template <int DQK>
struct PfSmem {
  static constexpr int QTILE = PF_BM * DQK * 2;  // bytes of one Q tile
  alignas(1024) uint8_t q[2][QTILE];
  alignas(1024) uint8_t k[PF_NS][2 * PF_KBOX];   // V2: K tile (dims 0-63 box, 64-127 box); V1: K1 box, K2 box
  alignas(1024) uint8_t v[PF_NS][2 * PF_KBOX];   // V tile, dv 0-63 box then 64-127 box
  alignas(16) uint8_t stage[8][16 * 128];          // per softmax warp: 16 output rows of 64 bf16 (epilogue)
  float l[2][PF_BM];
  float ss[2][PF_BM];
  float sp[2][PF_BM];     // epilogue exchange of <O_2, X> partial sums (training, RMSNorm)
  alignas(8) uint64_t q_full;
  uint64_t k_full[PF_NS];
  uint64_t v_full[PF_NS];
  uint64_t kv_empty[PF_NS];
  uint64_t s_full[2][2];  // [map][buffer]
  uint64_t p_full[2][2];
  uint64_t s_free[2][2];  // PV_m of the buffer's last tile complete: S may be overwritten
  uint64_t o_done[2];     // PV_m(j) complete (one phase per tile)
  uint64_t o_final;
  uint64_t xl;      // epilogue exchange of l (256 arrivals)
  uint64_t xs;      // epilogue exchange of RMS partial sums (256 arrivals)
  uint64_t drain[2];      // per issuer: all its MMAs complete
  uint32_t tmem_base;
  int abort_flag;
};

// Bounded wait of a whole warp: lane 0 waits, then broadcasts the outcome.
// With VOTE, every lane first tests the phase and the warp votes, so a phase
// that is already complete costs one test and one vote, with no divergence.
// Measured per kernel: the vote helps the prefill's softmax warps (V1 +3 %)
// and is neutral in the query-stationary backward kernel; the key-stationary
// one runs 8 % slower with it and keeps the plain form.
template <bool VOTE = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          const Watch& w) {
  if (VOTE && __all_sync(0xffffffffu, mbar_test(bar, parity))) return true;
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, abort_flag, w);
  return __shfl_sync(0xffffffffu, ok, 0);
}

// P = 2^(s*scale_log2 - mu) for the 64 keys of one row, stored over S in TMEM
// as bf16 P_hi (columns [0,32)) and, with RESID, the bf16 residual P - P_hi
// (columns [32,64)); returns the row sum of P in f32.  Chunks of 16 keys: each
// chunk's words go to TMEM as soon as they are ready (keeps register pressure
// down; the stores are asynchronous).
template <bool RESID>
__device__ __forceinline__ float pf_exp_store(const float (&s)[PF_BN], float2 sc2, float2 nm2, uint32_t tS) {
  const float2 neg1 = make_float2(-1.f, -1.f);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int ch = 0; ch < PF_BN / 16; ++ch) {
    uint32_t pk[8], pl[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = ch * 16 + 2 * i;
      const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), sc2, nm2);
      const float2 p = make_float2(ex2(x.x), ex2(x.y));
      acc[i & 3] = __fadd2_rn(acc[i & 3], p);
      const uint32_t hi = pack_bf16(p.x, p.y);
      pk[i] = hi;
      if (RESID) {
        const float2 hf = make_float2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xFFFF0000u));
        const float2 lo = __ffma2_rn(hf, neg1, p);   // p - hi, exact
        pl[i] = pack_bf16(lo.x, lo.y);
      }
    }
    tmem_st8p(tS + ch * 8, pk);
    if (RESID) tmem_st8p(tS + 32 + ch * 8, pl);
  }
  const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
  const float2 a03 = __fadd2_rn(a01, a23);
  return a03.x + a03.y;
}

// Store 64 bf16 columns of each of a warp's 32 rows (thread i holds row
// row_w0 + i): the warp stages 16 rows at a time in its shared buffer (16-byte
// chunks XOR-swizzled by row, conflict-free both ways) and writes them back as
// 4 rows x 128 contiguous bytes per instruction (a direct store of each
// thread's own row would touch 32 lines per instruction).  base points at
// column 0 of row 0; rows are `stride` elements apart (128 by default); rows
// >= Lq are skipped.
__device__ __forceinline__ void pf_store_rows(uint8_t* st, const float (&y)[64], __nv_bfloat16* base, int row_w0,
                                              int Lq, int lane, int stride = PF_DV) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    if ((lane >> 4) == half) {
      const int rr = lane & 15;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 v;
        v.x = pack_bf16(y[8 * c + 0], y[8 * c + 1]);
        v.y = pack_bf16(y[8 * c + 2], y[8 * c + 3]);
        v.z = pack_bf16(y[8 * c + 4], y[8 * c + 5]);
        v.w = pack_bf16(y[8 * c + 6], y[8 * c + 7]);
        *reinterpret_cast<uint4*>(st + rr * 128 + ((c ^ (rr & 7)) << 4)) = v;
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = 4 * i + (lane >> 3), c = lane & 7;
      const int row = row_w0 + 16 * half + rr;
      const uint4 v = *reinterpret_cast<const uint4*>(st + rr * 128 + ((c ^ (rr & 7)) << 4));
      if (row < Lq) *reinterpret_cast<uint4*>(base + (size_t)row * stride + c * 8) = v;
    }
    __syncwarp();
  }
}

// f32 variant of pf_store_rows: the warp stages all 32 rows (256 bytes each,
// 16-byte chunks XOR-swizzled by row, conflict-free both ways) in 8 KB and
// writes them back as 2 rows x 256 contiguous bytes per instruction.
constexpr int PF_STAGE_F32 = 32 * 64 * 4;
__device__ __forceinline__ void pf_store_rows_f32(uint8_t* st, const float (&y)[64], float* base, int row_w0,
                                                  int Lq, int lane) {
#pragma unroll
  for (int c = 0; c < 16; ++c)
    *reinterpret_cast<float4*>(st + lane * 256 + ((c ^ (lane & 15)) << 4)) =
        make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int rr = 2 * i + (lane >> 4), c = lane & 15;
    const float4 v = *reinterpret_cast<const float4*>(st + rr * 256 + ((c ^ (rr & 15)) << 4));
    const int row = row_w0 + rr;
    if (row < Lq) *reinterpret_cast<float4*>(base + (size_t)row * PF_DV + c * 4) = v;
  }
  __syncwarp();
}

// MODE: PF_INFER, PF_TRAIN (also the training outputs lse, o_maps) or
// PF_SINGLE (single-map outputs in f32); a template argument so the inference
// kernel carries none of the other modes' code.
template <int DQK, int MODE = PF_INFER>
__global__ void __launch_bounds__(PF_THREADS, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ1, const __grid_constant__ CUtensorMap tmQ2,
               const __grid_constant__ CUtensorMap tmK1, const __grid_constant__ CUtensorMap tmK2,
               const __grid_constant__ CUtensorMap tmV, PrefillArgs a) {
  static_assert(DQK == 64 || DQK == 128, "QK width 64 or 128");
  static_assert(sizeof(PfSmem<DQK>::k) + sizeof(PfSmem<DQK>::v) >= 8 * PF_STAGE_F32 &&
                    offsetof(PfSmem<DQK>, v) == offsetof(PfSmem<DQK>, k) + sizeof(PfSmem<DQK>::k),
                "the single-map epilogue stages 8 warps' rows in the contiguous K/V stages");
  constexpr bool TRAIN = MODE == PF_TRAIN, SINGLE = MODE == PF_SINGLE;
  constexpr int QBOXES = DQK / 64;
  extern __shared__ uint8_t smem_raw[];
  PfSmem<DQK>& S = *reinterpret_cast<PfSmem<DQK>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &S.abort_flag;

  // ---- work unit: heaviest row blocks first (causal), in groups of
  // rb_group row blocks of one head that are adjacent in the launch order, so
  // that co-resident CTAs of a head read its K/V tiles together from L2 ----
  const int BH = a.B * a.Hout;
  int rb, bh;
  {
    const int R = a.rb_group, n_full = a.n_rb / R;
    const long long idx = blockIdx.x, in_full = (long long)n_full * R * BH;
    if (idx < in_full) {
      const int rg = (int)(idx / ((long long)R * BH)), rem = (int)(idx % ((long long)R * BH));
      bh = rem / R;
      rb = a.n_rb - 1 - (rg * R + rem % R);
    } else {                                   // the last n_rb % R row blocks
      const int rr = a.n_rb - n_full * R, rem = (int)(idx - in_full);
      bh = rem / rr;
      rb = a.n_rb - 1 - (n_full * R + rem % rr);
    }
  }
  const int b = bh / a.Hout, h = bh % a.Hout;
  const int r0 = rb * PF_BM;
  int qh1, qh2, g;
  if (a.v1) { qh1 = qh2 = h; g = h / (a.Hq / a.Hkv); }
  else { qh1 = 2 * h; qh2 = 2 * h + 1; g = qh1 / (a.Hq / a.Hkv); }
  const int zq1 = b * a.Hq + qh1, zq2 = b * a.Hq + qh2, zkv = b * a.Hkv + g;
  // keys visible to the last row of the block
  long long kend = a.causal ? (long long)min(r0 + PF_BM, a.Lq) - 1 + (a.Lk - a.Lq) + 1 : a.Lk;
  kend = max(0LL, min(kend, (long long)a.Lk));
  const int nT = (int)((kend + PF_BN - 1) / PF_BN);
  // Residual choice per map: one lambda per output head, or in single-map
  // mode each head's own.  The training forward with RMSNorm keeps it for
  // every head: the backward's dlambda = -sum dX . O_2 is then a small
  // remainder of terms (dX is orthogonal to X, O_2 nearly parallel to it
  // when the maps are alike), and the 2^-9 rounding of a bf16-only P in O_2
  // would not be orthogonal to X.
  const bool all_resid = TRAIN && a.rms;
  const bool resid1 = all_resid || fabsf(1.f - a.lambda[SINGLE ? 2 * h : h]) < a.resid_tau;
  const bool resid2 = SINGLE ? fabsf(1.f - a.lambda[2 * h + 1]) < a.resid_tau : resid1;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&S.q_full), 1);
    for (int i = 0; i < PF_NS; ++i) {
      mbar_init(smem_u32(&S.k_full[i]), 1);
      mbar_init(smem_u32(&S.v_full[i]), 1);
      mbar_init(smem_u32(&S.kv_empty[i]), 1);
    }
    for (int m = 0; m < 2; ++m) {
      for (int bb = 0; bb < 2; ++bb) {
        mbar_init(smem_u32(&S.s_full[m][bb]), 1);
        mbar_init(smem_u32(&S.p_full[m][bb]), 4);   // one arrival per softmax warp of the map
        mbar_init(smem_u32(&S.s_free[m][bb]), 1);
      }
      mbar_init(smem_u32(&S.o_done[m]), 1);
      mbar_init(smem_u32(&S.drain[m]), 1);
    }
    mbar_init(smem_u32(&S.o_final), 1);
    mbar_init(smem_u32(&S.xl), 8);   // one arrival per softmax warp
    mbar_init(smem_u32(&S.xs), 8);
    S.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(&S.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0 && nT > 0) {
      tma_prefetch_desc(&tmK1);
      tma_prefetch_desc(&tmV);
      const uint32_t qb = smem_u32(&S.q_full);
      mbar_expect_tx(qb, 2 * PfSmem<DQK>::QTILE);
      for (int x = 0; x < QBOXES; ++x) {
        tma_load_3d(smem_u32(S.q[0]) + x * PF_QBOX, &tmQ1, qb, 64 * x, r0, zq1);
        tma_load_3d(smem_u32(S.q[1]) + x * PF_QBOX, &tmQ2, qb, 64 * x, r0, zq2);
      }
      int last_use[PF_NS];
      for (int i = 0; i < PF_NS; ++i) last_use[i] = -1;
      for (int j = 0; j < nT; ++j) {
        const int st = j % PF_NS, use = j / PF_NS;
        if (use > 0 && !wait_bar(smem_u32(&S.kv_empty[st]), (use - 1) & 1, abort_flag, a.watch)) break;
        const uint32_t kb = smem_u32(&S.k_full[st]), vb = smem_u32(&S.v_full[st]);
        const uint32_t kd = smem_u32(S.k[st]), vd = smem_u32(S.v[st]);
        mbar_expect_tx(kb, 2 * PF_KBOX);
        if (a.v1) {
          tma_load_3d(kd, &tmK1, kb, 0, j * PF_BN, zkv);
          tma_load_3d(kd + PF_KBOX, &tmK2, kb, 0, j * PF_BN, zkv);
        } else {
          tma_load_3d(kd, &tmK1, kb, 0, j * PF_BN, zkv);
          tma_load_3d(kd + PF_KBOX, &tmK1, kb, 64, j * PF_BN, zkv);
        }
        mbar_expect_tx(vb, 2 * PF_KBOX);
        tma_load_3d(vd, &tmV, vb, 0, j * PF_BN, zkv);
        tma_load_3d(vd + PF_KBOX, &tmV, vb, 64, j * PF_BN, zkv);
        last_use[st] = use;
      }
      // Every copy issued must have landed before the CTA may exit (returns at
      // once when the consumer has already seen the phase).
      drain_bar(qb, 0, a.watch.status);
      for (int i = 0; i < PF_NS; ++i)
        if (last_use[i] >= 0) {
          drain_bar(smem_u32(&S.k_full[i]), last_use[i] & 1, a.watch.status);
          drain_bar(smem_u32(&S.v_full[i]), last_use[i] & 1, a.watch.status);
        }
    }
  } else if (warp >= 9) {
    // --------------------------------------------------------- MMA issuers --
    if (lane == 0 && nT > 0) {
      // Descriptor words computed once; per MMA only the low word moves.
      constexpr uint32_t HI = umma_desc_hi(1024);
      constexpr uint32_t KSTAGE = (2 * PF_KBOX) >> 4;          // stage stride in 16-byte units
      const int issuer = warp - 9;                             // 0: PV, 1: QK
      bool ok = true;
      if (issuer == 0) {
        // PV_1(j), PV_2(j) as soon as the softmax has stored each map's P.
        constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, PF_DV, true);
        const uint32_t v_lo0 = umma_desc_lo(smem_u32(S.v[0]), PF_KBOX);
        for (int j = 0; ok && j < nT; ++j) {
          const int bb = j & 1, ph = (j >> 1) & 1;
          const uint32_t vlo = v_lo0 + (uint32_t)(j % PF_NS) * KSTAGE;
          if (!(ok = wait_bar(smem_u32(&S.v_full[j % PF_NS]), (j / PF_NS) & 1, abort_flag, a.watch))) break;
          for (int m = 0; m < 2; ++m) {
            if (!(ok = wait_bar(smem_u32(&S.p_full[m][bb]), ph, abort_flag, a.watch))) break;
            tc_fence_after();
            const uint32_t p = tmem + (uint32_t)(m * 128 + bb * 64), o = tmem + 256 + m * 128;
#pragma unroll
            for (int s = 0; s < PF_BN / 16; ++s)
              mma_ts_w(o, p + s * 8, vlo + (uint32_t)(s * (2048 >> 4)), HI, IDESC_PV, (j > 0 || s > 0));
            if (m ? resid2 : resid1) {
#pragma unroll
              for (int s = 0; s < PF_BN / 16; ++s)   // residual part of P
                mma_ts_w(o, p + 32 + s * 8, vlo + (uint32_t)(s * (2048 >> 4)), HI, IDESC_PV, 1);
            }
            mma_commit(smem_u32(&S.o_done[m]));
            mma_commit(smem_u32(&S.s_free[m][bb]));
          }
          if (!ok) break;
          // The stage's K was read by S(j), complete before P(j) existed.
          mma_commit(smem_u32(&S.kv_empty[j % PF_NS]));
        }
        if (ok) mma_commit(smem_u32(&S.o_final));
      } else {
        // S_m(j) once K(j) has landed and, for j >= 2, PV_m(j-2) -- the last
        // reader of the buffer -- has completed.
        constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, PF_BN, false);
        const uint32_t q_lo0 = umma_desc_lo(smem_u32(S.q[0]), 16), q_lo1 = umma_desc_lo(smem_u32(S.q[1]), 16);
        const uint32_t k_lo0 = umma_desc_lo(smem_u32(S.k[0]), 16);
        const uint32_t km_off = a.v1 ? (PF_KBOX >> 4) : 0u;         // V1: K2 box follows the K1 box
        ok = wait_bar(smem_u32(&S.q_full), 0, abort_flag, a.watch);
        for (int j = 0; ok && j < nT; ++j) {
          const int bb = j & 1;
          if (!(ok = wait_bar(smem_u32(&S.k_full[j % PF_NS]), (j / PF_NS) & 1, abort_flag, a.watch))) break;
          for (int m = 0; m < 2; ++m) {
            if (j >= 2 && !(ok = wait_bar(smem_u32(&S.s_free[m][bb]), ((j - 2) >> 1) & 1, abort_flag, a.watch)))
              break;
            tc_fence_after();
            const uint32_t klo = k_lo0 + (uint32_t)(j % PF_NS) * KSTAGE + (m ? km_off : 0u);
            const uint32_t qlo = m ? q_lo1 : q_lo0;
            const uint32_t d = tmem + (uint32_t)(m * 128 + bb * 64);
#pragma unroll
            for (int s = 0; s < DQK / 16; ++s) {
              const uint32_t qo = (uint32_t)((s >> 2) * (PF_QBOX >> 4) + (s & 3) * 2);
              const uint32_t ko = (uint32_t)((s >> 2) * (PF_KBOX >> 4) + (s & 3) * 2);
              mma_ss_w(d, qlo + qo, HI, klo + ko, HI, IDESC_QK, s > 0);
            }
            mma_commit(smem_u32(&S.s_full[m][bb]));
          }
        }
      }
      // Every MMA this thread issued must have completed before TMEM is freed.
      mma_commit(smem_u32(&S.drain[issuer]));
      drain_bar(smem_u32(&S.drain[issuer]), 0, a.watch.status);
    }
  } else {
    // ------------------------------------------------- softmax (two groups) --
    const int m = warp >> 2;                 // map
    const int wq = warp & 3;                 // TMEM lane quadrant
    const int r = threadIdx.x & 127;         // row within the block
    const int rg = r0 + r;                   // query row
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tO = tmem + lane_off + 256 + m * 128;
    // last visible key of this row
    const long long lastk = a.causal ? min((long long)a.Lk - 1, (long long)rg + (a.Lk - a.Lq)) : (long long)a.Lk - 1;
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nT; ++j) {
      const int bb = j & 1;
      const uint32_t tS = tmem + lane_off + m * 128 + bb * 64;
      if (!(ok = warp_wait<true>(smem_u32(&S.s_full[m][bb]), (j >> 1) & 1, abort_flag, a.watch))) break;
      tc_fence_after();
      float s[PF_BN];
      {
        uint32_t rr[PF_BN];
        tmem_ld32p(tS, rr);
        tmem_ld32p(tS + 32, rr + 32);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < PF_BN; ++i) s[i] = __uint_as_float(rr[i]);
      }
      const long long lim = lastk - (long long)j * PF_BN;   // columns > lim are masked
      if (lim < PF_BN - 1) {
#pragma unroll
        for (int c = 0; c < PF_BN; ++c)
          if (c > lim) s[c] = -INFINITY;
      }
      // row max: four independent 3-input max chains
      float mx;
      {
        float c0 = fmaxf(s[0], s[1]), c1 = fmaxf(s[2], s[3]), c2 = fmaxf(s[4], s[5]), c3 = fmaxf(s[6], s[7]);
#pragma unroll
        for (int c = 8; c < PF_BN; c += 8) {
          c0 = fmax3(c0, s[c], s[c + 1]);
          c1 = fmax3(c1, s[c + 2], s[c + 3]);
          c2 = fmax3(c2, s[c + 4], s[c + 5]);
          c3 = fmax3(c3, s[c + 6], s[c + 7]);
        }
        mx = fmax3(c0, c1, fmaxf(c2, c3));
      }
      const float mxs = mx * a.scale_log2;
      float alpha = 1.f;
      if (mxs > m_run + PF_RESCALE_THRESHOLD) {
        if (m_run != -INFINITY && j > 0) alpha = ex2(m_run - mxs);
        m_run = mxs;
      }
      const float mu = m_run == -INFINITY ? 0.f : m_run;
      const float2 nm2 = make_float2(-mu, -mu);
      // The residual choice is per head: branch once per tile, so each
      // variant's exp loop is one straight-line block the scheduler can
      // interleave across key pairs.
      const float rowsum =
          (m ? resid2 : resid1) ? pf_exp_store<true>(s, sc2, nm2, tS) : pf_exp_store<false>(s, sc2, nm2, tS);
      l_run = l_run * alpha + rowsum;
      // tcgen05.ld/st are warp-collective: rescale if any row of the warp needs
      // it (rows whose alpha is 1 multiply by 1).  O_m must be complete first:
      // wait for PV_m(j-1) (o_done phase j-1; PV_m(j-2) is known complete since
      // S_m(j) was issued only after s_free showed it, so the parity is
      // unambiguous).
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        if (!(ok = warp_wait<true>(smem_u32(&S.o_done[m]), (j - 1) & 1, abort_flag, a.watch))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < PF_DV / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32p(tO + c * 32, rr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
          tmem_st32p(tO + c * 32, rr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.p_full[m][bb]));
    }

    // --------------------------------------------------------- epilogue --
    // Rows that saw no key (l == 0) output zeros.
    const float lam = SINGLE ? 0.f : a.lambda[h];
    float y[64];
    bool have = false;
    float kx = 0.f;   // training with RMSNorm: c / rs, so that c X = kx y once y holds rs X
    if (ok && nT > 0) {
      S.l[m][r] = l_run;
      // the warp's stores, then one arrival for it
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.xl));
      ok = warp_wait<true>(smem_u32(&S.xl), 0, abort_flag, a.watch) &&
           warp_wait<true>(smem_u32(&S.o_final), 0, abort_flag, a.watch);
      if (ok && SINGLE) {
        tc_fence_after();
        have = true;
      } else if (ok) {
        tc_fence_after();
        const float l1 = S.l[0][r], l2 = S.l[1][r];
        const float c1 = l1 > 0.f ? 1.f / l1 : 0.f;
        const float c2 = l2 > 0.f ? lam / l2 : 0.f;
        const float i2 = l2 > 0.f ? 1.f / l2 : 0.f;
        float sp = 0.f;   // <O_2 / l_2, X> over this thread's 64 columns (training, RMSNorm)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o1[32], o2[32];
          tmem_ld32p(tmem + lane_off + 256 + m * 64 + c * 32, o1);
          tmem_ld32p(tmem + lane_off + 384 + m * 64 + c * 32, o2);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            y[c * 32 + i] = __fsub_rn(__fmul_rn(__uint_as_float(o1[i]), c1), __fmul_rn(__uint_as_float(o2[i]), c2));
            if (TRAIN) sp = fmaf(__uint_as_float(o2[i]) * i2, y[c * 32 + i], sp);
          }
        }
        have = true;
        if (a.rms) {
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < 64; ++i) ss = fmaf(y[i], y[i], ss);
          S.ss[m][r] = ss;
          if (TRAIN) S.sp[m][r] = sp;
          __threadfence_block();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&S.xs));
          ok = warp_wait<true>(smem_u32(&S.xs), 0, abort_flag, a.watch);
          have = ok;
          if (ok) {
            const float xx = S.ss[0][r] + S.ss[1][r];
            const float rs = rsqrtf(xx / (float)PF_DV + a.eps);
#pragma unroll
            for (int i = 0; i < 64; ++i) y[i] *= rs;
            if (TRAIN) {
              const float cq = (l_run > 0.f && xx > 0.f) ? (S.sp[0][r] + S.sp[1][r]) / xx : 0.f;
              kx = cq / rs;
              if (m == 0 && rg < a.Lq) {
                a.rstd[((size_t)b * a.Hout + h) * a.Lq + rg] = l_run > 0.f ? rs : 0.f;
                a.o2c[((size_t)b * a.Hout + h) * a.Lq + rg] = cq * a.eps * rs * rs;
              }
            }
          }
        }
      }
    } else if (nT == 0) {
#pragma unroll
      for (int i = 0; i < 64; ++i) y[i] = 0.f;
      have = true;
      if (TRAIN && a.rms && m == 0 && rg < a.Lq) {
        a.rstd[((size_t)b * a.Hout + h) * a.Lq + rg] = 0.f;
        a.o2c[((size_t)b * a.Hout + h) * a.Lq + rg] = 0.f;
      }
    }
    have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;   // warp-uniform (ok is)
    const int row_w0 = r0 + wq * 32;                          // first row of this warp
    if (have && !SINGLE)
      pf_store_rows(S.stage[warp], y, a.out + (((size_t)b * a.Hout + h) * a.Lq) * PF_DV + m * 64, row_w0, a.Lq,
                    lane);
    // Training outputs: this map's log-sum-exp, and 64 columns of both
    // normalised map outputs; with RMSNorm map 2's is stored as O_2 - c X.
    // Map 2 goes first: its correction reads y (rs X, just stored) before map
    // 1's values overwrite it.
    if (TRAIN && have) {
      const size_t stat = ((size_t)b * a.Hout + h) * 2;
      if (rg < a.Lq) a.lse[(stat + m) * a.Lq + rg] = l_run > 0.f ? m_run + log2f(l_run) : INFINITY;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int mm = 1 - t;
        const float inv = (nT > 0 && S.l[mm][r] > 0.f) ? 1.f / S.l[mm][r] : 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          if (nT > 0) {
            tmem_ld32p(tmem + lane_off + 256 + mm * 128 + m * 64 + c * 32, o);
            tmem_wait_ld();
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float on = nT > 0 ? __uint_as_float(o[i]) * inv : 0.f;
            y[c * 32 + i] = (mm == 1 && kx != 0.f) ? __fsub_rn(on, __fmul_rn(kx, y[c * 32 + i])) : on;
          }
        }
        pf_store_rows(S.stage[warp], y, a.o_maps + ((stat + mm) * a.Lq) * PF_DV + m * 64, row_w0, a.Lq, lane);
      }
    }
    // Single-map outputs: 64 columns of each head's O_m / l_m in f32.  Every
    // MMA has completed (o_final) and every K/V copy has been consumed, so the
    // K/V stages are free: each warp stages its rows in 8 KB of them.
    if (SINGLE && have) {
      const size_t stat = ((size_t)b * a.Hout + h) * 2;
      uint8_t* st = &S.k[0][0] + (size_t)warp * PF_STAGE_F32;
#pragma unroll
      for (int mm = 0; mm < 2; ++mm) {
        const float inv = (nT > 0 && S.l[mm][r] > 0.f) ? 1.f / S.l[mm][r] : 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          if (nT > 0) {
            tmem_ld32p(tmem + lane_off + 256 + mm * 128 + m * 64 + c * 32, o);
            tmem_wait_ld();
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) y[c * 32 + i] = nT > 0 ? __uint_as_float(o[i]) * inv : 0.f;
        }
        pf_store_rows_f32(st, y, a.o_f32 + ((stat + mm) * a.Lq) * PF_DV + m * 64, row_w0, a.Lq, lane);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace da
