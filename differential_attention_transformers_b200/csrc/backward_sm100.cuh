// backward_sm100.cuh -- gradients of the V2 differential attention prefill on tcgen05.
//
// Forward ("差分注意力" tutorial, section 差分思路 and Step 2; V2 layout from
// its section V1 到 V2 的 diff): per diff pair h, with maps m = 1, 2 on Q heads
// (2h, 2h+1) and the pair's KV head g,
//   A_m = softmax(Q_m K^T / sqrt(d)),  O = (A_1 - lambda A_2) V.
// Chain rule, given dO (the pages print no backward):
//   dV  = sum over the pairs of g of (A_1 - lambda A_2)^T dO
//   dW  = dO V^T,  D_m = rowsum(dO * O_m)  with O_m = A_m V
//   dS_1 = A_1 (dW - D_1),  dS_2 = -lambda A_2 (dW - D_2)
//   dQ_m = dS_m K / sqrt(d),  dK = sum over the group of dS_m^T Q_m / sqrt(d)
//   dlambda = -sum(dO * O_2)
// A_m is recomputed from the scores and the forward's per-row log-sum-exp
// (log2 units): A_m = 2^(S_m log2(e)/sqrt(d) - lse_m).
//
// Three kernels:
//   bwd_prep_kernel  D_m per row from dO and the forward's normalised map
//                    outputs, and the log-sum-exp, both negated into a padded
//                    layout (so the kernels below add them), and
//                    per-block partial sums of dlambda (reduced in a fixed
//                    order by bwd_dlambda_kernel, so the result is
//                    deterministic).
//   bwd_dq_kernel    query-stationary: one CTA per 128 rows of one Q head (one
//                    map).  Per 128-key tile: S = Q K^T and dP = dO V^T into
//                    TMEM (N = 128 products, with Q and dO in TMEM as their A
//                    operands), dS = c P (dP - D) written to shared memory as
//                    bf16, then dQ += dS K with dS as the shared A operand.
//                    The one score buffer is free as soon as the elementwise
//                    warps have loaded it, so the products of tile j + 1 run
//                    while tile j's elementwise phase does.
//   bwd_dkv_kernel   key-stationary: one CTA per 128 keys of one KV head.  Per
//                    64-row block, the two maps of each diff pair of the
//                    group in turn: S_m^T = K Q_m^T into TMEM, and once per
//                    pair dP^T = V dO^T (the maps share dO).  dS_m^T and
//                    (P_1 - lambda P_2)^T are written back as bf16, and
//                    dK += dS_m^T Q_m, dV += (P_1 - lambda P_2)^T dO take
//                    them as the TMEM operands.
// Computing dQ apart from dK/dV recomputes S and dP once more but needs no
// atomics, and each kernel fits TMEM (512 columns each).
// Both MMA kernels use the forward's pipeline: a TMA producer warp, one
// issuing thread for the S-type products and one for the accumulating ones,
// and eight warps (two per TMEM lane quadrant, one per 32-column chunk)
// between them.
#pragma once

#include "common.cuh"
#include "prefill_sm100.cuh"

namespace da {

// Warps 0-7 elementwise (warp w: TMEM lane quadrant w & 3, 32-column chunk
// w >> 2 of each 64-column buffer), 8 producer and TMEM owner, 9 accumulating
// MMAs, 10 S-type MMAs.  In every bf16 buffer a chunk keeps its values in its
// own 32 columns -- the hi parts in the first 16, the residuals (when used) in
// the next 16 -- so no warp overwrites scores another warp has yet to load.
constexpr int BW_THREADS = 352;
constexpr int BW_EW = 256;        // elementwise threads
constexpr int BW_EW_WARPS = BW_EW / 32;   // arrivals on the elementwise warps' barriers: one per warp
constexpr int BW_NS = 3;          // pipeline stages of the key-stationary kernel
constexpr int BWQ_NS = 3;         // K/V stages of the query-stationary kernel
constexpr int BWQ_BN = 128;       // keys per tile of the query-stationary kernel
constexpr int BW_RB = 64;         // rows per step of the key-stationary kernel

struct BwdArgs {
  const float* lambda;   // [Hp]
  const float* nlse;     // [B, Hp, 2, Lp] minus the log-sum-exp (log2 units), -inf past Lq
  const float* ndd;      // [B, Hp, 2, Lp] -D_m, 0 past Lq
  __nv_bfloat16* dq;     // [B, Hq, Lq, 128]; V1: dQ1 [B, Hq/2, Lq, 64]
  __nv_bfloat16* dk;     // [B, Hkv, Lk, 128]; V1: dK1 [B, Hkv, Lk, 64]
  __nv_bfloat16* dv;     // [B, Hkv, Lk, 128]
  __nv_bfloat16* dq2;    // V1 only: dQ2 [B, Hq/2, Lq, 64]
  __nv_bfloat16* dk2;    // V1 only: dK2 [B, Hkv, Lk, 64]
  int B, Hq, Hkv, Lq, Lk, Lp;
  int causal;
  float scale, scale_log2;
  // V2 heads with |1 - lambda| < resid_tau keep the bf16 residual of dS in
  // the key-stationary kernel (a second MMA for dK): with alike maps the sum
  // dK = sum over the pair's maps of dS_m^T Q_m cancels, and the separate bf16
  // roundings of the two maps' operands would be amplified as in the forward.
  // dV needs none: its operand is (P_1 - lambda P_2)^T, formed in f32 and
  // rounded once.  V1 keeps dK_1 and dK_2 apart, so it needs none either.
  float resid_tau;
  Watch watch;
};

// ------------------------------------------------------------------- prep --
struct BwdPrepArgs {
  const __nv_bfloat16* dout;    // [B, Hp, Lq, 128]
  const __nv_bfloat16* o_maps;  // [B, Hp, 2, Lq, 128]
  const float* lse;             // [B, Hp, 2, Lq]
  float* nlse;                  // [B, Hp, 2, Lp] -lse, -inf past Lq
  float* ndd;                   // [B, Hp, 2, Lp] -D_m, 0 past Lq
  float* part;                  // [B * Hp, Lp / 64] partial sums of -D_2
  int B, Hp, Lq, Lp;
  const float* d_in;            // [B, Hp, 2, Lq] D_m formed upstream (V1 with RMSNorm), or null
};

// grid (Lp / 64, B * Hp), 256 threads: warp w handles rows 8w .. 8w+7 of the
// block, four lanes a row (lane l: row 8w + l/4, columns 32 (l%4) .. +31), so
// the loads of all eight rows are in flight at once.
__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdPrepArgs a) {
  __shared__ float wsum[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int row = blockIdx.x * 64 + warp * 8 + (lane >> 2), part = lane & 3;
  float d[2] = {0.f, 0.f};
  if (a.d_in != nullptr) {
    if (row < a.Lq) {
      d[0] = a.d_in[((size_t)bh * 2) * a.Lq + row];
      d[1] = a.d_in[((size_t)bh * 2 + 1) * a.Lq + row];
    }
  } else {
    float s[2] = {0.f, 0.f};
    if (row < a.Lq) {
      const size_t col = (size_t)part * 32;
      const uint4* go = reinterpret_cast<const uint4*>(a.dout + ((size_t)bh * a.Lq + row) * 128 + col);
      const uint4* o1 = reinterpret_cast<const uint4*>(a.o_maps + (((size_t)bh * 2) * a.Lq + row) * 128 + col);
      const uint4* o2 = reinterpret_cast<const uint4*>(a.o_maps + (((size_t)bh * 2 + 1) * a.Lq + row) * 128 + col);
      uint4 gv[4], v1[4], v2[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        gv[q] = go[q];
        v1[q] = o1[q];
        v2[q] = o2[q];
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv[q]);
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&v1[q]);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v2[q]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 gf = __bfloat1622float2(g2[e]), af = __bfloat1622float2(a2[e]), bf = __bfloat1622float2(b2[e]);
          s[0] = fmaf(gf.x, af.x, s[0]);
          s[0] = fmaf(gf.y, af.y, s[0]);
          s[1] = fmaf(gf.x, bf.x, s[1]);
          s[1] = fmaf(gf.y, bf.y, s[1]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {   // the row's four lanes; rows past Lq add zeros
      s[m] += __shfl_xor_sync(0xffffffffu, s[m], 1);
      s[m] += __shfl_xor_sync(0xffffffffu, s[m], 2);
      d[m] = s[m];
    }
  }
  if (part < 2) {   // lane part m of the row writes map m's values
    const size_t at = ((size_t)bh * 2 + part) * a.Lp + row;
    a.ndd[at] = -d[part];
    a.nlse[at] = row < a.Lq ? -a.lse[((size_t)bh * 2 + part) * a.Lq + row] : -INFINITY;
  }
  // dlambda partial: the sum of -D_2 over the warp's eight rows, then the block's
  float acc = part == 0 ? -d[1] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) wsum[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += wsum[w];
    a.part[(size_t)bh * (a.Lp / 64) + blockIdx.x] = t;
  }
}

// One thread per pair: dlambda[h] = sum over batch and row blocks, fixed order.
__global__ void bwd_dlambda_kernel(const float* part, float* dlambda, int B, int Hp, int nblk) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= Hp) return;
  double t = 0.0;
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < nblk; ++i) t += (double)part[((size_t)b * Hp + h) * nblk + i];
  dlambda[h] = (float)t;
}

// ------------------------------------------------------------ dQ (Q-stationary) --
struct BwQSmem {
  // K/V stage st: the K tile (two [128 keys][64] boxes of the QK width; V1
  // one), then the V tile (two boxes).  Stage 2 first holds the Q tile (two
  // [128 rows][64] boxes; V1 one) and the dO tile: the elementwise warps copy
  // them into TMEM (qt_full) before a K/V tile is loaded there.
  alignas(1024) uint8_t kv[BWQ_NS][4 * PF_QBOX];
  // dS, bf16 [128 rows][128 keys]: two K-major, 128-byte-swizzled boxes of 64
  // keys (the A operand of dQ += dS K); the epilogue's staging once every
  // product has completed
  alignas(1024) uint8_t ds[2 * PF_QBOX];
  alignas(8) uint64_t q_full, qt_full;
  uint64_t k_full[BWQ_NS], v_full[BWQ_NS], kv_empty[BWQ_NS];
  uint64_t s_full, s_free, p_full, ds_free;
  uint64_t fin;
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
};

// A_PART: TMEM column offset of the s-th 16-element K slice of a chunk-laid
// bf16 buffer (slices 0, 1 in chunk 0; 2, 3 in chunk 1).
__device__ __forceinline__ uint32_t bw_slice(int s) { return (uint32_t)((s >> 1) * 32 + (s & 1) * 8); }

// One half-step of the query-stationary kernel for this thread's row and this
// warp's 32-key chunk: dS = c P (dP - D) with P = 2^(S scale_log2 - lse), in
// f32x2 pairs (each operation rounds as its scalar form would).  With MASK,
// columns past lim (-1..31) are masked.
template <bool MASK>
__device__ __forceinline__ void bw_q_elementwise(const uint32_t (&sv)[32], const uint32_t (&pv)[32], uint32_t (&ds)[16],
                                                 int lim, float2 sl2, float2 nl2, float2 nd2, float2 c2) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sl2, nl2);
    if (MASK) {
      if (2 * i > lim) x.x = -INFINITY;
      if (2 * i + 1 > lim) x.y = -INFINITY;
    }
    const float2 p = make_float2(ex2(x.x), ex2(x.y));
    const float2 t = __fadd2_rn(make_float2(__uint_as_float(pv[2 * i]), __uint_as_float(pv[2 * i + 1])), nd2);
    const float2 d = __fmul2_rn(__fmul2_rn(c2, p), t);
    ds[i] = pack_bf16(d.x, d.y);
  }
}

// V1: the V1 layout ("差分注意力" tutorial, section V1 到 V2 的 diff): Q head
// qh of the Hq = 2H heads is map qh & 1 of V1 head qh / 2, read from its own
// 64-wide tensor (tmQ for map 1, tmQ2 for map 2; tmK, tmK2 likewise), and dQ
// of map 2 goes to dq2.  The scores then contract over 64 dimensions and dQ
// is an N = 64 product.
//
// Tiles are 128 keys, so the score products S = Q K^T and dP = dO V^T are
// N = 128 (a tcgen05.mma of N = 64 runs at about two-thirds of the tensor
// rate, one of N = 128 at the full rate).  Q and dO, the same for every tile,
// sit in TMEM as their A operands.  S and dP have one TMEM buffer: the
// elementwise warps release it (s_free) once they have loaded both of its
// 64-key halves, and write dS to shared memory, so the products of tile j + 1
// run while tile j's elementwise phase does.
template <bool V1>
__global__ void __maxnreg__(168)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ2,
              const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmK2, const __grid_constant__ CUtensorMap tmV, BwdArgs a) {
  constexpr int QB = V1 ? 1 : 2;   // 64-wide boxes per Q / K row (the QK width / 64)
  extern __shared__ uint8_t smem_raw[];
  BwQSmem& S = *reinterpret_cast<BwQSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &S.abort_flag;

  // unit: rows r0..r0+127 of Q head qh of batch b, heaviest row blocks first
  const int BQ = a.B * a.Hq;
  const int n_rb = (a.Lq + PF_BM - 1) / PF_BM;
  const int rb = n_rb - 1 - (int)(blockIdx.x / BQ);
  const int b = (int)(blockIdx.x % BQ) / a.Hq, qh = (int)(blockIdx.x % BQ) % a.Hq;
  const int Hp = a.Hq / 2, h = qh / 2, m = qh & 1, g = qh / (a.Hq / a.Hkv);
  const int r0 = rb * PF_BM;
  long long kend = a.causal ? (long long)min(r0 + PF_BM, a.Lq) - 1 + (a.Lk - a.Lq) + 1 : a.Lk;
  kend = max(0LL, min(kend, (long long)a.Lk));
  const int nT = (int)((kend + BWQ_BN - 1) / BWQ_BN);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&S.q_full), 1);
    mbar_init(smem_u32(&S.qt_full), BW_EW_WARPS);
    for (int i = 0; i < BWQ_NS; ++i) {
      mbar_init(smem_u32(&S.k_full[i]), 1);
      mbar_init(smem_u32(&S.v_full[i]), 1);
      mbar_init(smem_u32(&S.kv_empty[i]), 1);
    }
    mbar_init(smem_u32(&S.s_full), 1);
    mbar_init(smem_u32(&S.s_free), BW_EW_WARPS);
    mbar_init(smem_u32(&S.p_full), BW_EW_WARPS);
    mbar_init(smem_u32(&S.ds_free), 1);
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&S.drain[i]), 1);
    mbar_init(smem_u32(&S.fin), 1);
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
  // S [0,128), dP [128,256), dQ [256, 256 + 64 QB), Q [384, 384 + 32 QB), dO [448,512)
  constexpr uint32_t T_S = 0, T_P = 128, T_DQ = 256, T_Q = 384, T_O = 448;
  constexpr uint32_t HI = umma_desc_hi(1024);
  constexpr int QO = BWQ_NS - 1;   // the stage that first holds Q and dO

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0 && nT > 0) {
      const uint32_t qb = smem_u32(&S.q_full), qo = smem_u32(S.kv[QO]);
      const CUtensorMap* tq = (V1 && m) ? &tmQ2 : &tmQ;
      const CUtensorMap* tk = (V1 && m) ? &tmK2 : &tmK;
      mbar_expect_tx(qb, (QB + 2) * PF_QBOX);
      for (int x = 0; x < QB; ++x) tma_load_3d(qo + x * PF_QBOX, tq, qb, 64 * x, r0, V1 ? b * Hp + h : b * a.Hq + qh);
      for (int x = 0; x < 2; ++x) tma_load_3d(qo + (2 + x) * PF_QBOX, &tmO, qb, 64 * x, r0, b * Hp + h);
      int last_use[BWQ_NS];
      for (int i = 0; i < BWQ_NS; ++i) last_use[i] = -1;
      for (int j = 0; j < nT; ++j) {
        const int st = j % BWQ_NS, use = j / BWQ_NS;
        if (use > 0 && !wait_bar(smem_u32(&S.kv_empty[st]), (use - 1) & 1, abort_flag, a.watch)) break;
        // the first tile into the Q / dO stage waits for their copy into TMEM
        if (j == QO && !wait_bar(smem_u32(&S.qt_full), 0, abort_flag, a.watch)) break;
        const uint32_t kb = smem_u32(&S.k_full[st]), vb = smem_u32(&S.v_full[st]), base = smem_u32(S.kv[st]);
        mbar_expect_tx(kb, QB * PF_QBOX);
        for (int x = 0; x < QB; ++x) tma_load_3d(base + x * PF_QBOX, tk, kb, 64 * x, j * BWQ_BN, b * a.Hkv + g);
        mbar_expect_tx(vb, 2 * PF_QBOX);
        for (int x = 0; x < 2; ++x) tma_load_3d(base + (2 + x) * PF_QBOX, &tmV, vb, 64 * x, j * BWQ_BN, b * a.Hkv + g);
        last_use[st] = use;
      }
      drain_bar(qb, 0, a.watch.status);
      for (int i = 0; i < BWQ_NS; ++i) {
        if (last_use[i] >= 0) {
          drain_bar(smem_u32(&S.k_full[i]), last_use[i] & 1, a.watch.status);
          drain_bar(smem_u32(&S.v_full[i]), last_use[i] & 1, a.watch.status);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------- dQ issuer --
    if (lane == 0 && nT > 0) {
      constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, 64 * QB, true);
      const uint32_t ds_lo = umma_desc_lo(smem_u32(S.ds), 16);   // dS as the K-major A operand
      bool ok = true;
      for (int j = 0; ok && j < nT; ++j) {
        const int st = j % BWQ_NS;
        // this thread reads the K stage too: acquire it here
        if (!(ok = wait_bar(smem_u32(&S.k_full[st]), (j / BWQ_NS) & 1, abort_flag, a.watch))) break;
        if (!(ok = wait_bar(smem_u32(&S.p_full), j & 1, abort_flag, a.watch))) break;
        tc_fence_after();
        // K as the N-major B operand: keys down the rows, 64-wide dimension boxes PF_QBOX apart
        const uint32_t klo = umma_desc_lo(smem_u32(S.kv[st]), PF_QBOX);
#pragma unroll
        for (int s = 0; s < BWQ_BN / 16; ++s) {   // dQ += dS K over the tile's 128 keys
          const uint32_t ao = (uint32_t)((s >> 2) * (PF_QBOX >> 4) + (s & 3) * 2);
          mma_ss_w(tmem + T_DQ, ds_lo + ao, HI, klo + (uint32_t)(s * (2048 >> 4)), HI, IDESC_ACC, (j > 0 || s > 0));
        }
        mma_commit(smem_u32(&S.ds_free));
        mma_commit(smem_u32(&S.kv_empty[st]));
      }
      if (ok) mma_commit(smem_u32(&S.fin));
      mma_commit(smem_u32(&S.drain[0]));
      drain_bar(smem_u32(&S.drain[0]), 0, a.watch.status);
    }
  } else if (warp == 10) {
    // --------------------------------------------- S and dP issuer --
    if (lane == 0 && nT > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BWQ_BN, false);
      bool ok = wait_bar(smem_u32(&S.qt_full), 0, abort_flag, a.watch);
      for (int j = 0; ok && j < nT; ++j) {
        const int st = j % BWQ_NS;
        if (!(ok = wait_bar(smem_u32(&S.k_full[st]), (j / BWQ_NS) & 1, abort_flag, a.watch))) break;
        if (!(ok = wait_bar(smem_u32(&S.v_full[st]), (j / BWQ_NS) & 1, abort_flag, a.watch))) break;
        // the one S / dP buffer: the elementwise warps have loaded tile j - 1's
        if (j >= 1 && !(ok = wait_bar(smem_u32(&S.s_free), (j - 1) & 1, abort_flag, a.watch))) break;
        tc_fence_after();
        const uint32_t base = smem_u32(S.kv[st]);
        const uint32_t klo = umma_desc_lo(base, 16), vlo = umma_desc_lo(base + 2 * PF_QBOX, 16);
#pragma unroll
        for (int s = 0; s < 4 * QB; ++s) {   // S = Q K^T over the QK width, Q from TMEM
          const uint32_t bo = (uint32_t)((s >> 2) * (PF_QBOX >> 4) + (s & 3) * 2);
          mma_ts_w(tmem + T_S, tmem + T_Q + (uint32_t)(s * 8), klo + bo, HI, IDESC_S, s > 0);
        }
#pragma unroll
        for (int s = 0; s < 8; ++s) {        // dP = dO V^T over the value width, dO from TMEM
          const uint32_t bo = (uint32_t)((s >> 2) * (PF_QBOX >> 4) + (s & 3) * 2);
          mma_ts_w(tmem + T_P, tmem + T_O + (uint32_t)(s * 8), vlo + bo, HI, IDESC_S, s > 0);
        }
        mma_commit(smem_u32(&S.s_full));
      }
      mma_commit(smem_u32(&S.drain[1]));
      drain_bar(smem_u32(&S.drain[1]), 0, a.watch.status);
    }
  } else if (warp < 8) {
    // ------------------------------------------- elementwise (thread = row) --
    const int wq = warp & 3, ch = warp >> 2, r = threadIdx.x & 127;
    const int rg = r0 + r;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t ds_base = smem_u32(S.ds);
    const size_t stat = (((size_t)b * Hp + h) * 2 + m) * a.Lp + rg;
    const float c = a.scale * (m == 0 ? 1.f : -a.lambda[h]);
    const float2 nl2 = make_float2(a.nlse[stat], a.nlse[stat]), nd2 = make_float2(a.ndd[stat], a.ndd[stat]);
    const float2 sl2 = make_float2(a.scale_log2, a.scale_log2), c2 = make_float2(c, c);
    const long long lastk = a.causal ? min((long long)a.Lk - 1, (long long)rg + (a.Lk - a.Lq)) : (long long)a.Lk - 1;
    bool ok = true;
    if (nT > 0) {
      // This row of Q (chunk 0's warps) or of dO (chunk 1's) into TMEM: each
      // 64-element box row from its 128-byte-swizzled tile, two bf16 a column.
      if ((ok = warp_wait<true>(smem_u32(&S.q_full), 0, abort_flag, a.watch))) {
        const uint8_t* tile = S.kv[QO] + (ch == 0 ? 0 : 2 * PF_QBOX);
        const int nbox = ch == 0 ? QB : 2;
        const uint32_t tdst = tmem + lane_off + (ch == 0 ? T_Q : T_O);
        for (int x = 0; x < nbox; ++x) {
          uint32_t wv[32];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + x * PF_QBOX + r * 128 + ((cc ^ (r & 7)) << 4));
            wv[4 * cc] = v.x; wv[4 * cc + 1] = v.y; wv[4 * cc + 2] = v.z; wv[4 * cc + 3] = v.w;
          }
          tmem_st32p(tdst + (uint32_t)(x * 32), wv);
        }
        tmem_wait_st();
        tc_fence_before();
        fence_proxy_async_smem();   // these reads come before the TMA writes of K/V tiles there
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S.qt_full));
      }
    }
    for (int j = 0; ok && j < nT; ++j) {
      if (!(ok = warp_wait<true>(smem_u32(&S.s_full), j & 1, abort_flag, a.watch))) break;
      tc_fence_after();
      // both halves into registers at once, then the buffer is released:
      // tile j + 1's products overlap all of this tile's arithmetic
      uint32_t sv[2][32], pv[2][32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld32p(tmem + lane_off + T_S + hh * 64 + ch * 32, sv[hh]);
        tmem_ld32p(tmem + lane_off + T_P + hh * 64 + ch * 32, pv[hh]);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.s_free));
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {   // the tile's two 64-key halves
        uint32_t ds[16];
        const long long lim = lastk - (long long)j * BWQ_BN - hh * 64 - ch * 32;   // columns > lim are masked
        // warp-uniform: the warp runs one straight-line variant per half
        if (__all_sync(0xffffffffu, lim >= 31))
          bw_q_elementwise<false>(sv[hh], pv[hh], ds, 0, sl2, nl2, nd2, c2);
        else
          bw_q_elementwise<true>(sv[hh], pv[hh], ds, (int)max(-1LL, min(lim, 31LL)), sl2, nl2, nd2, c2);
        // the dS buffer is free once dQ of tile j - 1 has completed
        if (hh == 0 && j >= 1 && !(ok = warp_wait<true>(smem_u32(&S.ds_free), (j - 1) & 1, abort_flag, a.watch))) break;
        // row r of box hh, keys 32 ch + 8 q .. + 7 of the box: logical chunk 4 ch + q
        const uint32_t row_at = ds_base + (uint32_t)hh * PF_QBOX + (uint32_t)r * 128, sw = (uint32_t)(r & 7);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          sts_u4(row_at + ((((uint32_t)(4 * ch + q)) ^ sw) << 4), ds[4 * q], ds[4 * q + 1], ds[4 * q + 2],
                 ds[4 * q + 3]);
      }
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.p_full));
    }
    // ---- epilogue: dQ rows ----
    bool have = nT == 0;
    float y[64];
    if (nT > 0 && ok) have = warp_wait<true>(smem_u32(&S.fin), 0, abort_flag, a.watch);
    if (have && ch < QB) {   // chunk ch writes dQ columns [64 ch, 64 ch + 64) of its rows
      if (nT > 0) tc_fence_after();
      __nv_bfloat16* base = V1 ? (m ? a.dq2 : a.dq) + ((size_t)b * Hp + h) * a.Lq * 64
                               : a.dq + ((size_t)b * a.Hq + qh) * a.Lq * 128;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t o[32];
        if (nT > 0) {
          tmem_ld32p(tmem + lane_off + T_DQ + ch * 64 + cc * 32, o);
          tmem_wait_ld();
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) y[cc * 32 + i] = nT > 0 ? __uint_as_float(o[i]) : 0.f;
      }
      // staging: the dS buffer, free once every product has completed (or never used)
      pf_store_rows(S.ds + warp * 16 * 128, y, base + ch * 64, r0 + wq * 32, a.Lq, lane, 64 * QB);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// --------------------------------------------------------- dK/dV (KV-stationary) --
struct BwKSmem {
  alignas(1024) uint8_t k[2 * PF_QBOX];             // K tile: 128 keys, dims 0-63 box, 64-127 box
  alignas(1024) uint8_t v[2 * PF_QBOX];             // V tile, same layout
  alignas(1024) uint8_t q[BW_NS][2 * PF_KBOX];      // Q rows: 64, two boxes
  alignas(1024) uint8_t o[BW_NS][2 * PF_KBOX];      // dO rows
  alignas(16) float nlse[BW_NS][BW_RB];
  alignas(16) float ndd[BW_NS][BW_RB];
  alignas(16) uint8_t stage[8][16 * 128];
  alignas(8) uint64_t kv_full;
  uint64_t st_full[BW_NS], st_empty[BW_NS];
  uint64_t s_full[2], p_full[2], sv_free[2], sd_free[2];
  uint64_t fin;
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// 16-byte load from shared memory (addr: a shared-window address).
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// The stage's 16 negated log-sum-exp and D values of half h of a 32-row chunk
// (one per row, the same for every key), as f32 pairs.
__device__ __forceinline__ void bw_kv_stats(uint32_t nl_s, uint32_t nd_s, int h, float2 (&nl)[8], float2 (&nd)[8]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 l4 = lds_f4(nl_s + (uint32_t)((h * 16 + q * 4) * 4));
    const float4 d4 = lds_f4(nd_s + (uint32_t)((h * 16 + q * 4) * 4));
    nl[2 * q] = make_float2(l4.x, l4.y); nl[2 * q + 1] = make_float2(l4.z, l4.w);
    nd[2 * q] = make_float2(d4.x, d4.y); nd[2 * q + 1] = make_float2(d4.z, d4.w);
  }
}

// The two steps of a diff pair in the key-stationary kernel, for this
// thread's key and this warp's 32-row chunk.  The pair's maps share dO, so
// dP^T = V dO^T is computed once, in the map-1 step, and the map-2 step takes
// it from registers; P_1 waits there too, so that dV's operand is the
// difference (P_1 - lambda P_2)^T formed in f32 and rounded once.  The
// arithmetic runs on f32x2 pairs (each operation rounds as its scalar form
// would).  vis0: the first visible row of the chunk (0..32); with MASK, rows
// before it give P = 0.  With RESID, dS^T's bf16 residual goes 16 columns
// after its hi part.
//
// Map 1: from S_1^T (tS) and dP^T (tP) write dS_1^T = c P_1 (dP - D_1) back
// over S_1^T, and keep P_1 and dP.
template <bool RESID, bool MASK>
__device__ __forceinline__ void bw_kv_map1(uint32_t tS, uint32_t tP, int vis0, float2 cd2, float2 sl2, uint32_t nl_s,
                                           uint32_t nd_s, float2 (&p1)[16], float2 (&dp)[16]) {
  uint32_t sv[32], pv[32], ds[16];
  tmem_ld32p(tS, sv);
  tmem_ld32p(tP, pv);
  tmem_wait_ld();
  uint32_t rds[RESID ? 16 : 1];
  const float2 neg1 = make_float2(-1.f, -1.f);
  float2 nl[8], nd[8];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if ((j & 7) == 0) bw_kv_stats(nl_s, nd_s, j >> 3, nl, nd);
    float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), sl2, nl[j & 7]);
    if (MASK) {
      if (2 * j < vis0) x.x = -INFINITY;
      if (2 * j + 1 < vis0) x.y = -INFINITY;
    }
    const float2 p = make_float2(ex2(x.x), ex2(x.y));
    p1[j] = p;
    dp[j] = make_float2(__uint_as_float(pv[2 * j]), __uint_as_float(pv[2 * j + 1]));
    const float2 d2 = __fmul2_rn(__fmul2_rn(cd2, p), __fadd2_rn(dp[j], nd[j & 7]));
    ds[j] = pack_bf16(d2.x, d2.y);
    if constexpr (RESID) {   // x - bf16(x), exact in f32
      const float2 dh = make_float2(__uint_as_float(ds[j] << 16), __uint_as_float(ds[j] & 0xFFFF0000u));
      const float2 rd = __ffma2_rn(dh, neg1, d2);
      rds[j] = pack_bf16(rd.x, rd.y);
    }
  }
  tmem_st16p(tS, ds);
  if constexpr (RESID) tmem_st16p(tS + 16, rds);
}

// Map 2: from S_2^T (tS) and the map-1 step's P_1 and dP, write
// (P_1 - lambda P_2)^T over S_2^T and dS_2^T = c P_2 (dP - D_2) at tD.
template <bool RESID, bool MASK>
__device__ __forceinline__ void bw_kv_map2(uint32_t tS, uint32_t tD, int vis0, float2 nlam2, float2 cd2, float2 sl2,
                                           uint32_t nl_s, uint32_t nd_s, const float2 (&p1)[16],
                                           const float2 (&dp)[16]) {
  uint32_t sv[32], cw[16], ds[16];
  tmem_ld32p(tS, sv);
  tmem_wait_ld();
  uint32_t rds[RESID ? 16 : 1];
  const float2 neg1 = make_float2(-1.f, -1.f);
  float2 nl[8], nd[8];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if ((j & 7) == 0) bw_kv_stats(nl_s, nd_s, j >> 3, nl, nd);
    float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), sl2, nl[j & 7]);
    if (MASK) {
      if (2 * j < vis0) x.x = -INFINITY;
      if (2 * j + 1 < vis0) x.y = -INFINITY;
    }
    const float2 p = make_float2(ex2(x.x), ex2(x.y));
    const float2 c = __ffma2_rn(nlam2, p, p1[j]);
    cw[j] = pack_bf16(c.x, c.y);
    const float2 d2 = __fmul2_rn(__fmul2_rn(cd2, p), __fadd2_rn(dp[j], nd[j & 7]));
    ds[j] = pack_bf16(d2.x, d2.y);
    if constexpr (RESID) {
      const float2 dh = make_float2(__uint_as_float(ds[j] << 16), __uint_as_float(ds[j] & 0xFFFF0000u));
      const float2 rd = __ffma2_rn(dh, neg1, d2);
      rds[j] = pack_bf16(rd.x, rd.y);
    }
  }
  tmem_st16p(tS, cw);
  tmem_st16p(tD, ds);
  if constexpr (RESID) tmem_st16p(tD + 16, rds);
}

// V1: as for bwd_dq_kernel.  The CTA holds K1 and K2 side by side in its
// 128-wide K tile; a step with map m scores against K_m's half and
// accumulates dK_m into its own 64 columns of the dK accumulator (dK1 in the
// first, dK2 in the second), which the epilogue writes to dk and dk2.
template <bool V1>
__global__ void __maxnreg__(168)
bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK2,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ,
               const __grid_constant__ CUtensorMap tmQ2, const __grid_constant__ CUtensorMap tmO, BwdArgs a) {
  constexpr int QB = V1 ? 1 : 2;   // 64-wide boxes per Q row (the QK width / 64)
  extern __shared__ uint8_t smem_raw[];
  BwKSmem& S = *reinterpret_cast<BwKSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &S.abort_flag;

  // unit: keys k0..k0+127 of KV head g of batch b; low key tiles (most rows) first
  const int BG = a.B * a.Hkv;
  const int kt = (int)(blockIdx.x / BG);
  const int b = (int)(blockIdx.x % BG) / a.Hkv, g = (int)(blockIdx.x % BG) % a.Hkv;
  const int k0 = kt * PF_BM;
  const int grp = a.Hq / a.Hkv, Hp = a.Hq / 2;
  const int off = a.Lk - a.Lq;
  // first 64-row block holding a row that sees key k0 (causal: row >= k0 - off)
  const int rb0 = (a.causal && k0 - off > 0) ? (k0 - off) / BW_RB : 0;
  const int n_rb = (a.Lq + BW_RB - 1) / BW_RB;
  const int per_head = max(0, n_rb - rb0);
  const int nS = grp * per_head;
  // Steps: (row block, head of the group), heads innermost.  The CTAs of one
  // group start at different row blocks (the first row that sees their keys)
  // and then advance one row block per grp steps, so they stay a fixed
  // distance apart and each Q / dO tile is read from DRAM about once and
  // from L2 by the others; with the heads outermost they drift onto different
  // heads and each re-reads its tiles.
  auto step_head = [&](int i) { return g * grp + i % grp; };
  auto step_rb = [&](int i) { return rb0 + i / grp; };

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&S.kv_full), 1);
    for (int i = 0; i < BW_NS; ++i) {
      mbar_init(smem_u32(&S.st_full[i]), 1);
      mbar_init(smem_u32(&S.st_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&S.s_full[i]), 1);
      mbar_init(smem_u32(&S.p_full[i]), BW_EW_WARPS);
      mbar_init(smem_u32(&S.sv_free[i]), 1);
      mbar_init(smem_u32(&S.sd_free[i]), 1);
      mbar_init(smem_u32(&S.drain[i]), 1);
    }
    mbar_init(smem_u32(&S.fin), 1);
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
  // TMEM: S_1^T [0,64), S_2^T [64,128), dP^T [128,192), dS_2^T [192,256), dV [256,384), dK [384,512)
  const uint32_t tmem = S.tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0 && nS > 0) {
      const uint32_t kvb = smem_u32(&S.kv_full);
      mbar_expect_tx(kvb, 4 * PF_QBOX);
      for (int x = 0; x < 2; ++x) {   // V1: box x is K_{x+1}
        tma_load_3d(smem_u32(S.k) + x * PF_QBOX, (V1 && x) ? &tmK2 : &tmK, kvb, V1 ? 0 : 64 * x, k0, b * a.Hkv + g);
        tma_load_3d(smem_u32(S.v) + x * PF_QBOX, &tmV, kvb, 64 * x, k0, b * a.Hkv + g);
      }
      int last_use[BW_NS];
      for (int i = 0; i < BW_NS; ++i) last_use[i] = -1;
      for (int i = 0; i < nS; ++i) {
        const int st = i % BW_NS, use = i / BW_NS;
        if (use > 0 && !wait_bar(smem_u32(&S.st_empty[st]), (use - 1) & 1, abort_flag, a.watch)) break;
        const int qh = step_head(i), rb = step_rb(i);
        const int hq = qh / 2, mq = qh & 1;
        const uint32_t fb = smem_u32(&S.st_full[st]);
        mbar_expect_tx(fb, (QB + 2) * PF_KBOX + 2 * BW_RB * 4);
        for (int x = 0; x < QB; ++x)
          tma_load_3d(smem_u32(S.q[st]) + x * PF_KBOX, (V1 && mq) ? &tmQ2 : &tmQ, fb, 64 * x, rb * BW_RB,
                      V1 ? b * Hp + hq : b * a.Hq + qh);
        for (int x = 0; x < 2; ++x)
          tma_load_3d(smem_u32(S.o[st]) + x * PF_KBOX, &tmO, fb, 64 * x, rb * BW_RB, b * Hp + hq);
        const size_t stat = (((size_t)b * Hp + hq) * 2 + mq) * a.Lp + (size_t)rb * BW_RB;
        bulk_load(smem_u32(S.nlse[st]), a.nlse + stat, BW_RB * 4, fb);
        bulk_load(smem_u32(S.ndd[st]), a.ndd + stat, BW_RB * 4, fb);
        last_use[st] = use;
      }
      drain_bar(kvb, 0, a.watch.status);
      for (int i = 0; i < BW_NS; ++i)
        if (last_use[i] >= 0) drain_bar(smem_u32(&S.st_full[i]), last_use[i] & 1, a.watch.status);
    }
  } else if (warp >= 9) {
    // --------------------------------------------------------- MMA issuers --
    if (lane == 0 && nS > 0) {
      constexpr uint32_t HI = umma_desc_hi(1024);
      constexpr uint32_t QSTAGE = (2 * PF_KBOX) >> 4;
      const int issuer = warp - 9;   // 0: dV, dK accumulation; 1: S^T and dP^T
      bool ok = true;
      if (issuer == 0) {
        constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, 128, true);
        constexpr uint32_t IDESC_DK = idesc_bf16_f32(128, 64 * QB, true);
        const uint32_t o_mn0 = umma_desc_lo(smem_u32(S.o[0]), PF_KBOX), q_mn0 = umma_desc_lo(smem_u32(S.q[0]), PF_KBOX);
        for (int i = 0; ok && i < nS; ++i) {
          const int bb = i & 1, st = i % BW_NS;
          const int qh = step_head(i);
          // dK's residual: V2 sums dK over the pair's maps, which cancel when
          // they are alike; V1 keeps dK_1 and dK_2 apart.  lambda is read
          // before the waits, so its load is not on the issue path.
          const bool resid = !V1 && fabsf(1.f - a.lambda[qh / 2]) < a.resid_tau;
          // this thread reads the stage's Q and dO too: acquire them here
          if (!(ok = wait_bar(smem_u32(&S.st_full[st]), (i / BW_NS) & 1, abort_flag, a.watch))) break;
          if (!(ok = wait_bar(smem_u32(&S.p_full[bb]), (i >> 1) & 1, abort_flag, a.watch))) break;
          tc_fence_after();
          const uint32_t olo = o_mn0 + (uint32_t)st * QSTAGE, qlo = q_mn0 + (uint32_t)st * QSTAGE;
          // V1: map m's dK lives in its own 64 columns and first receives a
          // value at step m (steps 0 and 1 are the two maps of the group's
          // first head); V2: one dK for both maps
          const uint32_t dk_t = tmem + 384 + (V1 ? (uint32_t)(bb * 64) : 0u);
          const bool dk_acc = V1 ? i > 1 : i > 0;
          // map 1: dS_1^T over S_1^T at [0, 64); map 2: (P_1 - lambda P_2)^T
          // over S_2^T at [64, 128) and dS_2^T at [192, 256)
          const uint32_t ds_t = tmem + (bb ? 192u : 0u);
          if (bb) {
            // dV += (P_1 - lambda P_2)^T dO; then S_2^T of the next pair may
            // overwrite [64, 128)
#pragma unroll
            for (int s = 0; s < BW_RB / 16; ++s)
              mma_ts_w(tmem + 256, tmem + 64 + bw_slice(s), olo + (uint32_t)(s * (2048 >> 4)), HI, IDESC_ACC,
                       (i > 1 || s > 0));
            mma_commit(smem_u32(&S.sv_free[1]));
          }
          // dK += dS_m^T Q_m and its residual
#pragma unroll
          for (int s = 0; s < BW_RB / 16; ++s)
            mma_ts_w(dk_t, ds_t + bw_slice(s), qlo + (uint32_t)(s * (2048 >> 4)), HI, IDESC_DK, (dk_acc || s > 0));
          if (resid) {
#pragma unroll
            for (int s = 0; s < BW_RB / 16; ++s)
              mma_ts_w(dk_t, ds_t + bw_slice(s) + 16, qlo + (uint32_t)(s * (2048 >> 4)), HI, IDESC_DK, 1);
          }
          // map 1: the next pair's S_1^T and dP^T may overwrite [0, 64) and
          // [128, 192); map 2: its dS_2^T may overwrite [192, 256)
          mma_commit(smem_u32(bb ? &S.sd_free[1] : &S.sv_free[0]));
          mma_commit(smem_u32(&S.st_empty[st]));
        }
        if (ok) mma_commit(smem_u32(&S.fin));
      } else {
        constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BW_RB, false);
        const uint32_t k_lo = umma_desc_lo(smem_u32(S.k), 16), v_lo = umma_desc_lo(smem_u32(S.v), 16);
        const uint32_t q_lo0 = umma_desc_lo(smem_u32(S.q[0]), 16), o_lo0 = umma_desc_lo(smem_u32(S.o[0]), 16);
        ok = wait_bar(smem_u32(&S.kv_full), 0, abort_flag, a.watch);
        for (int i = 0; ok && i < nS; ++i) {
          const int bb = i & 1, st = i % BW_NS;
          if (!(ok = wait_bar(smem_u32(&S.st_full[st]), (i / BW_NS) & 1, abort_flag, a.watch))) break;
          // S_m^T(i) overwrites what the accumulating products of step i - 2
          // read (dK_1 for map 1, dV for map 2)
          if (i >= 2 && !(ok = wait_bar(smem_u32(&S.sv_free[bb]), ((i - 2) >> 1) & 1, abort_flag, a.watch)))
            break;
          tc_fence_after();
          const uint32_t qlo = q_lo0 + (uint32_t)st * QSTAGE, olo = o_lo0 + (uint32_t)st * QSTAGE;
          // V1: the step's map m scores against K_m, box m of the K tile
          const uint32_t kmo = V1 ? (uint32_t)(bb * (PF_QBOX >> 4)) : 0u;
#pragma unroll
          for (int s = 0; s < 4 * QB; ++s) {   // S^T = K Q^T over the QK width
            const uint32_t ao = (uint32_t)((s >> 2) * (PF_QBOX >> 4) + (s & 3) * 2);
            const uint32_t bo = (uint32_t)((s >> 2) * (PF_KBOX >> 4) + (s & 3) * 2);
            mma_ss_w(tmem + bb * 64, k_lo + kmo + ao, HI, qlo + bo, HI, IDESC_S, s > 0);
          }
          if (bb == 0) {
            // dP^T = V dO^T, once per pair, into [128, 192): the elementwise
            // warps loaded it at step i - 2, before dK_1(i - 2) (sv_free[0])
#pragma unroll
            for (int s = 0; s < 8; ++s) {
              const uint32_t ao = (uint32_t)((s >> 2) * (PF_QBOX >> 4) + (s & 3) * 2);
              const uint32_t bo = (uint32_t)((s >> 2) * (PF_KBOX >> 4) + (s & 3) * 2);
              mma_ss_w(tmem + 128, v_lo + ao, HI, olo + bo, HI, IDESC_S, s > 0);
            }
          } else if (i >= 3 && !(ok = wait_bar(smem_u32(&S.sd_free[1]), ((i - 2) >> 1) & 1, abort_flag, a.watch))) {
            // map 2's elementwise step writes dS_2^T over [192, 256), which
            // dK_2(i - 2) read: the commit below follows this wait
            break;
          }
          mma_commit(smem_u32(&S.s_full[bb]));
        }
      }
      mma_commit(smem_u32(&S.drain[issuer]));
      drain_bar(smem_u32(&S.drain[issuer]), 0, a.watch.status);
    }
  } else {
    // ------------------------------------------- elementwise (thread = key) --
    const int wq = warp & 3, ch = warp >> 2, kr = threadIdx.x & 127;
    const int kg = k0 + kr;   // this thread's key
    const float2 sl2 = make_float2(a.scale_log2, a.scale_log2);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    bool ok = true;
    float2 p1[16], dp[16];   // P_1 and dP of this thread's key and chunk, from the map-1 step to the map-2 step
    for (int i = 0; i < nS; ++i) {
      // the group's heads are innermost and come in pairs, so step i is map
      // i & 1 of a pair, and steps 2k, 2k + 1 share their rows
      const int bb = i & 1, st = i % BW_NS;
      const int qh = step_head(i), rb = step_rb(i);
      // lambda read once, before the waits, so its load is not on the step's path
      const float lam = a.lambda[qh / 2];
      const bool resid = !V1 && fabsf(1.f - lam) < a.resid_tau;
      // The stage's log-sum-exp and D values came by bulk copy: wait for them here too.
      if (!(ok = warp_wait(smem_u32(&S.st_full[st]), (i / BW_NS) & 1, abort_flag, a.watch))) break;
      if (!(ok = warp_wait(smem_u32(&S.s_full[bb]), (i >> 1) & 1, abort_flag, a.watch))) break;
      tc_fence_after();
      // rows r = rb*64 + col see this key iff kg < Lk and (not causal or kg <= r + off)
      const int row0 = rb * BW_RB + ch * 32;
      const int vis0 = kg >= a.Lk ? 32 : (a.causal ? min(32, max(0, kg - off - row0)) : 0);
      // branch once per step, warp-uniformly (the TMEM stores inside are
      // warp-collective): each variant's loop is one straight-line block
      const bool full = __all_sync(0xffffffffu, vis0 == 0);
      const uint32_t nl_s = smem_u32(S.nlse[st] + ch * 32), nd_s = smem_u32(S.ndd[st] + ch * 32);
      const uint32_t t0 = tmem + lane_off + ch * 32;
      if (bb == 0) {
        const float2 cd2 = make_float2(a.scale, a.scale);
        if (resid) {
          if (full) bw_kv_map1<true, false>(t0, t0 + 128, 0, cd2, sl2, nl_s, nd_s, p1, dp);
          else bw_kv_map1<true, true>(t0, t0 + 128, vis0, cd2, sl2, nl_s, nd_s, p1, dp);
        } else {
          if (full) bw_kv_map1<false, false>(t0, t0 + 128, 0, cd2, sl2, nl_s, nd_s, p1, dp);
          else bw_kv_map1<false, true>(t0, t0 + 128, vis0, cd2, sl2, nl_s, nd_s, p1, dp);
        }
      } else {
        const float2 nlam2 = make_float2(-lam, -lam), cd2 = make_float2(-a.scale * lam, -a.scale * lam);
        if (resid) {
          if (full) bw_kv_map2<true, false>(t0 + 64, t0 + 192, 0, nlam2, cd2, sl2, nl_s, nd_s, p1, dp);
          else bw_kv_map2<true, true>(t0 + 64, t0 + 192, vis0, nlam2, cd2, sl2, nl_s, nd_s, p1, dp);
        } else {
          if (full) bw_kv_map2<false, false>(t0 + 64, t0 + 192, 0, nlam2, cd2, sl2, nl_s, nd_s, p1, dp);
          else bw_kv_map2<false, true>(t0 + 64, t0 + 192, vis0, nlam2, cd2, sl2, nl_s, nd_s, p1, dp);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.p_full[bb]));
    }
    // ---- epilogue: dV and dK rows of this tile's keys ----
    bool have = nS == 0;
    float y[64];
    if (nS > 0 && ok) have = warp_wait(smem_u32(&S.fin), 0, abort_flag, a.watch);
    if (have) {   // chunk 0 writes dV, chunk 1 dK (V1: dK1 then dK2, 64 columns each)
      if (nS > 0) tc_fence_after();
      const size_t kv_row0 = ((size_t)b * a.Hkv + g) * a.Lk;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        __nv_bfloat16* base = !ch ? a.dv + kv_row0 * 128 + hf * 64
                                  : (V1 ? (hf ? a.dk2 : a.dk) + kv_row0 * 64 : a.dk + kv_row0 * 128 + hf * 64);
        const int stride = (V1 && ch) ? 64 : 128;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t o[32];
          if (nS > 0) {
            tmem_ld32p(tmem + lane_off + 256 + ch * 128 + hf * 64 + cc * 32, o);
            tmem_wait_ld();
          }
#pragma unroll
          for (int t = 0; t < 32; ++t) y[cc * 32 + t] = nS > 0 ? __uint_as_float(o[t]) : 0.f;
        }
        pf_store_rows(S.stage[warp], y, base, k0 + wq * 32, a.Lk, lane, stride);
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
