// lowrank.cuh -- the fixed low-rank substitute for the second map: N V by prefix sums.
//
// The paper note "Understanding Differential Transformer Unchains Pretrained
// Self-Attentions" (sections 基于分析的改进建议 and 亮点与洞察) finds the noise
// component that A2 removes to be low-rank, and proposes a fixed low-rank
// matrix in place of the second attention.  It gives no form; the reading
// implemented here makes N a map like A2 (non-negative, zero on masked keys,
// rows summing to 1) built from fixed non-negative positional factors
// F [Lq, r] and G [Lk, r]:
//
//     N[i, j] = f_i . g_j / sum_{j' visible from i} f_i . g_j'
//     (N V)_i = f_i^T S_i / f_i^T z_i,  S_i = sum_{visible j} g_j v_j^T (r x dv),
//                                       z_i = sum_{visible j} g_j
//     out_i   = (A1 V)_i - lambda (N V)_i          (0 for N's row when f_i^T z_i = 0)
//
// Under the causal mask the keys row i sees are a prefix, j <= i + (Lk - Lq),
// so S_i and z_i are prefix sums over keys.  The keys are cut into slots: first
// n_lead slots of LR_C keys covering the leading keys [0, P_0) that every row
// sees, then one slot per chunk of LR_C query rows, row chunk c holding the
// keys [P_c, P_{c+1}) with P_c = clamp(c LR_C + Lk - Lq, 0, Lk), one per row.
// Three HBM-bound passes:
//
//   lr_totals_kernel  per slot, the sums of g_j v_j^T and g_j over its keys
//                     (unmasked: plain key chunks [c LR_C, (c+1) LR_C))
//   lr_prefix_kernel  exclusive prefix of those sums over the slots, plus the
//                     grand total in slot nc (used by every row when unmasked)
//   lr_emit_kernel    row chunk c starts from the prefix at its slot, i.e. the
//                     keys [0, P_c); each row adds its key i + Lk - Lq and
//                     writes out_i
//
// A1 V comes from the prefill's single-map mode: pairing heads (2j, 2j+1) of
// one KV group as a CTA's two maps gives every head's single-map attention
// without extra products.  It is written in f32, O_m / l_m straight from the
// accumulator, and P keeps its bf16 residual for heads with |1 - lambda| below
// the forward's threshold: when N is close to A1 and lambda close to 1 the
// output is a small difference of two near-equal terms, and a bf16 A1 V (or a
// bf16-only P) would leave an error of A1 V's own rounding scale in it.  The
// subtraction here is then the only rounding to bf16.
//
// One thread owns one of the 128 value columns and r <= LR_RMAX accumulators;
// there is no shared memory and no wait.  Each kernel body is a host-device
// function of (chunk, head, column), so the same code can be run over every
// index on the host.
#pragma once

#include <cuda_bf16.h>
#include <cstddef>

namespace da {

constexpr int LR_C = 256;     // query rows (keys) per chunk
constexpr int LR_DV = 128;    // value width; one thread per column
constexpr int LR_RMAX = 16;   // largest rank

struct LowrankArgs {
  const __nv_bfloat16* v;     // [B, Hkv, Lk, 128]
  const float* F;             // [H, Lq, r], >= 0
  const float* G;             // [H, Lk, r], >= 0
  const float* lambda;        // [H]
  const float* a1v;           // [B, H, Lq, 128]: A1 V per head, f32
  __nv_bfloat16* out;         // [B, H, Lq, 128]
  float* tot;                 // [B*H, nc + 1, r, 128] chunk sums of g v^T, then their prefix; slot nc = total
  float* ztot;                // [B*H, nc + 1, r] the same for g
  int B, H, Hkv, Lq, Lk, r, causal;
  int n_lead;                 // causal: slots of leading keys, ceil(clamp(Lk - Lq, 0, Lk) / LR_C); else 0
  int nc;                     // slots: n_lead + ceil(Lq / LR_C) causal, ceil(Lk / LR_C) unmasked
};

// Slot counts for the sizes in a (host and device use the same rule).
__host__ __device__ inline void lr_slots(int Lq, int Lk, int causal, int& n_lead, int& nc) {
  if (causal) {
    const long long off = (long long)Lk - Lq;
    const long long lead = off < 0 ? 0 : (off > Lk ? Lk : off);
    n_lead = (int)((lead + LR_C - 1) / LR_C);
    nc = n_lead + (int)(((long long)Lq + LR_C - 1) / LR_C);
  } else {
    n_lead = 0;
    nc = (int)(((long long)Lk + LR_C - 1) / LR_C);
  }
}

__host__ __device__ inline long long lr_clamp(long long x, long long hi) { return x < 0 ? 0 : (x > hi ? hi : x); }

// Keys whose sums slot c contributes (see the header).
__host__ __device__ inline void lr_key_range(const LowrankArgs& a, int c, long long& ks, long long& ke) {
  if (a.causal) {
    const long long off = (long long)a.Lk - a.Lq, lead = lr_clamp(off, a.Lk);
    if (c < a.n_lead) {            // leading keys, seen by every row
      ks = (long long)c * LR_C;
      ke = ks + LR_C < lead ? ks + LR_C : lead;
    } else {                       // the keys the rows of chunk c - n_lead add
      const long long rc = c - a.n_lead;
      ks = rc == 0 ? lead : lr_clamp(rc * LR_C + off, a.Lk);
      ke = lr_clamp((rc + 1) * LR_C + off, a.Lk);
    }
  } else {
    ks = (long long)c * LR_C;
    ke = lr_clamp((long long)(c + 1) * LR_C, a.Lk);
  }
}

__host__ __device__ inline void lr_add_key(const LowrankArgs& a, const __nv_bfloat16* vcol, const float* gh, long long j,
                                           float (&S)[LR_RMAX], float (&z)[LR_RMAX]) {
  const float vj = __bfloat162float(vcol[j * LR_DV]);
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t)
    if (t < a.r) {
      const float gj = gh[j * a.r + t];
      S[t] = fmaf(gj, vj, S[t]);
      z[t] += gj;
    }
}

__host__ __device__ inline void lr_totals_body(const LowrankArgs& a, int c, int bh, int col) {
  const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.Hkv);
  long long ks, ke;
  lr_key_range(a, c, ks, ke);
  float S[LR_RMAX], z[LR_RMAX];
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t) S[t] = z[t] = 0.f;
  const __nv_bfloat16* vcol = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * LR_DV + col;
  const float* gh = a.G + (size_t)h * a.Lk * a.r;
  for (long long j = ks; j < ke; ++j) lr_add_key(a, vcol, gh, j, S, z);
  const size_t slot = (size_t)bh * (a.nc + 1) + c;
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t)
    if (t < a.r) {
      a.tot[(slot * a.r + t) * LR_DV + col] = S[t];
      if (col == 0) a.ztot[slot * a.r + t] = z[t];
    }
}

__host__ __device__ inline void lr_prefix_body(const LowrankArgs& a, int bh, int col) {
  for (int t = 0; t < a.r; ++t) {
    float run = 0.f, zrun = 0.f;
    for (int c = 0; c < a.nc; ++c) {
      const size_t slot = (size_t)bh * (a.nc + 1) + c;
      float* p = a.tot + (slot * a.r + t) * LR_DV + col;
      const float x = *p;
      *p = run;
      run += x;
      if (col == 0) {
        float* q = a.ztot + slot * a.r + t;
        const float y = *q;
        *q = zrun;
        zrun += y;
      }
    }
    const size_t last = (size_t)bh * (a.nc + 1) + a.nc;
    a.tot[(last * a.r + t) * LR_DV + col] = run;
    if (col == 0) a.ztot[last * a.r + t] = zrun;
  }
}

// Row chunk c (rows [c LR_C, min(Lq, (c+1) LR_C))) of head bh, value column col.
__host__ __device__ inline void lr_emit_body(const LowrankArgs& a, int c, int bh, int col) {
  const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.Hkv);
  const size_t slot = (size_t)bh * (a.nc + 1) + (a.causal ? a.n_lead + c : a.nc);
  float S[LR_RMAX], z[LR_RMAX];
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t) {
    S[t] = t < a.r ? a.tot[(slot * a.r + t) * LR_DV + col] : 0.f;
    z[t] = t < a.r ? a.ztot[slot * a.r + t] : 0.f;
  }
  const long long off = (long long)a.Lk - a.Lq;
  const __nv_bfloat16* vcol = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * LR_DV + col;
  const float* gh = a.G + (size_t)h * a.Lk * a.r;
  const long long r0 = (long long)c * LR_C;
  const long long r1 = r0 + LR_C < a.Lq ? r0 + LR_C : a.Lq;
  const float lam = a.lambda[h];
  const float* fh = a.F + (size_t)h * a.Lq * a.r;
  const float* arow = a.a1v + (size_t)bh * a.Lq * LR_DV + col;
  __nv_bfloat16* orow = a.out + (size_t)bh * a.Lq * LR_DV + col;
  for (long long i = r0; i < r1; ++i) {
    if (a.causal) {
      const long long j = i + off;
      if (j >= 0 && j < a.Lk) lr_add_key(a, vcol, gh, j, S, z);
    }
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int t = 0; t < LR_RMAX; ++t)
      if (t < a.r) {
        const float f = fh[i * a.r + t];
        num = fmaf(f, S[t], num);
        den = fmaf(f, z[t], den);
      }
    const float nv = den > 0.f ? num / den : 0.f;
    orow[i * LR_DV] = __float2bfloat16_rn(arow[i * LR_DV] - lam * nv);
  }
}

#ifdef __CUDACC__
__global__ void __launch_bounds__(LR_DV) lr_totals_kernel(LowrankArgs a) {
  lr_totals_body(a, (int)blockIdx.x, (int)blockIdx.y, (int)threadIdx.x);
}
__global__ void __launch_bounds__(LR_DV) lr_prefix_kernel(LowrankArgs a) {
  lr_prefix_body(a, (int)blockIdx.x, (int)threadIdx.x);
}
__global__ void __launch_bounds__(LR_DV) lr_emit_kernel(LowrankArgs a) {
  lr_emit_body(a, (int)blockIdx.x, (int)blockIdx.y, (int)threadIdx.x);
}
#endif

}  // namespace da
