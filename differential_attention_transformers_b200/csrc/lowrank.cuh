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
// One thread owns one of the 128 value columns and r <= LR_RMAX accumulators.
// The CTA first stages the factor rows its loop reads (the same for every
// column) in shared memory; keys and rows are then taken several at a time
// with their global loads issued first, so the passes are not bound by load
// latency.  Each kernel body is a host-device function of (chunk, head,
// column) that takes those rows as pointers, so the same code can be run over
// every index on the host.
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

// Adds keys [ks, ke) of one value column: S[t] += g_j[t] v_j, z[t] += g_j[t].
// vcol: the column (keys LR_DV apart); gk: the G rows of these keys, gk[(j -
// ks) r + t].  Keys in ascending order, U at a time with their V loads issued
// first, so U loads are in flight per thread.
__host__ __device__ inline void lr_add_keys(int r, const __nv_bfloat16* vcol, const float* gk, long long ks,
                                            long long ke, float (&S)[LR_RMAX], float (&z)[LR_RMAX]) {
  constexpr int U = 8;
  long long j = ks;
  for (; j + U <= ke; j += U) {
    float vj[U];
#pragma unroll
    for (int u = 0; u < U; ++u) vj[u] = __bfloat162float(vcol[(j + u) * LR_DV]);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float* g = gk + (j - ks + u) * r;
#pragma unroll
      for (int t = 0; t < LR_RMAX; ++t)
        if (t < r) {
          S[t] = fmaf(g[t], vj[u], S[t]);
          z[t] += g[t];
        }
    }
  }
  for (; j < ke; ++j) {
    const float vj = __bfloat162float(vcol[j * LR_DV]);
    const float* g = gk + (j - ks) * r;
#pragma unroll
    for (int t = 0; t < LR_RMAX; ++t)
      if (t < r) {
        S[t] = fmaf(g[t], vj, S[t]);
        z[t] += g[t];
      }
  }
}

// Slot c of head bh, value column col; gk: the G rows of the slot's keys
// [ks, ke) (lr_key_range), gk[(j - ks) r + t].
__host__ __device__ inline void lr_totals_body(const LowrankArgs& a, int c, int bh, int col, const float* gk) {
  const int b = bh / a.H, g = (bh % a.H) / (a.H / a.Hkv);
  long long ks, ke;
  lr_key_range(a, c, ks, ke);
  float S[LR_RMAX], z[LR_RMAX];
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t) S[t] = z[t] = 0.f;
  const __nv_bfloat16* vcol = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * LR_DV + col;
  lr_add_keys(a.r, vcol, gk, ks, ke, S, z);
  const size_t slot = (size_t)bh * (a.nc + 1) + c;
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t)
    if (t < a.r) {
      a.tot[(slot * a.r + t) * LR_DV + col] = S[t];
      if (col == 0) a.ztot[slot * a.r + t] = z[t];
    }
}

// Exclusive prefix over the slots of head bh, rank index t, value column col
// (and, for col == 0, of the z sums), plus the grand total in slot nc.  Eight
// slots' values are loaded before their prefix is formed.
__host__ __device__ inline void lr_prefix_body(const LowrankArgs& a, int bh, int t, int col) {
  constexpr int U = 8;
  float run = 0.f, zrun = 0.f;
  const size_t s0 = (size_t)bh * (a.nc + 1);
  for (int c0 = 0; c0 < a.nc; c0 += U) {
    float x[U], y[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + u < a.nc) {
        x[u] = a.tot[((s0 + c0 + u) * a.r + t) * LR_DV + col];
        if (col == 0) y[u] = a.ztot[(s0 + c0 + u) * a.r + t];
      }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + u < a.nc) {
        a.tot[((s0 + c0 + u) * a.r + t) * LR_DV + col] = run;
        run += x[u];
        if (col == 0) {
          a.ztot[(s0 + c0 + u) * a.r + t] = zrun;
          zrun += y[u];
        }
      }
  }
  a.tot[((s0 + a.nc) * a.r + t) * LR_DV + col] = run;
  if (col == 0) a.ztot[(s0 + a.nc) * a.r + t] = zrun;
}

// The rows of row chunk c and the keys they add (causal: row i adds key
// i + Lk - Lq; none when unmasked), clamped to the tensors.
__host__ __device__ inline void lr_emit_range(const LowrankArgs& a, int c, long long& r0, long long& r1,
                                              long long& k0, long long& k1) {
  r0 = (long long)c * LR_C;
  r1 = r0 + LR_C < a.Lq ? r0 + LR_C : a.Lq;
  const long long off = (long long)a.Lk - a.Lq;
  k0 = a.causal ? lr_clamp(r0 + off, a.Lk) : 0;
  k1 = a.causal ? lr_clamp(r1 + off, a.Lk) : 0;
}

// Row chunk c (rows [r0, r1)) of head bh, value column col.  fk: the F rows
// of the chunk, fk[(i - r0) r + t]; gk: the G rows of the keys the rows add,
// gk[(j - k0) r + t] (lr_emit_range).
__host__ __device__ inline void lr_emit_body(const LowrankArgs& a, int c, int bh, int col, const float* fk,
                                             const float* gk) {
  const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.Hkv);
  const size_t slot = (size_t)bh * (a.nc + 1) + (a.causal ? a.n_lead + c : a.nc);
  float S[LR_RMAX], z[LR_RMAX];
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t) {
    S[t] = t < a.r ? a.tot[(slot * a.r + t) * LR_DV + col] : 0.f;
    z[t] = t < a.r ? a.ztot[slot * a.r + t] : 0.f;
  }
  long long r0, r1, k0, k1;
  lr_emit_range(a, c, r0, r1, k0, k1);
  const long long off = (long long)a.Lk - a.Lq;
  const __nv_bfloat16* vcol = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * LR_DV + col;
  const float lam = a.lambda[h];
  const float* arow = a.a1v + (size_t)bh * a.Lq * LR_DV + col;
  __nv_bfloat16* orow = a.out + (size_t)bh * a.Lq * LR_DV + col;
  constexpr int U = 4;
  for (long long i0 = r0; i0 < r1; i0 += U) {
    // this group's loads first: A1 V of each row and the V value of the key it adds
    float av[U], vj[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long i = i0 + u, j = i + off;
      av[u] = i < r1 ? arow[i * LR_DV] : 0.f;
      vj[u] = (a.causal && i < r1 && j >= 0 && j < a.Lk) ? __bfloat162float(vcol[j * LR_DV]) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long i = i0 + u, j = i + off;
      if (i >= r1) break;
      if (a.causal && j >= 0 && j < a.Lk) {
        const float* gj = gk + (j - k0) * a.r;
#pragma unroll
        for (int t = 0; t < LR_RMAX; ++t)
          if (t < a.r) {
            S[t] = fmaf(gj[t], vj[u], S[t]);
            z[t] += gj[t];
          }
      }
      const float* fi = fk + (i - r0) * a.r;
      float num = 0.f, den = 0.f;
#pragma unroll
      for (int t = 0; t < LR_RMAX; ++t)
        if (t < a.r) {
          num = fmaf(fi[t], S[t], num);
          den = fmaf(fi[t], z[t], den);
        }
      const float nv = den > 0.f ? num / den : 0.f;
      orow[i * LR_DV] = __float2bfloat16_rn(av[u] - lam * nv);
    }
  }
}

#ifdef __CUDACC__
// Copies n floats from global memory into shared memory, all threads of the CTA.
__device__ __forceinline__ void lr_stage(float* dst, const float* src, long long n) {
  for (long long i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src[i];
  __syncthreads();
}

__global__ void __launch_bounds__(LR_DV) lr_totals_kernel(LowrankArgs a) {
  __shared__ float sg[LR_C * LR_RMAX];
  const int c = (int)blockIdx.x, bh = (int)blockIdx.y, h = bh % a.H;
  long long ks, ke;
  lr_key_range(a, c, ks, ke);
  lr_stage(sg, a.G + ((size_t)h * a.Lk + ks) * a.r, (ke - ks) * a.r);
  lr_totals_body(a, c, bh, (int)threadIdx.x, sg);
}
__global__ void __launch_bounds__(LR_DV) lr_prefix_kernel(LowrankArgs a) {
  lr_prefix_body(a, (int)blockIdx.y, (int)blockIdx.x, (int)threadIdx.x);
}
__global__ void __launch_bounds__(LR_DV) lr_emit_kernel(LowrankArgs a) {
  __shared__ float sf[LR_C * LR_RMAX];
  __shared__ float sg[LR_C * LR_RMAX];
  const int c = (int)blockIdx.x, bh = (int)blockIdx.y, h = bh % a.H;
  long long r0, r1, k0, k1;
  lr_emit_range(a, c, r0, r1, k0, k1);
  for (long long i = threadIdx.x; i < (r1 - r0) * a.r; i += blockDim.x) sf[i] = a.F[((size_t)h * a.Lq + r0) * a.r + i];
  lr_stage(sg, a.G + ((size_t)h * a.Lk + k0) * a.r, (k1 - k0) * a.r);
  lr_emit_body(a, c, bh, (int)threadIdx.x, sf, sg);
}
#endif

}  // namespace da
