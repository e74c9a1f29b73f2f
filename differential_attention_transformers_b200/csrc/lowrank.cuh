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
// column) in shared memory, each padded with zeros to LR_RMAX floats, so a row
// is four 16-byte loads and the rank loops run to LR_RMAX without a test (the
// padded ranks add exact zeros).  Keys and rows are then taken several at a
// time with their global loads issued first.  Each kernel body is a host-device function of (chunk, head,
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

// Element e of the padded copy of n rows of r factors (rows LR_RMAX apart,
// ranks >= r zero); src: the rows, r apart.
__host__ __device__ inline float lr_padded(const float* src, int r, long long e) {
  const int t = (int)(e % LR_RMAX);
  return t < r ? src[(e / LR_RMAX) * r + t] : 0.f;
}

// The LR_RMAX factors of one padded row (16-byte aligned).
__host__ __device__ inline void lr_row(const float* row, float (&x)[LR_RMAX]) {
#pragma unroll
  for (int q = 0; q < LR_RMAX / 4; ++q) {
    const float4 v = reinterpret_cast<const float4*>(row)[q];
    x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
  }
}

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

// Adds keys [ks, ke) of one value column: S[t] += g_j[t] v_j.  vcol: the
// column (keys LR_DV apart); gk: the padded G rows of these keys, row j - ks
// at gk + (j - ks) LR_RMAX.
// Keys in ascending order, U at a time; the V loads of the next U keys are
// issued before this group's arithmetic, so a group's memory latency overlaps
// the one before it.
__host__ __device__ inline void lr_add_keys(const __nv_bfloat16* vcol, const float* gk, long long ks, long long ke,
                                            float (&S)[LR_RMAX]) {
  constexpr int U = 8;
  float vj[U], vn[U];
#pragma unroll
  for (int u = 0; u < U; ++u) vj[u] = ks + u < ke ? __bfloat162float(vcol[(ks + u) * LR_DV]) : 0.f;
  for (long long j = ks; j < ke; j += U) {
#pragma unroll
    for (int u = 0; u < U; ++u) vn[u] = j + U + u < ke ? __bfloat162float(vcol[(j + U + u) * LR_DV]) : 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (j + u >= ke) break;
      float g[LR_RMAX];
      lr_row(gk + (j - ks + u) * LR_RMAX, g);
#pragma unroll
      for (int t = 0; t < LR_RMAX; ++t) S[t] = fmaf(g[t], vj[u], S[t]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) vj[u] = vn[u];
  }
}

// Slot c of head bh, value column col; gk: the padded G rows of the slot's
// keys [ks, ke) (lr_key_range).  The sums of g do not depend on the column:
// column t < r forms the one of rank t.
__host__ __device__ inline void lr_totals_body(const LowrankArgs& a, int c, int bh, int col, const float* gk) {
  const int b = bh / a.H, g = (bh % a.H) / (a.H / a.Hkv);
  long long ks, ke;
  lr_key_range(a, c, ks, ke);
  float S[LR_RMAX];
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t) S[t] = 0.f;
  const __nv_bfloat16* vcol = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * LR_DV + col;
  lr_add_keys(vcol, gk, ks, ke, S);
  const size_t slot = (size_t)bh * (a.nc + 1) + c;
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t)
    if (t < a.r) a.tot[(slot * a.r + t) * LR_DV + col] = S[t];
  if (col < a.r) {
    float z = 0.f;
    for (long long j = ks; j < ke; ++j) z += gk[(j - ks) * LR_RMAX + col];
    a.ztot[slot * a.r + col] = z;
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

// Slot of row chunk c of head bh: the prefix sums the chunk starts from.
__host__ __device__ inline size_t lr_emit_slot(const LowrankArgs& a, int c, int bh) {
  return (size_t)bh * (a.nc + 1) + (a.causal ? a.n_lead + c : a.nc);
}

// The key row i of a causal chunk adds (its G row at gk + (key - k0) LR_RMAX),
// or -1 when it adds none.
__host__ __device__ inline long long lr_row_key(const LowrankArgs& a, long long i, long long r1) {
  const long long j = i + ((long long)a.Lk - a.Lq);
  return (a.causal && i < r1 && j >= 0 && j < a.Lk) ? j : -1;
}

// The row normaliser of row chunk c of head bh, serially: rd[i - r0] =
// 1 / (f_i . z_i), or 0 when that is not positive, with z_i = the chunk's
// starting z plus the G rows of the keys rows r0..i add.  fk, gk as for
// lr_emit_body.  (The kernel forms the same sums in parallel, lr_emit_norm.)
__host__ __device__ inline void lr_emit_norm_serial(const LowrankArgs& a, int c, int bh, const float* fk,
                                                    const float* gk, float* rd) {
  const size_t slot = lr_emit_slot(a, c, bh);
  long long r0, r1, k0, k1;
  lr_emit_range(a, c, r0, r1, k0, k1);
  float z[LR_RMAX];
  for (int t = 0; t < LR_RMAX; ++t) z[t] = t < a.r ? a.ztot[slot * a.r + t] : 0.f;
  for (long long i = r0; i < r1; ++i) {
    const long long j = lr_row_key(a, i, r1);
    if (j >= 0)
      for (int t = 0; t < LR_RMAX; ++t) z[t] += gk[(j - k0) * LR_RMAX + t];
    float den = 0.f;
    for (int t = 0; t < LR_RMAX; ++t) den = fmaf(fk[(i - r0) * LR_RMAX + t], z[t], den);
    rd[i - r0] = den > 0.f ? 1.f / den : 0.f;
  }
}

// Row chunk c (rows [r0, r1)) of head bh, value column col.  fk: the padded F
// rows of the chunk, row i - r0 at fk + (i - r0) LR_RMAX; gk: the padded G
// rows of the keys the rows add, row j - k0 at gk + (j - k0) LR_RMAX
// (lr_emit_range); rd: the chunk's row normalisers (lr_emit_norm_serial).
__host__ __device__ inline void lr_emit_body(const LowrankArgs& a, int c, int bh, int col, const float* fk,
                                             const float* gk, const float* rd) {
  const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.Hkv);
  const size_t slot = lr_emit_slot(a, c, bh);
  float S[LR_RMAX];
#pragma unroll
  for (int t = 0; t < LR_RMAX; ++t) S[t] = t < a.r ? a.tot[(slot * a.r + t) * LR_DV + col] : 0.f;
  long long r0, r1, k0, k1;
  lr_emit_range(a, c, r0, r1, k0, k1);
  const __nv_bfloat16* vcol = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * LR_DV + col;
  const float lam = a.lambda[h];
  const float* arow = a.a1v + (size_t)bh * a.Lq * LR_DV + col;
  __nv_bfloat16* orow = a.out + (size_t)bh * a.Lq * LR_DV + col;
  // Rows U at a time; the loads of the next group (A1 V of each row and the
  // V value of the key it adds) are issued before this group's arithmetic,
  // so a group's memory latency overlaps the one before it.
  constexpr int U = 4;
  float av[U], vj[U], an[U], vn[U];
  auto load = [&](long long i0, float (&A)[U], float (&W)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long i = i0 + u, j = lr_row_key(a, i, r1);
      A[u] = i < r1 ? arow[i * LR_DV] : 0.f;
      W[u] = j >= 0 ? __bfloat162float(vcol[j * LR_DV]) : 0.f;
    }
  };
  load(r0, av, vj);
  for (long long i0 = r0; i0 < r1; i0 += U) {
    load(i0 + U, an, vn);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long i = i0 + u, j = lr_row_key(a, i, r1);
      if (i >= r1) break;
      if (j >= 0) {
        float gj[LR_RMAX];
        lr_row(gk + (j - k0) * LR_RMAX, gj);
#pragma unroll
        for (int t = 0; t < LR_RMAX; ++t) S[t] = fmaf(gj[t], vj[u], S[t]);
      }
      float fi[LR_RMAX];
      lr_row(fk + (i - r0) * LR_RMAX, fi);
      float num = 0.f;
#pragma unroll
      for (int t = 0; t < LR_RMAX; ++t) num = fmaf(fi[t], S[t], num);
      orow[i * LR_DV] = __float2bfloat16_rn(av[u] - lam * (num * rd[i - r0]));
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      av[u] = an[u];
      vj[u] = vn[u];
    }
  }
}

#ifdef __CUDACC__
// Stages n padded factor rows (lr_padded) into shared memory, all threads of the CTA.
__device__ __forceinline__ void lr_stage(float* dst, const float* src, int r, long long n) {
  for (long long e = threadIdx.x; e < n * LR_RMAX; e += blockDim.x) dst[e] = lr_padded(src, r, e);
  __syncthreads();
}

__global__ void __launch_bounds__(LR_DV) lr_totals_kernel(LowrankArgs a) {
  __shared__ alignas(16) float sg[LR_C * LR_RMAX];
  const int c = (int)blockIdx.x, bh = (int)blockIdx.y, h = bh % a.H;
  long long ks, ke;
  lr_key_range(a, c, ks, ke);
  lr_stage(sg, a.G + ((size_t)h * a.Lk + ks) * a.r, a.r, ke - ks);
  lr_totals_body(a, c, bh, (int)threadIdx.x, sg);
}
__global__ void __launch_bounds__(LR_DV) lr_prefix_kernel(LowrankArgs a) {
  lr_prefix_body(a, (int)blockIdx.y, (int)blockIdx.x, (int)threadIdx.x);
}
// The row normalisers of a chunk (as lr_emit_norm_serial), by the CTA's 128
// threads: thread t takes rank component t % 16 of the rows in segment t / 16
// (LR_C / 8 rows each).  The segments' sums of the added G rows go to seg;
// each thread then runs its component's prefix down its segment, and the 16
// threads of a segment (a half-warp) add their f_i[t] z_i[t] by shuffles.
// Every lane runs the same trip count, so the shuffles are warp-uniform.
constexpr int LR_SEGS = LR_DV / LR_RMAX;
constexpr int LR_SEG_ROWS = LR_C / LR_SEGS;
static_assert(LR_SEGS * LR_RMAX == LR_DV && LR_SEG_ROWS * LR_SEGS == LR_C, "normaliser thread layout");
__device__ __forceinline__ void lr_emit_norm(const LowrankArgs& a, int c, int bh, const float* fk, const float* gk,
                                             float* rd, float (*seg)[LR_RMAX]) {
  const int t = (int)threadIdx.x, q = t % LR_RMAX, sg = t / LR_RMAX;
  long long r0, r1, k0, k1;
  lr_emit_range(a, c, r0, r1, k0, k1);
  const long long i_beg = r0 + (long long)sg * LR_SEG_ROWS;
  float part = 0.f;
  for (int u = 0; u < LR_SEG_ROWS; ++u) {
    const long long j = lr_row_key(a, i_beg + u, r1);
    if (j >= 0) part += gk[(j - k0) * LR_RMAX + q];
  }
  seg[sg][q] = part;
  __syncthreads();
  const size_t slot = lr_emit_slot(a, c, bh);
  float z = q < a.r ? a.ztot[slot * a.r + q] : 0.f;
  for (int s2 = 0; s2 < sg; ++s2) z += seg[s2][q];
  for (int u = 0; u < LR_SEG_ROWS; ++u) {
    const long long i = i_beg + u, j = lr_row_key(a, i, r1);
    if (j >= 0) z += gk[(j - k0) * LR_RMAX + q];
    float p = i < r1 ? fk[(i - r0) * LR_RMAX + q] * z : 0.f;
#pragma unroll
    for (int o = LR_RMAX / 2; o >= 1; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
    if (q == 0 && i < r1) rd[i - r0] = p > 0.f ? 1.f / p : 0.f;
  }
  __syncthreads();
}

// Six CTAs per SM: the 33.5 KB of staged factor rows and normalisers allow no
// more, and the register budget keeps the prefetched group within it.
__global__ void __launch_bounds__(LR_DV, 6) lr_emit_kernel(LowrankArgs a) {
  __shared__ alignas(16) float sf[LR_C * LR_RMAX];
  __shared__ alignas(16) float sg[LR_C * LR_RMAX];
  __shared__ float srd[LR_C];
  __shared__ float sseg[LR_SEGS][LR_RMAX];
  const int c = (int)blockIdx.x, bh = (int)blockIdx.y, h = bh % a.H;
  long long r0, r1, k0, k1;
  lr_emit_range(a, c, r0, r1, k0, k1);
  for (long long e = threadIdx.x; e < (r1 - r0) * LR_RMAX; e += blockDim.x)
    sf[e] = lr_padded(a.F + ((size_t)h * a.Lq + r0) * a.r, a.r, e);
  lr_stage(sg, a.G + ((size_t)h * a.Lk + k0) * a.r, a.r, k1 - k0);
  lr_emit_norm(a, c, bh, sf, sg, srd, sseg);
  lr_emit_body(a, c, bh, (int)threadIdx.x, sf, sg, srd);
}
#endif

}  // namespace da
