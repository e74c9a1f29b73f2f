// lambda_simt.cuh -- the per-head lambda kernel and the exact fp32 SIMT
// forward used for f32 inputs (any head width, any query length).
#pragma once

#include "common.cuh"

namespace da {

// lambda[h] = exp(lq1[h].lk1[h]) - exp(lq2[h].lk2[h]) + lambda_init
// ("差分注意力" tutorial, Step 4 λ 参数化).  fp64 throughout: the products of
// two fp32 values are exact in fp64, the dot products are summed in index
// order, and the result is rounded once to fp32.
//
// One warp per head.  The warp stages a chunk of each of the four parameter
// rows in shared memory with coalesced loads; lane 0 then runs the sequential
// sums out of shared memory, so the order of the additions (and with it every
// bit of the result) is that of a plain loop over the index.
constexpr int LAM_WARPS = 4;      // heads per block
constexpr int LAM_CHUNK = 128;    // elements of each row staged at a time

__device__ __forceinline__ void lambda_dots(const float* __restrict__ lq1, const float* __restrict__ lk1,
                                            const float* __restrict__ lq2, const float* __restrict__ lk2,
                                            size_t base, int dim, float (*st)[LAM_CHUNK], int lane, double& d1,
                                            double& d2) {
  d1 = 0.0;
  d2 = 0.0;
  for (int c0 = 0; c0 < dim; c0 += LAM_CHUNK) {
    const int n = min(LAM_CHUNK, dim - c0);
    for (int i = lane; i < n; i += 32) {
      st[0][i] = lq1[base + c0 + i];
      st[1][i] = lk1[base + c0 + i];
      st[2][i] = lq2[base + c0 + i];
      st[3][i] = lk2[base + c0 + i];
    }
    __syncwarp();
    if (lane == 0) {
#pragma unroll 8
      for (int i = 0; i < n; ++i) {
        d1 = __dadd_rn(d1, __dmul_rn((double)st[0][i], (double)st[1][i]));
        d2 = __dadd_rn(d2, __dmul_rn((double)st[2][i], (double)st[3][i]));
      }
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(32 * LAM_WARPS)
lambda_kernel(const float* __restrict__ lq1, const float* __restrict__ lk1, const float* __restrict__ lq2,
              const float* __restrict__ lk2, int heads, int dim, double lambda_init, float* __restrict__ out) {
  __shared__ float st[LAM_WARPS][4][LAM_CHUNK];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * LAM_WARPS + w;
  if (h >= heads) return;   // warp-uniform
  double d1, d2;
  lambda_dots(lq1, lk1, lq2, lk2, (size_t)h * dim, dim, st[w], lane, d1, d2);
  if (lane == 0) out[h] = (float)__dadd_rn(__dsub_rn(exp(d1), exp(d2)), lambda_init);
}

// Gradients of the four λ parameter vectors given dlambda[h] (the chain rule
// of the λ above): dlq1 = g e1 lk1, dlk1 = g e1 lq1, dlq2 = -g e2 lk2,
// dlk2 = -g e2 lq2 with e_i = exp(lq_i . lk_i), in fp64, rounded once to f32.
// One warp per head: the dot products as in lambda_kernel, then every lane
// writes its share of the four gradient rows (coalesced).
__global__ void __launch_bounds__(32 * LAM_WARPS)
lambda_backward_kernel(const float* __restrict__ lq1, const float* __restrict__ lk1, const float* __restrict__ lq2,
                       const float* __restrict__ lk2, const float* __restrict__ dlambda, int heads, int dim,
                       float* __restrict__ dlq1, float* __restrict__ dlk1, float* __restrict__ dlq2,
                       float* __restrict__ dlk2) {
  __shared__ float st[LAM_WARPS][4][LAM_CHUNK];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * LAM_WARPS + w;
  if (h >= heads) return;   // warp-uniform
  const size_t base = (size_t)h * dim;
  double d1, d2, g1 = 0.0, g2 = 0.0;
  lambda_dots(lq1, lk1, lq2, lk2, base, dim, st[w], lane, d1, d2);
  if (lane == 0) {
    const double g = (double)dlambda[h];
    g1 = g * exp(d1);
    g2 = -g * exp(d2);
  }
  g1 = __shfl_sync(0xffffffffu, g1, 0);
  g2 = __shfl_sync(0xffffffffu, g2, 0);
  for (int i = lane; i < dim; i += 32) {
    dlq1[base + i] = (float)(g1 * (double)lk1[base + i]);
    dlk1[base + i] = (float)(g1 * (double)lq1[base + i]);
    dlq2[base + i] = (float)(g2 * (double)lk2[base + i]);
    dlk2[base + i] = (float)(g2 * (double)lq2[base + i]);
  }
}

// Where each operand of one (batch, output head) lives, for both layouts.
struct SimtArgs {
  const float* q1;   // V1: q1 [B,H,Lq,d];  V2: q [B,Hq,Lq,D]
  const float* q2;   // V1: q2;             V2: q (same tensor)
  const float* k1;   // V1: k1 [B,Hkv,Lk,d]; V2: k
  const float* k2;   // V1: k2;             V2: k (same tensor)
  const float* v;    // [B,Hkv,Lk,dv]
  const float* lambda;
  float* out;        // [B,Hout,Lq,dv]
  int B, Hout, Hq, Hkv, Lq, Lk, d, dv;
  int v2;            // 1: V2 pairing (Q heads 2h, 2h+1)
  int causal, rms;
  float eps, scale;
};

constexpr int SIMT_THREADS = 256;
constexpr int SIMT_MAXD = 256;
constexpr int SIMT_MAXCOL = 16;  // dv <= 16 * 256
constexpr int SIMT_CHUNK = 256;  // keys per weight chunk

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  for (int o = 16; o > 0; o >>= 1) {
    float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < SIMT_THREADS / 32; ++i) r = is_max ? fmaxf(r, red[i]) : r + red[i];
  return r;
}

// One CTA per (batch, output head, query row).  Three exact passes over the
// visible keys: row maxima, normalisers, then the weighted sum of V with
// weight A1 - lambda*A2 per key.  All fp32; expf is the full-precision one.
__global__ void __launch_bounds__(SIMT_THREADS) simt_forward_kernel(SimtArgs a) {
  __shared__ float sq1[SIMT_MAXD], sq2[SIMT_MAXD];
  __shared__ float sw[SIMT_CHUNK];
  __shared__ float red[SIMT_THREADS / 32];

  const int row = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.Hout, h = bh % a.Hout;
  const int tid = threadIdx.x;
  int hq1, hq2, g;
  if (a.v2) {
    hq1 = 2 * h; hq2 = 2 * h + 1; g = hq1 / (a.Hq / a.Hkv);
  } else {
    hq1 = h; hq2 = h; g = h / (a.Hq / a.Hkv);
  }
  const float* q1 = a.q1 + (((size_t)b * a.Hq + hq1) * a.Lq + row) * a.d;
  const float* q2 = a.q2 + (((size_t)b * a.Hq + hq2) * a.Lq + row) * a.d;
  const float* k1 = a.k1 + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * a.d;
  const float* k2 = a.k2 + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * a.d;
  const float* v = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lk * a.dv;
  float* out = a.out + (((size_t)b * a.Hout + h) * a.Lq + row) * a.dv;
  const float lam = a.lambda[h];

  for (int i = tid; i < a.d; i += SIMT_THREADS) { sq1[i] = q1[i]; sq2[i] = q2[i]; }
  __syncthreads();

  long long nvis_l = a.causal ? (long long)row + (a.Lk - a.Lq) + 1 : a.Lk;
  const int nvis = (int)max(0LL, min((long long)a.Lk, nvis_l));

  // pass 1: maxima
  float m1 = -INFINITY, m2 = -INFINITY;
  for (int j = tid; j < nvis; j += SIMT_THREADS) {
    float s1 = 0.f, s2 = 0.f;
    const float* r1 = k1 + (size_t)j * a.d;
    const float* r2 = k2 + (size_t)j * a.d;
    for (int t = 0; t < a.d; ++t) { s1 = fmaf(sq1[t], r1[t], s1); s2 = fmaf(sq2[t], r2[t], s2); }
    m1 = fmaxf(m1, s1 * a.scale);
    m2 = fmaxf(m2, s2 * a.scale);
  }
  m1 = block_reduce(m1, red, true);
  m2 = block_reduce(m2, red, true);
  // pass 2: normalisers
  float l1 = 0.f, l2 = 0.f;
  for (int j = tid; j < nvis; j += SIMT_THREADS) {
    float s1 = 0.f, s2 = 0.f;
    const float* r1 = k1 + (size_t)j * a.d;
    const float* r2 = k2 + (size_t)j * a.d;
    for (int t = 0; t < a.d; ++t) { s1 = fmaf(sq1[t], r1[t], s1); s2 = fmaf(sq2[t], r2[t], s2); }
    l1 += expf(s1 * a.scale - m1);
    l2 += expf(s2 * a.scale - m2);
  }
  l1 = block_reduce(l1, red, false);
  l2 = block_reduce(l2, red, false);
  const float c1 = nvis > 0 ? 1.f / l1 : 0.f;
  const float c2 = nvis > 0 ? lam / l2 : 0.f;

  // pass 3: weighted sum of V rows, SIMT_CHUNK keys at a time
  float acc[SIMT_MAXCOL];
#pragma unroll
  for (int i = 0; i < SIMT_MAXCOL; ++i) acc[i] = 0.f;
  for (int j0 = 0; j0 < nvis; j0 += SIMT_CHUNK) {
    const int j = j0 + tid;
    __syncthreads();
    if (tid < SIMT_CHUNK) {
      float w = 0.f;
      if (j < nvis) {
        float s1 = 0.f, s2 = 0.f;
        const float* r1 = k1 + (size_t)j * a.d;
        const float* r2 = k2 + (size_t)j * a.d;
        for (int t = 0; t < a.d; ++t) { s1 = fmaf(sq1[t], r1[t], s1); s2 = fmaf(sq2[t], r2[t], s2); }
        w = expf(s1 * a.scale - m1) * c1 - expf(s2 * a.scale - m2) * c2;
      }
      sw[tid] = w;
    }
    __syncthreads();
    const int jn = min(SIMT_CHUNK, nvis - j0);
    for (int jj = 0; jj < jn; ++jj) {
      const float w = sw[jj];
      const float* vr = v + (size_t)(j0 + jj) * a.dv;
#pragma unroll
      for (int i = 0; i < SIMT_MAXCOL; ++i) {
        const int c = tid + i * SIMT_THREADS;
        if (c < a.dv) acc[i] = fmaf(w, vr[c], acc[i]);
      }
    }
  }
  float rscale = 1.f;
  if (a.rms) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < SIMT_MAXCOL; ++i) {
      const int c = tid + i * SIMT_THREADS;
      if (c < a.dv) ss = fmaf(acc[i], acc[i], ss);
    }
    ss = block_reduce(ss, red, false);
    rscale = rsqrtf(ss / (float)a.dv + a.eps);
  }
#pragma unroll
  for (int i = 0; i < SIMT_MAXCOL; ++i) {
    const int c = tid + i * SIMT_THREADS;
    if (c < a.dv) out[c] = acc[i] * rscale;
  }
}

}  // namespace da
