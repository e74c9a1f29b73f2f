// Runs the low-rank scan kernels' bodies (lowrank.cuh) on the host, over every
// index and in launch order, so that their index arithmetic and results can be
// checked against the oracle without a GPU.
//
//   lowrank_host <input file> <output file>
//
// Input (little-endian): int32 B, H, Hkv, Lq, Lk, r, causal; then v bf16 bits
// [B, Hkv, Lk, 128]; F f32 [H, Lq, r]; G f32 [H, Lk, r]; lambda f32 [H];
// a1v f32 [B, H, Lq, 128].  Output: out bf16 bits [B, H, Lq, 128].
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../../differential_attention_transformers_b200/csrc/lowrank.cuh"

using da::LowrankArgs;

template <typename T>
static bool read_n(FILE* f, std::vector<T>& v, size_t n) {
  v.resize(n);
  return n == 0 || fread(v.data(), sizeof(T), n, f) == n;
}

int main(int argc, char** argv) {
  if (argc != 3) {
    fprintf(stderr, "usage: %s <in> <out>\n", argv[0]);
    return 2;
  }
  FILE* f = fopen(argv[1], "rb");
  if (!f) return 3;
  int32_t hdr[7];
  if (fread(hdr, sizeof(int32_t), 7, f) != 7) return 4;
  const int B = hdr[0], H = hdr[1], Hkv = hdr[2], Lq = hdr[3], Lk = hdr[4], r = hdr[5], causal = hdr[6];
  std::vector<uint16_t> v;
  std::vector<float> F, G, lam, a1v;
  const size_t BH = (size_t)B * H;
  if (!read_n(f, v, (size_t)B * Hkv * Lk * da::LR_DV) || !read_n(f, F, (size_t)H * Lq * r) ||
      !read_n(f, G, (size_t)H * Lk * r) || !read_n(f, lam, (size_t)H) || !read_n(f, a1v, BH * Lq * da::LR_DV))
    return 5;
  fclose(f);

  LowrankArgs a{};
  a.B = B; a.H = H; a.Hkv = Hkv; a.Lq = Lq; a.Lk = Lk; a.r = r; a.causal = causal;
  da::lr_slots(Lq, Lk, causal, a.n_lead, a.nc);
  std::vector<float> tot(BH * (a.nc + 1) * r * da::LR_DV, 0.f), ztot(BH * (a.nc + 1) * r, 0.f);
  std::vector<uint16_t> out(BH * Lq * da::LR_DV, 0);
  a.v = reinterpret_cast<const __nv_bfloat16*>(v.data());
  a.F = F.data();
  a.G = G.data();
  a.lambda = lam.data();
  a.a1v = a1v.data();
  a.out = reinterpret_cast<__nv_bfloat16*>(out.data());
  a.tot = tot.data();
  a.ztot = ztot.data();

  // The kernels stage the factor rows a CTA reads in shared memory, padded to
  // LR_RMAX floats a row; here the same padded rows are built per CTA.
  std::vector<float> pf, pg;
  auto pad = [&](std::vector<float>& dst, const float* src, long long n) {
    dst.assign((size_t)(n > 0 ? n : 0) * da::LR_RMAX, 0.f);
    for (long long e = 0; e < n * da::LR_RMAX; ++e) dst[e] = da::lr_padded(src, r, e);
  };
  if (a.nc > 0 && Lk > 0)
    for (int bh = 0; bh < (int)BH; ++bh)
      for (int c = 0; c < a.nc; ++c) {
        long long ks, ke;
        da::lr_key_range(a, c, ks, ke);
        pad(pg, G.data() + ((size_t)(bh % H) * Lk + ks) * r, ke - ks);
        for (int col = 0; col < da::LR_DV; ++col) da::lr_totals_body(a, c, bh, col, pg.data());
      }
  for (int bh = 0; bh < (int)BH; ++bh)
    for (int t = 0; t < r; ++t)
      for (int col = 0; col < da::LR_DV; ++col) da::lr_prefix_body(a, bh, t, col);
  const int nrc = (Lq + da::LR_C - 1) / da::LR_C;
  for (int bh = 0; bh < (int)BH; ++bh)
    for (int c = 0; c < nrc; ++c) {
      long long r0, r1, k0, k1;
      da::lr_emit_range(a, c, r0, r1, k0, k1);
      pad(pf, F.data() + ((size_t)(bh % H) * Lq + r0) * r, r1 - r0);
      pad(pg, G.data() + ((size_t)(bh % H) * Lk + k0) * r, k1 - k0);
      float rd[da::LR_C];
      da::lr_emit_norm_serial(a, c, bh, pf.data(), pg.data(), rd);
      for (int col = 0; col < da::LR_DV; ++col) da::lr_emit_body(a, c, bh, col, pf.data(), pg.data(), rd);
    }

  FILE* g = fopen(argv[2], "wb");
  if (!g) return 6;
  if (!out.empty() && fwrite(out.data(), sizeof(uint16_t), out.size(), g) != out.size()) return 7;
  fclose(g);
  return 0;
}
