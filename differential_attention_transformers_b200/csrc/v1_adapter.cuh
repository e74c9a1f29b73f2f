// v1_adapter.cuh -- the RMSNorm pass of the V1-layout backward.
//
// ("差分注意力" tutorial, section V1 到 V2 的 diff): a V1 head applies a
// per-head RMSNorm (unit weight, eps) to its difference output x,
//
//     y = r x,  r = 1 / sqrt(mean(x^2) + eps)   =>   dX = r (dY - y <y, dY> / n)
//
// and the attention backward (backward_sm100.cuh, V1 instantiations) then
// runs on dX.  This pass is an HBM-bound stream of 8-byte vectors.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace da {

constexpr int V1A_THREADS = 256;

// dX = r (dY - y <y, dY> / 128) per 128-wide row, one warp per row, 4 elements
// a lane.  y is the normalised forward output, r its saved 1/rms (0 for a row
// that saw no key, whose output and gradient are zero).
//
// The same pass forms the backward's row terms D_m = dX . O_m from the f32 dX
// (before its rounding to bf16), with the training forward's stored map
// outputs: O_1 / l_1 and, for map 2, its part orthogonal to the difference
// output X, O_2' = O_2 / l_2 - c X, and per row e = c eps r^2.  Since
//   dX . X = r (X . dY - r |X|^2 <y, dY> / n) = <y, dY> (1 - r^2 ms) = <y, dY> eps r^2
// (r^2 = 1 / (ms + eps)), D_2 = dX . O_2' + e <y, dY>: a sum whose terms are
// of the size of O_2', so its rounding no longer scales with the part of O_2
// along X that the sum cancels.  D [rows of (b, h), 2, Lq] f32.
struct V1RmsArgs {
  const __nv_bfloat16 *dy, *y;
  const float* rstd;
  __nv_bfloat16* dx;
  long long rows;
  const __nv_bfloat16* o_maps;   // [B*H, 2, Lq, 128]: O_1 / l_1, O_2 / l_2 - c X
  const float* o2c;              // [B*H, Lq]: e = c eps r^2
  float* dd;                     // [B*H, 2, Lq]: D_1, D_2
  int Lq;
};

__global__ void __launch_bounds__(V1A_THREADS) v1_rms_backward_kernel(V1RmsArgs a) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < a.rows;
       row += warps) {
    const uint2 gy = reinterpret_cast<const uint2*>(a.dy + row * 128)[lane];
    const uint2 yy = reinterpret_cast<const uint2*>(a.y + row * 128)[lane];
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gy);
    const __nv_bfloat162* y2 = reinterpret_cast<const __nv_bfloat162*>(&yy);
    float g[4], y[4];
    for (int j = 0; j < 2; ++j) {
      const float2 gf = __bfloat1622float2(g2[j]), yf = __bfloat1622float2(y2[j]);
      g[2 * j] = gf.x; g[2 * j + 1] = gf.y;
      y[2 * j] = yf.x; y[2 * j + 1] = yf.y;
    }
    float dot = 0.f;
    for (int j = 0; j < 4; ++j) dot = fmaf(g[j], y[j], dot);
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float r = a.rstd[row], c = dot * (1.f / 128.f);
    float dxf[4];
    for (int j = 0; j < 4; ++j) dxf[j] = r * fmaf(-y[j], c, g[j]);
    uint2 out;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&out);
    for (int j = 0; j < 2; ++j) o2[j] = __floats2bfloat162_rn(dxf[2 * j], dxf[2 * j + 1]);
    reinterpret_cast<uint2*>(a.dx + row * 128)[lane] = out;
    // D_1, D_2 from the f32 dX
    const long long bh = row / a.Lq, l = row - bh * a.Lq;
    float d[2];
    for (int m = 0; m < 2; ++m) {
      const uint2 ov = reinterpret_cast<const uint2*>(a.o_maps + ((bh * 2 + m) * a.Lq + l) * 128)[lane];
      const __nv_bfloat162* om = reinterpret_cast<const __nv_bfloat162*>(&ov);
      float s = 0.f;
      for (int j = 0; j < 2; ++j) {
        const float2 of = __bfloat1622float2(om[j]);
        s = fmaf(dxf[2 * j], of.x, s);
        s = fmaf(dxf[2 * j + 1], of.y, s);
      }
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      d[m] = s;
    }
    if (lane == 0) {
      a.dd[(bh * 2) * a.Lq + l] = d[0];
      a.dd[(bh * 2 + 1) * a.Lq + l] = fmaf(a.o2c[row], dot, d[1]);
    }
  }
}

}  // namespace da
