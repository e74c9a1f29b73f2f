// diffattn.cu -- C ABI of libdiffattn.so (declared in include/diffattn.h).
//
// Host side: argument validation (before any launch), TMA tensor-map
// encoding, launch configuration, the device status word.  All device work
// lives in the kernels included below; nothing here computes on the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/diffattn.h"
#include "common.cuh"
#include "decode.cuh"
#include "lambda_simt.cuh"
#include "prefill_sm100.cuh"
#include "backward_sm100.cuh"
#include "v1_adapter.cuh"
#include "lowrank.cuh"

using namespace da;

// |1 - lambda| below which the prefill keeps the bf16 residual of P (see
// PrefillArgs).  Without the residual the error of O relative to max|O| is
// about 5e-4 * (1+|lambda|)/|1-lambda| on near-uniform, alike maps: ~0.6 % at
// |1 - lambda| = 0.15, a third of the bf16 parity bound.
#ifndef DIFFATTN_RESID_TAU
#define DIFFATTN_RESID_TAU 0.15f
#endif

// Device status word (timeouts of bounded waits), one per device.
__device__ unsigned g_diffattn_status;

namespace {

thread_local std::string t_last_error;
std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int ok() {
  t_last_error.clear();
  return DIFFATTN_OK;
}

#define CUDA_TRY(expr)                                                                  \
  do {                                                                                  \
    cudaError_t e_ = (expr);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(DIFFATTN_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));   \
  } while (0)

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  int sms = 0;
  unsigned* status = nullptr;
  bool attrs_set = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

template <int DQK>
constexpr size_t prefill_smem() { return sizeof(PfSmem<DQK>) + 1024; }
constexpr int kDecNst = 2;
constexpr size_t decode_smem() { return sizeof(DecSmem<kDecNst>) + 1024; }
constexpr size_t decode_paged_smem() { return sizeof(DecSmem<kDecNst, true>) + 1024; }
constexpr size_t bwd_dq_smem() { return sizeof(BwQSmem) + 1024; }
constexpr size_t bwd_dkv_smem() { return sizeof(BwKSmem) + 1024; }
static_assert(bwd_dq_smem() <= 227 * 1024 && bwd_dkv_smem() <= 227 * 1024,
              "backward shared memory above the 227 KB a block may use");
// the dS buffer holds 128 rows of 128 bf16 keys as two 16 KB boxes, and also
// the epilogue's staging (8 warps x 16 rows x 128 bytes)
static_assert(sizeof(BwQSmem::ds) == 2 * 128 * 128 && sizeof(BwQSmem::ds) >= 8 * 16 * 128, "dS buffer size");
constexpr int kDecCtasPerSm = 2;

// Per-device set-up: SM count, status word address, kernel attributes,
// tensor-map encoder.  Called with the target device current.
int device_setup(DeviceInfo** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(DIFFATTN_ERR_CUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0;
    CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    if (major != 10 || minor != 0)
      return fail(DIFFATTN_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                  major, minor);
    CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    void* p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_diffattn_status));
    d.status = static_cast<unsigned*>(p);
    CUDA_TRY(cudaFuncSetAttribute(prefill_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)prefill_smem<64>()));
    CUDA_TRY(cudaFuncSetAttribute(prefill_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)prefill_smem<128>()));
    CUDA_TRY(cudaFuncSetAttribute(prefill_kernel<128, PF_TRAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)prefill_smem<128>()));
    CUDA_TRY(cudaFuncSetAttribute(prefill_kernel<64, PF_TRAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)prefill_smem<64>()));
    CUDA_TRY(cudaFuncSetAttribute(prefill_kernel<128, PF_SINGLE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)prefill_smem<128>()));
    CUDA_TRY(cudaFuncSetAttribute(decode_split_kernel<kDecNst>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)decode_smem()));
    CUDA_TRY(cudaFuncSetAttribute(decode_split_kernel<kDecNst, true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)decode_paged_smem()));
    CUDA_TRY(cudaFuncSetAttribute(bwd_dq_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)bwd_dq_smem()));
    CUDA_TRY(cudaFuncSetAttribute(bwd_dq_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)bwd_dq_smem()));
    CUDA_TRY(cudaFuncSetAttribute(bwd_dkv_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)bwd_dkv_smem()));
    CUDA_TRY(cudaFuncSetAttribute(bwd_dkv_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)bwd_dkv_smem()));
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      CUDA_TRY(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || !fn)
        return fail(DIFFATTN_ERR_CUDA, "cuTensorMapEncodeTiled not available from the driver");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.init = true;
  }
  *out = &d;
  return DIFFATTN_OK;
}

Watch make_watch(const DeviceInfo* d) { return Watch{d->status, g_wait_limit_ns.load()}; }

// 3-D bf16 tensor map over a contiguous [Z, Y, X] tensor, box {64, box_y, 1},
// 128-byte swizzle, zero fill outside the tensor.
int make_map(CUtensorMap* m, const void* base, int X, long long Y, long long Z, int box_y) {
  cuuint64_t dims[3] = {(cuuint64_t)X, (cuuint64_t)Y, (cuuint64_t)Z};
  cuuint64_t strides[2] = {(cuuint64_t)X * 2, (cuuint64_t)X * 2 * (cuuint64_t)Y};
  cuuint32_t box[3] = {64, (cuuint32_t)box_y, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DIFFATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DIFFATTN_OK;
}

// 4-D bf16 tensor map over a token-major page pool [num_pages, page_size, Hkv,
// 128]: box {64 dims, 1 head, min(page_size, 64) tokens, 1 page}, 128-byte
// swizzle, zero fill outside the pool (so a page id out of range reads zeros).
int make_map_paged(CUtensorMap* m, const void* base, int Hkv, int page_size, int num_pages) {
  cuuint64_t dims[4] = {128, (cuuint64_t)Hkv, (cuuint64_t)page_size, (cuuint64_t)num_pages};
  cuuint64_t strides[3] = {256, (cuuint64_t)Hkv * 256, (cuuint64_t)page_size * Hkv * 256};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)std::min(page_size, DEC_KB), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DIFFATTN_ERR_CUDA, "cuTensorMapEncodeTiled (paged) failed (%d)", (int)r);
  return DIFFATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_bf16_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!aligned16(p)) return fail(DIFFATTN_ERR_MISALIGNED, "bf16 tensor pointer %p is not 16-byte aligned", p);
  return DIFFATTN_OK;
}

float log2e_over_sqrt(int d) { return (float)(1.4426950408889634 / std::sqrt((double)d)); }

int launch_simt(const SimtArgs& a, cudaStream_t s) {
  if (a.Lq == 0 || a.B == 0 || a.Hout == 0) return ok();
  if ((long long)a.B * a.Hout > 65535) return fail(DIFFATTN_ERR_UNSUPPORTED, "B * heads > 65535 on the f32 path");
  dim3 grid((unsigned)a.Lq, (unsigned)(a.B * a.Hout));
  simt_forward_kernel<<<grid, SIMT_THREADS, 0, s>>>(a);
  CUDA_TRY(cudaGetLastError());
  return ok();
}

// Launch order of the prefill's row blocks (see PrefillArgs::rb_group).  When
// every output head has K/V of its own (V1 without GQA: 2 MB of K1, K2 and V
// per head at N = 4096, 256 MB over the workload's 128 heads), row blocks of
// one head launched BH CTAs apart find its K/V evicted from L2; grouping 4 row
// blocks of a head keeps them co-resident.  With GQA the output heads of a KV
// group are already adjacent.  DIFFATTN_PREFILL_RB_GROUP overrides the choice.
int prefill_rb_group(bool v1, int Hq, int Hkv, int n_rb) {
  int r = (v1 && Hq == Hkv) ? 4 : 1;
  if (const char* e = std::getenv("DIFFATTN_PREFILL_RB_GROUP")) {
    const int x = std::atoi(e);
    if (x >= 1) r = x;
  }
  return std::max(1, std::min(r, std::max(1, n_rb)));
}

int launch_prefill(const void* q1, const void* q2, const void* k1, const void* k2, const void* v,
                   const float* lambda, void* out, int B, int Hout, int Hq, int Hkv, int Lq, int Lk, int dqk,
                   bool v1, int causal, int rms, float eps, cudaStream_t s, float* lse = nullptr,
                   void* o_maps = nullptr, float* rstd = nullptr, float* o_f32 = nullptr, float* o2c = nullptr) {
  DeviceInfo* dev = nullptr;
  if (int e = device_setup(&dev)) return e;
  if (Lq == 0 || B == 0 || Hout == 0) return ok();
  CUtensorMap mq1, mq2, mk1, mk2, mv;
  // Q maps: V2 reads both maps from one tensor [B*Hq, Lq, dqk]
  if (int e = make_map(&mq1, q1, dqk, Lq, (long long)B * Hq, PF_BM)) return e;
  if (int e = make_map(&mq2, q2, dqk, Lq, (long long)B * Hq, PF_BM)) return e;
  const long long Lk_map = Lk > 0 ? Lk : 1;  // a zero extent is not encodable; Lk == 0 launches no loads
  if (int e = make_map(&mk1, k1, dqk, Lk_map, (long long)B * Hkv, PF_BN)) return e;
  if (int e = make_map(&mk2, k2, dqk, Lk_map, (long long)B * Hkv, PF_BN)) return e;
  if (int e = make_map(&mv, v, PF_DV, Lk_map, (long long)B * Hkv, PF_BN)) return e;
  PrefillArgs a;
  a.lambda = lambda;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.B = B; a.Hout = Hout; a.Hq = Hq; a.Hkv = Hkv; a.Lq = Lq; a.Lk = Lk;
  a.v1 = v1 ? 1 : 0;
  a.causal = causal ? 1 : 0;
  a.rms = rms ? 1 : 0;
  a.eps = eps;
  a.scale_log2 = log2e_over_sqrt(dqk);
  a.n_rb = (Lq + PF_BM - 1) / PF_BM;
  a.rb_group = prefill_rb_group(v1, Hq, Hkv, a.n_rb);
  a.resid_tau = DIFFATTN_RESID_TAU;
  a.watch = make_watch(dev);
  a.lse = lse;
  a.o_maps = static_cast<__nv_bfloat16*>(o_maps);
  a.rstd = rstd;
  a.o2c = o2c;
  a.o_f32 = o_f32;
  const long long units = (long long)a.n_rb * B * Hout;
  if (units > 0x7fffffffLL) return fail(DIFFATTN_ERR_UNSUPPORTED, "too many row blocks");
  if (o_f32 != nullptr)               // single-map outputs (V2 layout)
    prefill_kernel<128, PF_SINGLE><<<(unsigned)units, PF_THREADS, prefill_smem<128>(), s>>>(mq1, mq2, mk1, mk2, mv,
                                                                                           a);
  else if (lse != nullptr && dqk == 128)   // training forward (V2)
    prefill_kernel<128, PF_TRAIN><<<(unsigned)units, PF_THREADS, prefill_smem<128>(), s>>>(mq1, mq2, mk1, mk2, mv, a);
  else if (lse != nullptr)            // training forward (V1, d = 64)
    prefill_kernel<64, PF_TRAIN><<<(unsigned)units, PF_THREADS, prefill_smem<64>(), s>>>(mq1, mq2, mk1, mk2, mv, a);
  else if (dqk == 64)
    prefill_kernel<64><<<(unsigned)units, PF_THREADS, prefill_smem<64>(), s>>>(mq1, mq2, mk1, mk2, mv, a);
  else
    prefill_kernel<128><<<(unsigned)units, PF_THREADS, prefill_smem<128>(), s>>>(mq1, mq2, mk1, mk2, mv, a);
  CUDA_TRY(cudaGetLastError());
  return ok();
}

struct DecodePlan {
  int grid = 1;
  int maxseg = 1;
  long long nblk = 0, total = 0;
  size_t bytes_per_pass = 0;
};

DecodePlan plan_decode(int sms, int B, int Hkv, int T) {
  DecodePlan p;
  p.nblk = ((long long)T + DEC_KB - 1) / DEC_KB;
  p.total = (long long)B * Hkv * p.nblk;
  long long g = (long long)sms * kDecCtasPerSm;
  if (g > p.total) g = p.total;
  if (g < 1) g = 1;
  p.grid = (int)g;
  const long long per = (p.total + p.grid - 1) / p.grid;
  p.maxseg = p.nblk > 0 ? (int)((per + p.nblk - 1) / p.nblk + 1) : 1;
  p.bytes_per_pass = (size_t)p.grid * p.maxseg * DEC_REC * sizeof(float);
  return p;
}

int launch_decode(const void* q1, const void* q2, const void* k1, const void* k2, const void* v,
                  const float* lambda, void* out, int B, int Hq, int Hkv, int T, bool v1, int fused, void* ws,
                  size_t ws_bytes, cudaStream_t s) {
  DeviceInfo* dev = nullptr;
  if (int e = device_setup(&dev)) return e;
  if (B == 0) return ok();
  const DecodePlan p = plan_decode(dev->sms, B, Hkv, T);
  const int passes = (v1 && !fused) ? 2 : 1;
  const size_t need = p.bytes_per_pass * passes;
  if (p.total > 0 && (ws == nullptr || ws_bytes < need))
    return fail(DIFFATTN_ERR_WORKSPACE, "decode workspace %zu B < required %zu B", ws_bytes, need);
  if (p.total > 0 && !aligned16(ws)) return fail(DIFFATTN_ERR_MISALIGNED, "workspace not 16-byte aligned");
  if (p.total > 0) {
    CUtensorMap mk1, mk2, mv;
    const int dk = v1 ? 64 : 128;
    if (int e = make_map(&mk1, k1, dk, T, (long long)B * Hkv, DEC_KB)) return e;
    if (int e = make_map(&mk2, v1 ? k2 : k1, dk, T, (long long)B * Hkv, DEC_KB)) return e;
    if (int e = make_map(&mv, v, 128, T, (long long)B * Hkv, DEC_KB)) return e;
    DecodeArgs a{};
    a.q1 = static_cast<const __nv_bfloat16*>(q1);
    a.q2 = static_cast<const __nv_bfloat16*>(v1 ? q2 : q1);
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T = T;
    a.v1 = v1 ? 1 : 0;
    a.grid = p.grid; a.maxseg = p.maxseg; a.nblk = p.nblk; a.total = p.total;
    a.scale_log2 = log2e_over_sqrt(dk);
    a.watch = make_watch(dev);
    for (int pass = 0; pass < passes; ++pass) {
      a.maps = passes == 1 ? 3 : (1 << pass);
      a.ws = static_cast<float*>(ws) + (size_t)pass * (p.bytes_per_pass / sizeof(float));
      decode_split_kernel<kDecNst><<<p.grid, DEC_THREADS, decode_smem(), s>>>(mk1, mk2, mv, a);
      CUDA_TRY(cudaGetLastError());
    }
  }
  CombineArgs c{};
  c.ws = static_cast<const float*>(ws);
  c.lambda = lambda;
  c.out = static_cast<__nv_bfloat16*>(out);
  c.B = B; c.Hq = Hq; c.Hkv = Hkv; c.v1 = v1 ? 1 : 0;
  c.grid = p.grid; c.maxseg = p.maxseg; c.nblk = p.nblk; c.total = p.total;
  c.two_pass = passes == 2 ? 1 : 0;
  c.half_floats = p.bytes_per_pass / sizeof(float);
  c.cu = nullptr;
  decode_combine_kernel<<<(unsigned)(B * Hkv), 128, 0, s>>>(c);   // one CTA per (batch, KV head)
  CUDA_TRY(cudaGetLastError());
  return ok();
}

// Backward workspace: padded log-sum-exp and D values [B, Hp, 2, Lp] (Lp = Lq
// rounded up to 128; +inf / 0 past Lq), then the dlambda partials [B*Hp, Lp/64].
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
int bwd_rows_padded(int Lq) { return (Lq + PF_BM - 1) / PF_BM * PF_BM; }
size_t bwd_ws_bytes(int B, int Hq, int Lq) {
  const size_t Hp = (size_t)Hq / 2, Lp = (size_t)bwd_rows_padded(Lq);
  return 2 * align256((size_t)B * Hp * 2 * Lp * 4) + align256((size_t)B * Hp * (Lp / 64) * 4);
}

// Both layouts.  V2 (v1 = false): q [B, Hq, Lq, 128], k, v [B, Hkv, Lk, 128];
// q2, k2, dq2 and dk2 are unused.  V1 (v1 = true): Q head qh of Hq = 2H is map
// qh & 1 of V1 head qh / 2, so q, q2 are Q1, Q2 [B, H, Lq, 64], k, k2 are K1,
// K2 [B, Hkv, Lk, 64], and dq, dq2, dk, dk2 their gradients; the score scale
// is then 1/sqrt(64).  dout is [B, Hq/2, Lq, 128] in both.  d_in: the row
// terms D_m formed upstream (V1 with RMSNorm), else null.
int launch_backward(const void* q, const void* q2, const void* k, const void* k2, const void* v,
                    const float* lambda, const void* dout, const float* lse, const void* o_maps, void* dq, void* dq2,
                    void* dk, void* dk2, void* dv, float* dlambda, int B, int Hq, int Hkv, int Lq, int Lk, int causal,
                    void* ws, size_t ws_bytes, cudaStream_t s, bool v1, const float* d_in = nullptr) {
  DeviceInfo* dev = nullptr;
  if (int e = device_setup(&dev)) return e;
  const size_t need = bwd_ws_bytes(B, Hq, Lq);
  if (ws == nullptr || ws_bytes < need)
    return fail(DIFFATTN_ERR_WORKSPACE, "backward workspace %zu B < required %zu B", ws_bytes, need);
  if (!aligned16(ws)) return fail(DIFFATTN_ERR_MISALIGNED, "workspace not 16-byte aligned");
  const int Hp = Hq / 2, Lp = bwd_rows_padded(Lq);
  const int w = v1 ? 64 : 128;   // QK width
  float* nlse = static_cast<float*>(ws);
  float* ndd = reinterpret_cast<float*>(static_cast<char*>(ws) + align256((size_t)B * Hp * 2 * Lp * 4));
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + 2 * align256((size_t)B * Hp * 2 * Lp * 4));
  if (Lp > 0) {
    BwdPrepArgs pa{static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(o_maps), lse,
                   nlse, ndd, part, B, Hp, Lq, Lp, d_in};
    bwd_prep_kernel<<<dim3((unsigned)(Lp / 64), (unsigned)(B * Hp)), 256, 0, s>>>(pa);
    CUDA_TRY(cudaGetLastError());
  }
  bwd_dlambda_kernel<<<(Hp + 127) / 128, 128, 0, s>>>(part, dlambda, B, Hp, Lp / 64);
  CUDA_TRY(cudaGetLastError());
  BwdArgs a{};
  a.lambda = lambda; a.nlse = nlse; a.ndd = ndd;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dq2 = static_cast<__nv_bfloat16*>(dq2);
  a.dk2 = static_cast<__nv_bfloat16*>(dk2);
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Lq = Lq; a.Lk = Lk; a.Lp = Lp;
  a.causal = causal ? 1 : 0;
  a.scale = (float)(1.0 / std::sqrt((double)w));
  a.scale_log2 = log2e_over_sqrt(w);
  a.resid_tau = DIFFATTN_RESID_TAU;
  a.watch = make_watch(dev);
  if (!v1) { q2 = q; k2 = k; }
  const long long Lk_map = Lk > 0 ? Lk : 1;   // a zero extent is not encodable; no key is then loaded
  const long long Lq_map = Lq > 0 ? Lq : 1;
  const long long zq = v1 ? (long long)B * Hp : (long long)B * Hq;   // Q rows' third coordinate extent
  if (Lq > 0) {   // dQ: one CTA per 128 rows of each Q head
    CUtensorMap mq, mq2, mo, mk, mk2, mv;
    if (int e = make_map(&mq, q, w, Lq_map, zq, PF_BM)) return e;
    if (int e = make_map(&mq2, q2, w, Lq_map, zq, PF_BM)) return e;
    if (int e = make_map(&mo, dout, 128, Lq_map, (long long)B * Hp, PF_BM)) return e;
    if (int e = make_map(&mk, Lk > 0 ? k : q, w, Lk_map, (long long)B * Hkv, BWQ_BN)) return e;
    if (int e = make_map(&mk2, Lk > 0 ? k2 : q, w, Lk_map, (long long)B * Hkv, BWQ_BN)) return e;
    if (int e = make_map(&mv, Lk > 0 ? v : dout, 128, Lk_map, (long long)B * Hkv, BWQ_BN)) return e;
    const long long units = (long long)((Lq + PF_BM - 1) / PF_BM) * B * Hq;
    if (v1)
      bwd_dq_kernel<true><<<(unsigned)units, BW_THREADS, bwd_dq_smem(), s>>>(mq, mq2, mo, mk, mk2, mv, a);
    else
      bwd_dq_kernel<false><<<(unsigned)units, BW_THREADS, bwd_dq_smem(), s>>>(mq, mq2, mo, mk, mk2, mv, a);
    CUDA_TRY(cudaGetLastError());
  }
  if (Lk > 0) {   // dK, dV: one CTA per 128 keys of each KV head
    CUtensorMap mk, mk2, mv, mq, mq2, mo;
    if (int e = make_map(&mk, k, w, Lk_map, (long long)B * Hkv, PF_BM)) return e;
    if (int e = make_map(&mk2, k2, w, Lk_map, (long long)B * Hkv, PF_BM)) return e;
    if (int e = make_map(&mv, v, 128, Lk_map, (long long)B * Hkv, PF_BM)) return e;
    if (int e = make_map(&mq, Lq > 0 ? q : k, w, Lq_map, zq, BW_RB)) return e;
    if (int e = make_map(&mq2, Lq > 0 ? q2 : k, w, Lq_map, zq, BW_RB)) return e;
    if (int e = make_map(&mo, Lq > 0 ? dout : v, 128, Lq_map, (long long)B * Hp, BW_RB)) return e;
    const long long units = (long long)((Lk + PF_BM - 1) / PF_BM) * B * Hkv;
    if (v1)
      bwd_dkv_kernel<true><<<(unsigned)units, BW_THREADS, bwd_dkv_smem(), s>>>(mk, mk2, mv, mq, mq2, mo, a);
    else
      bwd_dkv_kernel<false><<<(unsigned)units, BW_THREADS, bwd_dkv_smem(), s>>>(mk, mk2, mv, mq, mq2, mo, a);
    CUDA_TRY(cudaGetLastError());
  }
  return ok();
}

// V1 backward workspace: with RMSNorm only, the input gradient dX (B*H*Lq
// rows of 128) and the row terms D_m [B*H, 2, Lq] f32; then the backward's
// own workspace.
struct V1BwdLayout {
  size_t dx, dd, bw, total;
};
V1BwdLayout v1_bwd_layout(int B, int H, int Hkv, int Lq, int Lk, int rms) {
  (void)Hkv;
  (void)Lk;
  const size_t nq = (size_t)B * H * Lq;
  V1BwdLayout l;
  l.dx = 0;
  l.dd = l.dx + (rms ? align256(nq * 256) : 0);
  l.bw = l.dd + (rms ? align256(nq * 2 * 4) : 0);
  l.total = l.bw + bwd_ws_bytes(B, 2 * H, Lq);
  return l;
}

unsigned stream_grid(const DeviceInfo* dev, long long items, int per_block) {
  long long g = (items + per_block - 1) / per_block;
  const long long cap = (long long)dev->sms * 8;
  return (unsigned)(g < 1 ? 1 : (g > cap ? cap : g));
}

int launch_backward_v1(const void* q1, const void* k1, const void* q2, const void* k2, const void* v,
                       const float* lambda, const void* dout, const void* out, const float* lse, const void* o_maps,
                       const float* rstd, const float* o2c, void* dq1, void* dk1, void* dq2, void* dk2, void* dv,
                       float* dlambda, int B, int H, int Hkv, int Lq, int Lk, int causal, int rms, void* ws,
                       size_t ws_bytes, cudaStream_t s) {
  DeviceInfo* dev = nullptr;
  if (int e = device_setup(&dev)) return e;
  const V1BwdLayout L = v1_bwd_layout(B, H, Hkv, Lq, Lk, rms);
  if (ws == nullptr || ws_bytes < L.total)
    return fail(DIFFATTN_ERR_WORKSPACE, "V1 backward workspace %zu B < required %zu B", ws_bytes, L.total);
  if (!aligned16(ws)) return fail(DIFFATTN_ERR_MISALIGNED, "workspace not 16-byte aligned");
  char* w = static_cast<char*>(ws);
  const long long nq = (long long)B * H * Lq;
  const void* g = dout;
  const float* d_in = nullptr;
  if (rms && nq > 0) {
    float* dd = reinterpret_cast<float*>(w + L.dd);
    V1RmsArgs ra{static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(out), rstd,
                 reinterpret_cast<__nv_bfloat16*>(w + L.dx), nq, static_cast<const __nv_bfloat16*>(o_maps), o2c, dd,
                 Lq};
    v1_rms_backward_kernel<<<stream_grid(dev, nq, V1A_THREADS / 32), V1A_THREADS, 0, s>>>(ra);
    CUDA_TRY(cudaGetLastError());
    g = w + L.dx;
    d_in = dd;
  }
  return launch_backward(q1, q2, k1, k2, v, lambda, g, lse, o_maps, dq1, dq2, dk1, dk2, dv, dlambda, B, 2 * H, Hkv,
                         Lq, Lk, causal, w + L.bw, ws_bytes - L.bw, s, true, d_in);
}

// Low-rank forward workspace: the per-head single-map outputs A1 V
// [B, H, Lq, 128] f32, then the chunk sums [B*H, nc+1, r, 128] and
// [B*H, nc+1, r] f32.
struct LowrankLayout {
  size_t a1v, tot, ztot, total;
  int n_lead, nc;
};
LowrankLayout lowrank_layout(int B, int H, int Lq, int Lk, int r, int causal) {
  LowrankLayout l;
  lr_slots(Lq, Lk, causal, l.n_lead, l.nc);
  const size_t BH = (size_t)B * H;
  l.a1v = 0;
  l.tot = l.a1v + align256(BH * Lq * LR_DV * 4);
  l.ztot = l.tot + align256(BH * (l.nc + 1) * r * LR_DV * 4);
  l.total = l.ztot + align256(BH * (l.nc + 1) * r * 4);
  return l;
}

// Paged decode workspace: the block prefix (B+1 ints, padded to 256 bytes),
// then one partial record per slot CTA + b*Hkv + g, i.e. grid + B*Hkv records.
int paged_grid(const DeviceInfo* dev) { return dev->sms * kDecCtasPerSm; }
size_t paged_prefix_bytes(int B) { return ((size_t)(B + 1) * sizeof(int) + 255) & ~(size_t)255; }
size_t paged_ws_bytes(const DeviceInfo* dev, int B, int Hkv) {
  return paged_prefix_bytes(B) + ((size_t)paged_grid(dev) + (size_t)B * Hkv) * DEC_REC * sizeof(float);
}

int launch_decode_paged(const void* q, const void* kp, const void* vp, const int* table, const int* lens,
                        const float* lambda, void* out, int B, int Hq, int Hkv, int num_pages, int page_size,
                        int max_pages, void* ws, size_t ws_bytes, cudaStream_t s) {
  DeviceInfo* dev = nullptr;
  if (int e = device_setup(&dev)) return e;
  const size_t need = paged_ws_bytes(dev, B, Hkv);
  if (ws == nullptr || ws_bytes < need)
    return fail(DIFFATTN_ERR_WORKSPACE, "paged decode workspace %zu B < required %zu B", ws_bytes, need);
  if (!aligned16(ws)) return fail(DIFFATTN_ERR_MISALIGNED, "workspace not 16-byte aligned");
  CUtensorMap mk, mv;
  if (int e = make_map_paged(&mk, kp, Hkv, page_size, num_pages)) return e;
  if (int e = make_map_paged(&mv, vp, Hkv, page_size, num_pages)) return e;
  int* cu = static_cast<int*>(ws);
  float* rec = reinterpret_cast<float*>(static_cast<char*>(ws) + paged_prefix_bytes(B));
  DecodeArgs a{};
  a.q1 = a.q2 = static_cast<const __nv_bfloat16*>(q);
  a.ws = rec;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T = 0;
  a.v1 = 0; a.maps = 3;
  a.grid = paged_grid(dev); a.maxseg = 0; a.nblk = 0; a.total = 0;
  a.scale_log2 = log2e_over_sqrt(128);
  a.watch = make_watch(dev);
  a.block_table = table; a.seq_lens = lens; a.cu_out = cu;
  a.max_pages = max_pages; a.page_size = page_size;
  a.page_shift = 0;
  while ((1 << a.page_shift) < page_size) ++a.page_shift;
  decode_split_kernel<kDecNst, true><<<a.grid, DEC_THREADS, decode_paged_smem(), s>>>(mk, mk, mv, a);
  CUDA_TRY(cudaGetLastError());
  CombineArgs c{};
  c.ws = rec;
  c.lambda = lambda;
  c.out = static_cast<__nv_bfloat16*>(out);
  c.B = B; c.Hq = Hq; c.Hkv = Hkv; c.v1 = 0;
  c.grid = a.grid; c.maxseg = 0; c.nblk = 0; c.total = 0;
  c.two_pass = 0; c.half_floats = 0;
  c.cu = cu;
  decode_combine_kernel<<<(unsigned)(B * Hkv), 128, 0, s>>>(c);   // one CTA per (batch, KV head)
  CUDA_TRY(cudaGetLastError());
  return ok();
}

// Scratch for diffattn_decode_v2_noalloc: split-KV partial records of the
// decode, for callers that cannot allocate device memory.  One copy per
// device, reserved when the module is first loaded on it and kept until exit.  Host code
// must not pass `g_noalloc_scratch` itself to a kernel (on the host it names a
// stand-in, not device memory): it uses the address looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DIFFATTN_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[kMaxDevices] = {};

// Once per device, with that device current: the device address of the scratch.
int noalloc_scratch(void** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(DIFFATTN_ERR_CUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(DIFFATTN_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DIFFATTN_OK;
}

}  // namespace

// ============================================================================
extern "C" {

const char* diffattn_version(void) { return "diffattn 0.1 sm_100a"; }

double diffattn_lambda_init(int layer) {
  if (layer < 1) return NAN;
  return 0.8 - 0.6 * std::exp(-0.3 * (double)(layer - 1));
}

const char* diffattn_last_error(void) { return t_last_error.c_str(); }

void diffattn_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns.store(ns); }

int diffattn_last_status(void* stream) {
  DeviceInfo* dev = nullptr;
  if (int e = device_setup(&dev)) return e;
  CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  unsigned v = 0;
  CUDA_TRY(cudaMemcpy(&v, dev->status, sizeof(v), cudaMemcpyDeviceToHost));
  const unsigned zero = 0;
  CUDA_TRY(cudaMemcpy(dev->status, &zero, sizeof(zero), cudaMemcpyHostToDevice));
  if (v & STATUS_TIMEOUT) return fail(DIFFATTN_ERR_TIMEOUT, "a bounded device wait expired");
  return ok();
}

int diffattn_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2, int heads, int dim,
                    double lambda_init, float* lambda_out, void* stream) {
  if (!lq1 || !lk1 || !lq2 || !lk2 || !lambda_out) return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (heads < 1 || dim < 1) return fail(DIFFATTN_ERR_INVALID_ARG, "heads and dim must be >= 1");
  lambda_kernel<<<(heads + LAM_WARPS - 1) / LAM_WARPS, 32 * LAM_WARPS, 0, static_cast<cudaStream_t>(stream)>>>(
      lq1, lk1, lq2, lk2, heads, dim, lambda_init, lambda_out);
  CUDA_TRY(cudaGetLastError());
  return ok();
}

int diffattn_fwd_v1(const void* q1, const void* k1, const void* q2, const void* k2, const void* v,
                    const float* lambda, void* out, diffattn_dtype dtype, int B, int H, int Hkv, int Lq, int Lk,
                    int d, int dv, int causal, int rmsnorm, float eps, void* stream) {
  if (B < 0 || H < 1 || Hkv < 1 || Lq < 0 || Lk < 0 || d < 1 || dv < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d H=%d Hkv=%d Lq=%d Lk=%d d=%d dv=%d)", B, H, Hkv, Lq,
                Lk, d, dv);
  if (H % Hkv) return fail(DIFFATTN_ERR_INVALID_ARG, "H=%d is not a multiple of Hkv=%d", H, Hkv);
  if (rmsnorm && !(eps >= 0.f)) return fail(DIFFATTN_ERR_INVALID_ARG, "eps must be >= 0");
  if (B == 0 || Lq == 0) return ok();  // nothing to compute; pointers may be null
  if (!q1 || !q2 || !lambda || !out || (Lk > 0 && (!k1 || !k2 || !v)))
    return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (Lk == 0) k1 = k2 = v = q1;  // never read: no key is visible
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DIFFATTN_F32) {
    if (d > SIMT_MAXD || dv > SIMT_MAXCOL * SIMT_THREADS)
      return fail(DIFFATTN_ERR_UNSUPPORTED, "f32 path supports d <= %d, dv <= %d", SIMT_MAXD,
                  SIMT_MAXCOL * SIMT_THREADS);
    SimtArgs a{static_cast<const float*>(q1), static_cast<const float*>(q2), static_cast<const float*>(k1),
               static_cast<const float*>(k2), static_cast<const float*>(v), lambda, static_cast<float*>(out),
               B, H, H, Hkv, Lq, Lk, d, dv, 0, causal ? 1 : 0, rmsnorm ? 1 : 0, eps,
               (float)(1.0 / std::sqrt((double)d))};
    return launch_simt(a, s);
  }
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (!(d == 64 || d == 128) || dv != 128)
    return fail(DIFFATTN_ERR_UNSUPPORTED, "bf16 V1 path needs d in {64,128} and dv == 128 (got d=%d dv=%d)", d, dv);
  if (int e = check_bf16_ptrs({q1, k1, q2, k2, v, out})) return e;
  return launch_prefill(q1, q2, k1, k2, v, lambda, out, B, H, H, Hkv, Lq, Lk, d, true, causal, rmsnorm, eps, s);
}

int diffattn_fwd_v2(const void* q, const void* k, const void* v, const float* lambda, void* out,
                    diffattn_dtype dtype, int B, int Hq, int Hkv, int Lq, int Lk, int D, int causal,
                    void* stream) {
  if (B < 0 || Hq < 2 || Hkv < 1 || Lq < 0 || Lk < 0 || D < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d Hq=%d Hkv=%d Lq=%d Lk=%d D=%d)", B, Hq, Hkv, Lq, Lk, D);
  if (Hq % 2 || Hq % Hkv || (Hq / Hkv) % 2)
    return fail(DIFFATTN_ERR_INVALID_ARG, "need Hq even and Hq/Hkv even (Hq=%d Hkv=%d)", Hq, Hkv);
  if (B == 0 || Lq == 0) return ok();  // nothing to compute; pointers may be null
  if (!q || !lambda || !out || (Lk > 0 && (!k || !v))) return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (Lk == 0) k = v = q;  // never read: no key is visible
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DIFFATTN_F32) {
    if (D > SIMT_MAXD) return fail(DIFFATTN_ERR_UNSUPPORTED, "f32 path supports D <= %d", SIMT_MAXD);
    SimtArgs a{static_cast<const float*>(q), static_cast<const float*>(q), static_cast<const float*>(k),
               static_cast<const float*>(k), static_cast<const float*>(v), lambda, static_cast<float*>(out),
               B, Hq / 2, Hq, Hkv, Lq, Lk, D, D, 1, causal ? 1 : 0, 0, 0.f, (float)(1.0 / std::sqrt((double)D))};
    return launch_simt(a, s);
  }
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (D != 128) return fail(DIFFATTN_ERR_UNSUPPORTED, "bf16 V2 path needs D == 128 (got %d)", D);
  if (int e = check_bf16_ptrs({q, k, v, out})) return e;
  return launch_prefill(q, q, k, k, v, lambda, out, B, Hq / 2, Hq, Hkv, Lq, Lk, 128, false, causal, 0, 0.f, s);
}

size_t diffattn_decode_workspace_size(int B, int Hkv, int T, int dv) {
  (void)dv;
  if (B < 0 || Hkv < 1 || T < 0) return 0;
  DeviceInfo* dev = nullptr;
  if (device_setup(&dev)) return 0;
  return plan_decode(dev->sms, B, Hkv, T).bytes_per_pass * 2;  // room for the two-pass V1 comparison
}

size_t diffattn_decode_v2_workspace_size(int B, int Hq, int T, int D) {
  if (B < 0 || Hq < 2 || Hq % 2 || T < 0 || D < 1) return 0;
  size_t best = 0;
  for (int Hkv = 1; Hkv <= Hq / 2; ++Hkv)
    if (Hq % Hkv == 0 && (Hq / Hkv) % 2 == 0 && Hq / Hkv <= 8) {
      const size_t n = diffattn_decode_workspace_size(B, Hkv, T, D);
      if (n > best) best = n;
    }
  return best;
}

int diffattn_decode_v2(const void* q, const void* kc, const void* vc, const float* lambda, void* out,
                       diffattn_dtype dtype, int B, int Hq, int Hkv, int T, int D, void* ws, size_t ws_bytes,
                       void* stream) {
  if (B < 0 || Hq < 2 || Hkv < 1 || T < 0 || D < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d Hq=%d Hkv=%d T=%d D=%d)", B, Hq, Hkv, T, D);
  if (Hq % 2 || Hq % Hkv || (Hq / Hkv) % 2)
    return fail(DIFFATTN_ERR_INVALID_ARG, "need Hq even and Hq/Hkv even (Hq=%d Hkv=%d)", Hq, Hkv);
  if (B == 0) return ok();
  if (!q || !lambda || !out || (T > 0 && (!kc || !vc))) return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (T == 0) kc = vc = q;  // never read: the cache is empty
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DIFFATTN_F32)
    return diffattn_fwd_v2(q, kc, vc, lambda, out, dtype, B, Hq, Hkv, 1, T, D, 1, stream);
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (D != 128 || Hq / Hkv > 8)
    return fail(DIFFATTN_ERR_UNSUPPORTED, "bf16 decode needs D == 128 and Hq/Hkv <= 8 (D=%d Hq=%d Hkv=%d)", D, Hq,
                Hkv);
  if (int e = check_bf16_ptrs({q, kc, vc, out})) return e;
  return launch_decode(q, nullptr, kc, nullptr, vc, lambda, out, B, Hq, Hkv, T, false, 1, ws, ws_bytes, s);
}

int diffattn_fwd_v2_train(const void* q, const void* k, const void* v, const float* lambda, void* out, float* lse,
                          void* o_maps, diffattn_dtype dtype, int B, int Hq, int Hkv, int Lq, int Lk, int D,
                          int causal, void* stream) {
  if (B < 0 || Hq < 2 || Hkv < 1 || Lq < 0 || Lk < 0 || D < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d Hq=%d Hkv=%d Lq=%d Lk=%d D=%d)", B, Hq, Hkv, Lq, Lk, D);
  if (Hq % 2 || Hq % Hkv || (Hq / Hkv) % 2)
    return fail(DIFFATTN_ERR_INVALID_ARG, "need Hq even and Hq/Hkv even (Hq=%d Hkv=%d)", Hq, Hkv);
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_UNSUPPORTED, "the training forward takes bf16 only");
  if (D != 128) return fail(DIFFATTN_ERR_UNSUPPORTED, "bf16 V2 path needs D == 128 (got %d)", D);
  if (B == 0 || Lq == 0) return ok();
  if (!q || !lambda || !out || !lse || !o_maps || (Lk > 0 && (!k || !v)))
    return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (Lk == 0) k = v = q;
  if (int e = check_bf16_ptrs({q, k, v, out, o_maps})) return e;
  return launch_prefill(q, q, k, k, v, lambda, out, B, Hq / 2, Hq, Hkv, Lq, Lk, 128, false, causal, 0, 0.f,
                        static_cast<cudaStream_t>(stream), lse, o_maps);
}

size_t diffattn_bwd_v2_workspace_size(int B, int Hq, int Lq) {
  if (B < 0 || Hq < 2 || Hq % 2 || Lq < 0) return 0;
  return bwd_ws_bytes(B, Hq, Lq);
}

int diffattn_bwd_v2(const void* q, const void* k, const void* v, const float* lambda, const void* dout,
                    const float* lse, const void* o_maps, void* dq, void* dk, void* dv, float* dlambda,
                    diffattn_dtype dtype, int B, int Hq, int Hkv, int Lq, int Lk, int D, int causal, void* ws,
                    size_t ws_bytes, void* stream) {
  if (B < 0 || Hq < 2 || Hkv < 1 || Lq < 0 || Lk < 0 || D < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d Hq=%d Hkv=%d Lq=%d Lk=%d D=%d)", B, Hq, Hkv, Lq, Lk, D);
  if (Hq % 2 || Hq % Hkv || (Hq / Hkv) % 2)
    return fail(DIFFATTN_ERR_INVALID_ARG, "need Hq even and Hq/Hkv even (Hq=%d Hkv=%d)", Hq, Hkv);
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_UNSUPPORTED, "the backward takes bf16 only");
  if (D != 128) return fail(DIFFATTN_ERR_UNSUPPORTED, "bf16 V2 backward needs D == 128 (got %d)", D);
  if (!lambda || !dlambda) return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (B == 0) {   // nothing to differentiate: dlambda is an empty sum
    CUDA_TRY(cudaMemsetAsync(dlambda, 0, sizeof(float) * (size_t)(Hq / 2), static_cast<cudaStream_t>(stream)));
    return ok();
  }
  if ((Lq > 0 && (!q || !dout || !lse || !o_maps || !dq)) || (Lk > 0 && (!k || !v || !dk || !dv)))
    return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  for (const void* p : std::initializer_list<const void*>{q, k, v, dout, o_maps, dq, dk, dv})
    if (p && !aligned16(p)) return fail(DIFFATTN_ERR_MISALIGNED, "bf16 tensor pointer %p is not 16-byte aligned", p);
  return launch_backward(q, nullptr, k, nullptr, v, lambda, dout, lse, o_maps, dq, nullptr, dk, nullptr, dv, dlambda,
                         B, Hq, Hkv, Lq, Lk, causal, ws, ws_bytes, static_cast<cudaStream_t>(stream), false);
}

int diffattn_fwd_v1_train(const void* q1, const void* k1, const void* q2, const void* k2, const void* v,
                          const float* lambda, void* out, float* lse, void* o_maps, float* rstd, float* o2_coef,
                          diffattn_dtype dtype, int B, int H, int Hkv, int Lq, int Lk, int d, int dv, int causal,
                          int rmsnorm, float eps, void* stream) {
  if (B < 0 || H < 1 || Hkv < 1 || Lq < 0 || Lk < 0 || d < 1 || dv < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d H=%d Hkv=%d Lq=%d Lk=%d d=%d dv=%d)", B, H, Hkv, Lq,
                Lk, d, dv);
  if (H % Hkv) return fail(DIFFATTN_ERR_INVALID_ARG, "H=%d is not a multiple of Hkv=%d", H, Hkv);
  if (rmsnorm && !(eps >= 0.f)) return fail(DIFFATTN_ERR_INVALID_ARG, "eps must be >= 0");
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_UNSUPPORTED, "the training forward takes bf16 only");
  if (d != 64 || dv != 128)
    return fail(DIFFATTN_ERR_UNSUPPORTED, "V1 training path needs d == 64 and dv == 128 (got d=%d dv=%d)", d, dv);
  if (B == 0 || Lq == 0) return ok();
  if (!q1 || !q2 || !lambda || !out || !lse || !o_maps || (rmsnorm && (!rstd || !o2_coef)) ||
      (Lk > 0 && (!k1 || !k2 || !v)))
    return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (Lk == 0) k1 = k2 = v = q1;
  if (int e = check_bf16_ptrs({q1, k1, q2, k2, v, out, o_maps})) return e;
  return launch_prefill(q1, q2, k1, k2, v, lambda, out, B, H, H, Hkv, Lq, Lk, 64, true, causal, rmsnorm, eps,
                        static_cast<cudaStream_t>(stream), lse, o_maps, rstd, nullptr, o2_coef);
}

size_t diffattn_bwd_v1_workspace_size(int B, int H, int Hkv, int Lq, int Lk, int rmsnorm) {
  if (B < 0 || H < 1 || Hkv < 1 || Lq < 0 || Lk < 0 || H % Hkv) return 0;
  return v1_bwd_layout(B, H, Hkv, Lq, Lk, rmsnorm ? 1 : 0).total;
}

int diffattn_bwd_v1(const void* q1, const void* k1, const void* q2, const void* k2, const void* v,
                    const float* lambda, const void* dout, const void* out, const float* lse, const void* o_maps,
                    const float* rstd, const float* o2_coef, void* dq1, void* dk1, void* dq2, void* dk2, void* dv, float* dlambda,
                    diffattn_dtype dtype, int B, int H, int Hkv, int Lq, int Lk, int d, int dv_width, int causal,
                    int rmsnorm, void* ws, size_t ws_bytes, void* stream) {
  if (B < 0 || H < 1 || Hkv < 1 || Lq < 0 || Lk < 0 || d < 1 || dv_width < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d H=%d Hkv=%d Lq=%d Lk=%d d=%d dv=%d)", B, H, Hkv, Lq,
                Lk, d, dv_width);
  if (H % Hkv) return fail(DIFFATTN_ERR_INVALID_ARG, "H=%d is not a multiple of Hkv=%d", H, Hkv);
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_UNSUPPORTED, "the backward takes bf16 only");
  if (d != 64 || dv_width != 128)
    return fail(DIFFATTN_ERR_UNSUPPORTED, "V1 backward needs d == 64 and dv == 128 (got d=%d dv=%d)", d, dv_width);
  if (!lambda || !dlambda) return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  const int rms = rmsnorm ? 1 : 0;
  if (B == 0) {   // nothing to differentiate: dlambda is an empty sum
    CUDA_TRY(cudaMemsetAsync(dlambda, 0, sizeof(float) * (size_t)H, static_cast<cudaStream_t>(stream)));
    return ok();
  }
  if ((Lq > 0 && (!q1 || !q2 || !dout || !lse || !o_maps || !dq1 || !dq2 || (rms && (!out || !rstd || !o2_coef)))) ||
      (Lk > 0 && (!k1 || !k2 || !v || !dk1 || !dk2 || !dv)))
    return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  for (const void* p : std::initializer_list<const void*>{q1, k1, q2, k2, v, dout, out, o_maps, dq1, dk1, dq2, dk2,
                                                          dv})
    if (p && !aligned16(p)) return fail(DIFFATTN_ERR_MISALIGNED, "bf16 tensor pointer %p is not 16-byte aligned", p);
  return launch_backward_v1(q1, k1, q2, k2, v, lambda, dout, out, lse, o_maps, rstd, o2_coef, dq1, dk1, dq2, dk2, dv,
                            dlambda, B, H, Hkv, Lq, Lk, causal, rms, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t diffattn_fwd_lowrank_workspace_size(int B, int H, int Lq, int Lk, int r, int causal) {
  if (B < 0 || H < 2 || H % 2 || Lq < 0 || Lk < 0 || r < 1 || r > LR_RMAX) return 0;
  return lowrank_layout(B, H, Lq, Lk, r, causal ? 1 : 0).total;
}

int diffattn_fwd_lowrank(const void* q, const void* k, const void* v, const float* F, const float* G,
                         const float* lambda, void* out, diffattn_dtype dtype, int B, int H, int Hkv, int Lq, int Lk,
                         int D, int r, int causal, void* ws, size_t ws_bytes, void* stream) {
  if (B < 0 || H < 2 || Hkv < 1 || Lq < 0 || Lk < 0 || D < 1 || r < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d H=%d Hkv=%d Lq=%d Lk=%d D=%d r=%d)", B, H, Hkv, Lq, Lk, D,
                r);
  if (H % Hkv || (H / Hkv) % 2)
    return fail(DIFFATTN_ERR_INVALID_ARG, "need H/Hkv even: heads run in pairs over a KV head (H=%d Hkv=%d)", H, Hkv);
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_UNSUPPORTED, "the low-rank forward takes bf16 only");
  if (D != 128) return fail(DIFFATTN_ERR_UNSUPPORTED, "the low-rank forward needs D == 128 (got %d)", D);
  if (r > LR_RMAX) return fail(DIFFATTN_ERR_UNSUPPORTED, "rank r=%d above %d", r, LR_RMAX);
  if ((long long)B * H > 65535) return fail(DIFFATTN_ERR_UNSUPPORTED, "B*H=%lld above 65535", (long long)B * H);
  if (B == 0 || Lq == 0) return ok();
  if (!q || !F || !lambda || !out || (Lk > 0 && (!k || !v || !G))) return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (Lk == 0) k = v = q;   // never read: no key is visible
  if (int e = check_bf16_ptrs({q, k, v, out})) return e;
  const LowrankLayout L = lowrank_layout(B, H, Lq, Lk, r, causal ? 1 : 0);
  if (ws == nullptr || ws_bytes < L.total)
    return fail(DIFFATTN_ERR_WORKSPACE, "low-rank workspace %zu B < required %zu B", ws_bytes, L.total);
  if (!aligned16(ws)) return fail(DIFFATTN_ERR_MISALIGNED, "workspace not 16-byte aligned");
  DeviceInfo* dev = nullptr;
  if (int e = device_setup(&dev)) return e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  // A1 V for every head in f32: the single-map prefill runs heads (2j, 2j+1)
  // of one KV group as the two maps of a CTA and writes each one's O / l,
  // [B, H/2, 2, Lq, 128] = [B, H, Lq, 128]; lambda only sets each head's
  // residual choice there.
  if (int e = launch_prefill(q, q, k, k, v, lambda, nullptr, B, H / 2, H, Hkv, Lq, Lk, 128, false, causal, 0, 0.f,
                             s, nullptr, nullptr, nullptr, reinterpret_cast<float*>(w + L.a1v)))
    return e;
  LowrankArgs a{};
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.F = F; a.G = G; a.lambda = lambda;
  a.a1v = reinterpret_cast<const float*>(w + L.a1v);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.tot = reinterpret_cast<float*>(w + L.tot);
  a.ztot = reinterpret_cast<float*>(w + L.ztot);
  a.B = B; a.H = H; a.Hkv = Hkv; a.Lq = Lq; a.Lk = Lk; a.r = r; a.causal = causal ? 1 : 0;
  a.n_lead = L.n_lead;
  a.nc = L.nc;
  const unsigned BH = (unsigned)(B * H);
  if (L.nc > 0 && Lk > 0) {
    lr_totals_kernel<<<dim3((unsigned)L.nc, BH), LR_DV, 0, s>>>(a);
    CUDA_TRY(cudaGetLastError());
  } else if (L.nc > 0) {   // no key: every chunk sum is zero
    CUDA_TRY(cudaMemsetAsync(a.tot, 0, sizeof(float) * (size_t)BH * (L.nc + 1) * r * LR_DV, s));
    CUDA_TRY(cudaMemsetAsync(a.ztot, 0, sizeof(float) * (size_t)BH * (L.nc + 1) * r, s));
  }
  lr_prefix_kernel<<<dim3((unsigned)r, BH), LR_DV, 0, s>>>(a);
  CUDA_TRY(cudaGetLastError());
  lr_emit_kernel<<<dim3((unsigned)((Lq + LR_C - 1) / LR_C), BH), LR_DV, 0, s>>>(a);
  CUDA_TRY(cudaGetLastError());
  return ok();
}

int diffattn_lambda_backward(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                             const float* dlambda, int heads, int dim, float* dlq1, float* dlk1, float* dlq2,
                             float* dlk2, void* stream) {
  if (!lq1 || !lk1 || !lq2 || !lk2 || !dlambda || !dlq1 || !dlk1 || !dlq2 || !dlk2)
    return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (heads < 1 || dim < 1) return fail(DIFFATTN_ERR_INVALID_ARG, "heads and dim must be >= 1");
  lambda_backward_kernel<<<(heads + LAM_WARPS - 1) / LAM_WARPS, 32 * LAM_WARPS, 0,
                           static_cast<cudaStream_t>(stream)>>>(
      lq1, lk1, lq2, lk2, dlambda, heads, dim, dlq1, dlk1, dlq2, dlk2);
  CUDA_TRY(cudaGetLastError());
  return ok();
}

size_t diffattn_decode_paged_workspace_size(int B, int Hkv) {
  if (B < 1 || B > DEC_MAXB || Hkv < 1) return 0;
  DeviceInfo* dev = nullptr;
  if (device_setup(&dev)) return 0;
  return paged_ws_bytes(dev, B, Hkv);
}

int diffattn_decode_v2_paged(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                             const int* seq_lens, const float* lambda, void* out, diffattn_dtype dtype, int B,
                             int Hq, int Hkv, int num_pages, int page_size, int max_pages, void* ws,
                             size_t ws_bytes, void* stream) {
  if (B < 1 || B > DEC_MAXB || Hq < 2 || Hkv < 1 || num_pages < 1 || max_pages < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d Hq=%d Hkv=%d num_pages=%d max_pages=%d; 1 <= B <= %d)",
                B, Hq, Hkv, num_pages, max_pages, DEC_MAXB);
  if (Hq % 2 || Hq % Hkv || (Hq / Hkv) % 2)
    return fail(DIFFATTN_ERR_INVALID_ARG, "need Hq even and Hq/Hkv even (Hq=%d Hkv=%d)", Hq, Hkv);
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128 && page_size != 256)
    return fail(DIFFATTN_ERR_UNSUPPORTED, "page_size %d: must be 16, 32, 64, 128 or 256", page_size);
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_UNSUPPORTED, "the paged decode takes bf16 only");
  if (Hq / Hkv > 8) return fail(DIFFATTN_ERR_UNSUPPORTED, "paged decode needs Hq/Hkv <= 8 (Hq=%d Hkv=%d)", Hq, Hkv);
  const long long max_blocks = ((long long)max_pages * page_size + DEC_KB - 1) / DEC_KB;
  if ((long long)B * Hkv * max_blocks >= (1LL << 31))
    return fail(DIFFATTN_ERR_UNSUPPORTED, "B * Hkv * max_pages * page_size / 64 must stay below 2^31");
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !lambda || !out)
    return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (int e = check_bf16_ptrs({q, k_pages, v_pages, out})) return e;
  if ((reinterpret_cast<uintptr_t>(block_table) | reinterpret_cast<uintptr_t>(seq_lens)) & 3u)
    return fail(DIFFATTN_ERR_MISALIGNED, "block_table / seq_lens not 4-byte aligned");
  return launch_decode_paged(q, k_pages, v_pages, block_table, seq_lens, lambda, out, B, Hq, Hkv, num_pages,
                             page_size, max_pages, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int diffattn_decode_v2_noalloc(const void* q, const void* kc, const void* vc, const float* lambda, void* out,
                               diffattn_dtype dtype, int B, int Hq, int Hkv, int T, int D, void* stream) {
  if (B < 0 || Hq < 2 || Hkv < 1 || T < 0 || D < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d Hq=%d Hkv=%d T=%d D=%d)", B, Hq, Hkv, T, D);
  if (dtype == DIFFATTN_BF16 && B > 0) {
    DeviceInfo* dev = nullptr;
    if (int e = device_setup(&dev)) return e;
    const size_t need = plan_decode(dev->sms, B, Hkv, T).bytes_per_pass;
    if (need > DIFFATTN_NOALLOC_SCRATCH_BYTES)
      return fail(DIFFATTN_ERR_UNSUPPORTED,
                  "decode needs %zu B of partial records, above the %u B scratch of the no-allocation entry point",
                  need, (unsigned)DIFFATTN_NOALLOC_SCRATCH_BYTES);
  }
  void* scratch = nullptr;
  if (int e = noalloc_scratch(&scratch)) return e;
  return diffattn_decode_v2(q, kc, vc, lambda, out, dtype, B, Hq, Hkv, T, D, scratch,
                            DIFFATTN_NOALLOC_SCRATCH_BYTES, stream);
}

int diffattn_decode_v1(const void* q1, const void* k1, const void* q2, const void* k2, const void* v,
                       const float* lambda, void* out, diffattn_dtype dtype, int B, int H, int Hkv, int T, int d,
                       int dv, int fused, void* ws, size_t ws_bytes, void* stream) {
  if (B < 0 || H < 1 || Hkv < 1 || T < 0 || d < 1 || dv < 1)
    return fail(DIFFATTN_ERR_INVALID_ARG, "bad sizes (B=%d H=%d Hkv=%d T=%d d=%d dv=%d)", B, H, Hkv, T, d, dv);
  if (H % Hkv) return fail(DIFFATTN_ERR_INVALID_ARG, "H=%d is not a multiple of Hkv=%d", H, Hkv);
  if (B == 0) return ok();
  if (!q1 || !q2 || !lambda || !out || (T > 0 && (!k1 || !k2 || !v)))
    return fail(DIFFATTN_ERR_INVALID_ARG, "null pointer");
  if (T == 0) k1 = k2 = v = q1;  // never read: the cache is empty
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DIFFATTN_F32)
    return diffattn_fwd_v1(q1, k1, q2, k2, v, lambda, out, dtype, B, H, Hkv, 1, T, d, dv, 1, 0, 0.f, stream);
  if (dtype != DIFFATTN_BF16) return fail(DIFFATTN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (d != 64 || dv != 128 || H / Hkv > 4)
    return fail(DIFFATTN_ERR_UNSUPPORTED, "bf16 V1 decode needs d == 64, dv == 128, H/Hkv <= 4");
  if (int e = check_bf16_ptrs({q1, k1, q2, k2, v, out})) return e;
  return launch_decode(q1, q2, k1, k2, v, lambda, out, B, H, Hkv, T, true, fused, ws, ws_bytes, s);
}

}  // extern "C"
