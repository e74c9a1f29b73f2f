/*
 * diffattn.h -- C ABI of libdiffattn.so, B200 (sm_100a) differential
 * attention: prefill and decode forward, the training forward and backward,
 * and the low-rank substitute for the second map.
 *
 * The operation (sources cited by page title and section):
 *
 *   A1 = softmax(Q1 K1^T / sqrt(d)),  A2 = softmax(Q2 K2^T / sqrt(d))
 *   O  = (A1 - lambda * A2) V
 *       "差分注意力" tutorial (aiknowledge.cn), section 差分思路 and
 *       二、从零实现 Step 2; the paper note "Understanding Differential
 *       Transformer Unchains Pretrained Self-Attentions", section 关键设计.
 *   lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init
 *       "差分注意力" tutorial, section 差分思路 and Step 4 (λ 参数化).
 *   lambda_init = 0.8 - 0.6 exp(-0.3 (layer - 1))
 *       "Differential Transformer：用“差分降噪”重塑LLM注意力机制" (mcipr.com),
 *       section 3 工程实践.
 *   V1 layout (half-width Q/K per head, one V, optional per-head RMSNorm) and
 *   V2 layout (Q heads doubled over shared KV heads, no norm)
 *       "差分注意力" tutorial, section V1 到 V2 的 diff.
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, last dimension contiguous, no padding.
 *     The shapes are given per argument.  "bf16" is IEEE bfloat16, "f32" IEEE
 *     binary32.  Output precision equals input precision; all arithmetic is
 *     fp32 (lambda: fp64) whatever the input type.
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library
 *     keeps no reference after the call and allocates no device memory.  Work
 *     is queued asynchronously on `stream` (a cudaStream_t; NULL = legacy
 *     default stream); the call returns before the GPU finishes.
 *   - Every bf16 tensor must start on a 16-byte boundary and its row
 *     (last-dimension) length in bytes must be a multiple of 16 (tensor-map
 *     copies require it); violations return DIFFATTN_ERR_MISALIGNED before
 *     any launch.
 *   - Causal masking is bottom-right aligned: query row i sees key j iff
 *     j <= i + (Lk - Lq).  A row that sees no key outputs zeros.
 *   - Errors: every argument error is reported before anything is launched,
 *     as a negative status; diffattn_last_error() then describes it.  No C++
 *     exception crosses this boundary.  A device-side bounded wait that runs
 *     out does not fault the GPU: the kernel records DIFFATTN_ERR_TIMEOUT in a
 *     device status word, releases what it holds and returns; read it with
 *     diffattn_last_status().
 */
#ifndef DIFFATTN_H_
#define DIFFATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DIFFATTN_API __attribute__((visibility("default")))
#else
#define DIFFATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { DIFFATTN_F32 = 0, DIFFATTN_BF16 = 1 } diffattn_dtype;

enum {
  DIFFATTN_OK = 0,
  DIFFATTN_ERR_INVALID_ARG = -1, /* null pointer, negative size, head counts that do not divide */
  DIFFATTN_ERR_UNSUPPORTED = -2, /* valid but not implemented (e.g. bf16 with an unsupported width) */
  DIFFATTN_ERR_MISALIGNED = -3,  /* pointer or row length not 16-byte aligned (bf16 paths) */
  DIFFATTN_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed; message has the CUDA error */
  DIFFATTN_ERR_TIMEOUT = -5,     /* a bounded device wait expired (read via diffattn_last_status) */
  DIFFATTN_ERR_WORKSPACE = -6    /* workspace pointer null or smaller than required */
};

/* Library version string, e.g. "diffattn 0.1 sm_100a". */
DIFFATTN_API const char* diffattn_version(void);

/* lambda_init for a 1-based layer index: 0.8 - 0.6*exp(-0.3*(layer-1)).
 * Returns NaN for layer < 1.  Host-only, no GPU needed.
 * Source: "Differential Transformer" (mcipr.com), section 3 工程实践. */
DIFFATTN_API double diffattn_lambda_init(int layer);

/* lambda[h] = exp(lq1[h].lk1[h]) - exp(lq2[h].lk2[h]) + lambda_init, h < heads.
 *   lq1, lk1, lq2, lk2 : device f32 [heads, dim]
 *   lambda_out         : device f32 [heads]
 * Dot products are sequential fp64 sums, exp is fp64, the result is rounded
 * once to f32.  heads, dim >= 1.
 * Source: "差分注意力" tutorial, Step 4 (λ 参数化). */
DIFFATTN_API int diffattn_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                    int heads, int dim, double lambda_init, float* lambda_out, void* stream);

/* V1-layout forward ("差分注意力" tutorial, section V1 到 V2 的 diff).
 *   q1, q2 : [B, H,   Lq, d]      k1, k2 : [B, Hkv, Lk, d]
 *   v      : [B, Hkv, Lk, dv]     lambda : device f32 [H]
 *   out    : [B, H,   Lq, dv]     (same dtype as the inputs)
 * Head h reads KV head h / (H / Hkv); H % Hkv == 0 required.
 * rmsnorm != 0 applies y = x / sqrt(mean(x^2) + eps) over dv per row (unit
 * weight) to the difference output.
 * bf16: tensor-core path, requires d in {64, 128} and dv == 128.
 * f32 : exact-softmax SIMT path, any d <= 256, dv <= 4096.
 * Lq == 0 or B == 0 is a no-op; Lk == 0 writes zeros. */
DIFFATTN_API int diffattn_fwd_v1(const void* q1, const void* k1, const void* q2, const void* k2, const void* v,
                    const float* lambda, void* out, diffattn_dtype dtype,
                    int B, int H, int Hkv, int Lq, int Lk, int d, int dv,
                    int causal, int rmsnorm, float eps, void* stream);

/* V2-layout forward (same section).
 *   q      : [B, Hq,  Lq, D]      k, v : [B, Hkv, Lk, D]
 *   lambda : device f32 [Hq/2]    out  : [B, Hq/2, Lq, D]
 * Diff pair h = Q heads (2h, 2h+1) = (map 1, map 2); both read KV head
 * 2h / (Hq / Hkv).  Requires Hq even, Hq % Hkv == 0 and (Hq/Hkv) even so that
 * a pair never straddles two KV groups.
 * bf16: tensor-core path, D == 128.  f32: SIMT path, D <= 256. */
DIFFATTN_API int diffattn_fwd_v2(const void* q, const void* k, const void* v, const float* lambda, void* out,
                    diffattn_dtype dtype, int B, int Hq, int Hkv, int Lq, int Lk, int D,
                    int causal, void* stream);

/* Bytes of device workspace diffattn_decode_v2 / diffattn_decode_v1 need for
 * a batch of B sequences, Hkv KV heads, cache length T and value width dv on
 * the current device.  The caller allocates it (any alignment >= 16 B). */
DIFFATTN_API size_t diffattn_decode_workspace_size(int B, int Hkv, int T, int dv);

/* The same size in terms of the V2 decode's query shape, for a caller that
 * sizes the workspace before it knows the KV-head count: bytes that suffice
 * for diffattn_decode_v2 with B sequences, Hq Q heads, cache length T, head
 * width D and ANY valid Hkv (Hq % Hkv == 0, (Hq/Hkv) even, Hq/Hkv <= 8), i.e.
 * the largest diffattn_decode_workspace_size(B, Hkv, T, D) over those Hkv.
 * 0 for invalid sizes (Hq odd or < 2, B < 0, T < 0, D < 1). */
DIFFATTN_API size_t diffattn_decode_v2_workspace_size(int B, int Hq, int T, int D);

/* Single-token V2 decode over a KV cache (tutorial section V1 到 V2 的 diff:
 * doubled Q heads, K/V read once per KV group for both maps).
 *   q      : [B, Hq, D]           kc, vc : [B, Hkv, T, D]  (bf16)
 *   lambda : device f32 [Hq/2]    out    : [B, Hq/2, D]
 *   ws     : device workspace of ws_bytes >= diffattn_decode_workspace_size(B, Hkv, T, D)
 * The new token sees every cached key.  bf16: D == 128 and Hq/Hkv in
 * {2,4,6,8}.  f32: routed to the SIMT path (no workspace used).  Two launches
 * (split-KV partials, then a combine) on `stream`. */
DIFFATTN_API int diffattn_decode_v2(const void* q, const void* kc, const void* vc, const float* lambda, void* out,
                       diffattn_dtype dtype, int B, int Hq, int Hkv, int T, int D,
                       void* ws, size_t ws_bytes, void* stream);

/* Single-token V1-layout decode: q1, q2 [B, H, d]; k1, k2 [B, Hkv, T, d];
 * v [B, Hkv, T, dv]; lambda [H]; out [B, H, dv].  bf16: d == 64, dv == 128,
 * H/Hkv <= 4.  K1, K2 and V are each read once for both maps (fused).
 * fused == 0 instead runs the two maps as two passes that each read V (the
 * "V cache loaded twice" behaviour the tutorial attributes to V1), for
 * comparison only. */
DIFFATTN_API int diffattn_decode_v1(const void* q1, const void* k1, const void* q2, const void* k2,
                       const void* v, const float* lambda, void* out, diffattn_dtype dtype,
                       int B, int H, int Hkv, int T, int d, int dv, int fused,
                       void* ws, size_t ws_bytes, void* stream);

/* Message of the last error returned on this host thread ("" if none). */
DIFFATTN_API const char* diffattn_last_error(void);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device: DIFFATTN_OK, DIFFATTN_ERR_TIMEOUT if a kernel's bounded
 * wait expired since the last call, or DIFFATTN_ERR_CUDA if the stream
 * reports an error. */
DIFFATTN_API int diffattn_last_status(void* stream);

/* Upper bound, in nanoseconds, of every device-side wait (mbarrier phases
 * between warps of one CTA).  Default 2e9 (2 s).  0 makes any wait that is
 * not already satisfied expire at once (used to test the timeout path).
 * Applies to launches made after the call, process-wide. */
DIFFATTN_API void diffattn_set_wait_limit_ns(unsigned long long ns);

/* Maximum scratch, in bytes, that diffattn_decode_v2_noalloc can use. */
#define DIFFATTN_NOALLOC_SCRATCH_BYTES (4u << 20)

/* Single-token V2 decode that allocates nothing and takes no workspace.
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot call cudaMalloc, e.g. code running inside a memory pool or an
 * allocator hook that must not re-enter the allocator, or a runtime that owns
 * all device memory and hands this library only its tensors.
 * Arguments, layouts and results are those of diffattn_decode_v2 without
 * `ws` / `ws_bytes`: the split-KV partial records live instead in a static
 * device array of DIFFATTN_NOALLOC_SCRATCH_BYTES (4 MiB) in the library's
 * module.  It is reserved on a device when the module is first loaded there
 * (with CUDA's lazy module loading, at the library's first use on that
 * device) and kept until the process exits.  Its address is looked up once
 * per device and cached; after cudaDeviceReset of a device the cached
 * addresses (this one and the library's status word) are stale, so the
 * library must not be called on that device again in the same process.
 *   - Sizes whose partial records need more than that (see
 *     diffattn_decode_workspace_size; about 2.5 MB for 16 sequences x 8 KV
 *     heads x 65536 tokens) return DIFFATTN_ERR_UNSUPPORTED before any launch.
 *   - The first call on a device does a one-time set-up on that device (the
 *     scratch address and kernel attributes are looked up); make that first
 *     call before any stream capture.
 *   - Every call on a device shares the one scratch array, and it keeps the
 *     last call's contents.  Nothing in it needs to start at zero: each call
 *     writes every record it later reads.  Calls that can overlap on the GPU
 *     (different streams without ordering between them) race on the scratch
 *     and produce wrong results; serialise them on one stream.
 *   - No cudaMalloc, cudaFree or any other allocating call is made. */
DIFFATTN_API int diffattn_decode_v2_noalloc(const void* q, const void* kc, const void* vc, const float* lambda,
                                            void* out, diffattn_dtype dtype, int B, int Hq, int Hkv, int T,
                                            int D, void* stream);

/* Training forward, V2 layout, bf16 (same operation and arguments as
 * diffattn_fwd_v2, D == 128), that also writes what the backward needs:
 *   lse    : f32 [B, Hq/2, 2, Lq]: per row and map, log2 of the softmax
 *            normaliser of the scores scaled by log2(e)/sqrt(D), i.e.
 *            A_m[i, j] = 2^(S_m[i, j] log2(e)/sqrt(D) - lse[.., m, i]);
 *            +inf for a row that sees no key.                    (device)
 *   o_maps : bf16 [B, Hq/2, 2, Lq, 128]: O_m = A_m V per map.    (device)
 * The λ parameterisation (tutorial, Step 4) makes λ learnable, so the layer
 * is trained; the pages print no backward. */
DIFFATTN_API int diffattn_fwd_v2_train(const void* q, const void* k, const void* v, const float* lambda, void* out,
                                       float* lse, void* o_maps, diffattn_dtype dtype, int B, int Hq, int Hkv,
                                       int Lq, int Lk, int D, int causal, void* stream);

/* Workspace, in bytes, for diffattn_bwd_v2 (B sequences, Hq Q heads, Lq rows). */
DIFFATTN_API size_t diffattn_bwd_v2_workspace_size(int B, int Hq, int Lq);

/* Backward of the V2 forward (bf16, D == 128), the chain rule of
 *   A_m = softmax(Q_m K^T / sqrt(D)),  O = (A_1 - λ A_2) V:
 *   dV = Σ (A_1 - λ A_2)^T dO,  dS_1 = A_1 (dO V^T - D_1),
 *   dS_2 = -λ A_2 (dO V^T - D_2),  D_m = rowsum(dO * O_m),
 *   dQ_m = dS_m K / sqrt(D),  dK = Σ dS_m^T Q_m / sqrt(D),
 *   dλ = -Σ dO * O_2.
 *   q, k, v, lambda : the forward's inputs                        (device)
 *   dout            : bf16 [B, Hq/2, Lq, 128]                     (device)
 *   lse, o_maps     : from diffattn_fwd_v2_train                  (device)
 *   dq              : bf16 [B, Hq, Lq, 128]; dk, dv : bf16 [B, Hkv, Lk, 128]
 *   dlambda         : f32 [Hq/2], summed over batch and rows in a fixed
 *                     order (deterministic)                      (device)
 *   ws              : diffattn_bwd_v2_workspace_size bytes, 16-byte aligned.
 * dK and dV sum over every Q head of a KV group and both maps. */
DIFFATTN_API int diffattn_bwd_v2(const void* q, const void* k, const void* v, const float* lambda, const void* dout,
                                 const float* lse, const void* o_maps, void* dq, void* dk, void* dv, float* dlambda,
                                 diffattn_dtype dtype, int B, int Hq, int Hkv, int Lq, int Lk, int D, int causal,
                                 void* ws, size_t ws_bytes, void* stream);

/* Training forward, V1 layout, bf16 (same operation and arguments as
 * diffattn_fwd_v1, with d == 64 and dv == 128), that also writes what
 * diffattn_bwd_v1 needs:
 *   lse    : f32 [B, H, 2, Lq], as for diffattn_fwd_v2_train, with the scores
 *            of map m = Q_m K_m^T scaled by log2(e)/sqrt(d)       (device)
 *   o_maps : bf16 [B, H, 2, Lq, 128]: O_m = A_m V per map; with rmsnorm != 0
 *            map 2's entry is instead O_2 - c X, its part orthogonal to the
 *            difference output X = O_1 - λ O_2, c = <O_2, X> / <X, X> per row
 *            (formed in f32)                                       (device)
 *   rstd   : f32 [B, H, Lq]: with rmsnorm != 0, the row's r =
 *            1/sqrt(mean(x^2) + eps) of the difference output x (0 for a row
 *            that sees no key); not touched, and may be NULL, without. (device)
 *   o2_coef: f32 [B, H, Lq]: with rmsnorm != 0, c eps r^2 per row (0 for a
 *            row that sees no key); not touched, and may be NULL, without.
 * The per-head RMSNorm is the tutorial's (section V1 到 V2 的 diff).  Why map
 * 2 is stored that way: dλ = -Σ dX·O_2, and the RMSNorm gradient dX is
 * orthogonal to X, to which O_2 is nearly parallel when the two maps are
 * alike; the sum is then a small remainder of large terms, and a bf16 O_2
 * would leave an error of the terms' size.  With X·dX = <y, dY> eps r^2,
 * dX·O_2 = dX·(O_2 - c X) + o2_coef <y, dY> needs only the small part.  For
 * the same reason, with rmsnorm != 0 every head keeps the bf16 residual of P
 * (the inference forward keeps it only for |1 - λ| < 0.15), so that O_2 has
 * no 2^-9 rounding along X either. */
DIFFATTN_API int diffattn_fwd_v1_train(const void* q1, const void* k1, const void* q2, const void* k2,
                                       const void* v, const float* lambda, void* out, float* lse, void* o_maps,
                                       float* rstd, float* o2_coef, diffattn_dtype dtype, int B, int H, int Hkv,
                                       int Lq, int Lk, int d, int dv, int causal, int rmsnorm, float eps,
                                       void* stream);

/* Workspace, in bytes, for diffattn_bwd_v1.  0 for invalid sizes. */
DIFFATTN_API size_t diffattn_bwd_v1_workspace_size(int B, int H, int Hkv, int Lq, int Lk, int rmsnorm);

/* Backward of the V1 forward (bf16, d == 64, dv == 128), with the RMSNorm
 * gradient dX = r (dY - y <y, dY> / dv) first when rmsnorm != 0:
 *   q1, k1, q2, k2, v, lambda : the forward's inputs               (device)
 *   dout            : bf16 [B, H, Lq, 128], the gradient of out    (device)
 *   out, lse, o_maps,
 *   rstd, o2_coef   : from diffattn_fwd_v1_train (out, rstd and o2_coef are
 *                     read only with rmsnorm != 0 and may be NULL without)
 *                                                                   (device)
 *   dq1, dq2        : bf16 [B, H, Lq, 64]; dk1, dk2 : bf16 [B, Hkv, Lk, 64];
 *   dv              : bf16 [B, Hkv, Lk, 128]; dlambda : f32 [H]    (device)
 *   ws              : diffattn_bwd_v1_workspace_size bytes, 16-byte aligned.
 * The maps are those of diffattn_bwd_v2 with Q_1 K_1^T and Q_2 K_2^T as the
 * scores (scale 1/sqrt(64)), computed by V1 instances of the same kernels:
 * the scores contract over the 64-wide Q_m, K_m read from their own tensors,
 * and dQ_m, dK_m are 64-wide products.  dK1, dK2 and dV sum over the heads of
 * a KV group.  With rmsnorm != 0 the RMSNorm pass also
 * forms the row terms D_m = dX·O_m from its f32 dX, D_2 as
 * dX·o_maps[.., 1, ..] + o2_coef <y, dY> (see diffattn_fwd_v1_train). */
DIFFATTN_API int diffattn_bwd_v1(const void* q1, const void* k1, const void* q2, const void* k2, const void* v,
                                 const float* lambda, const void* dout, const void* out, const float* lse,
                                 const void* o_maps, const float* rstd, const float* o2_coef, void* dq1, void* dk1,
                                 void* dq2, void* dk2, void* dv, float* dlambda, diffattn_dtype dtype, int B, int H,
                                 int Hkv, int Lq, int Lk, int d, int dv_width, int causal, int rmsnorm, void* ws,
                                 size_t ws_bytes,
                                 void* stream);

/* Workspace, in bytes, for diffattn_fwd_lowrank.  0 for invalid sizes. */
DIFFATTN_API size_t diffattn_fwd_lowrank_workspace_size(int B, int H, int Lq, int Lk, int r, int causal);

/* Differential attention with a fixed low-rank map N in place of A2 (paper
 * note "Understanding Differential Transformer Unchains Pretrained
 * Self-Attentions", sections 基于分析的改进建议 and 亮点与洞察; the note gives
 * the idea, the form below is this library's reading):
 *   N[i, j] = f_i.g_j / Σ_{j' visible from i} f_i.g_j'  on visible keys, 0 elsewhere
 *             (a row with zero mass is 0)
 *   out     = softmax(Q K^T / sqrt(D)) V - λ N V        per head
 *   q      : bf16 [B, H, Lq, 128]       k, v : bf16 [B, Hkv, Lk, 128]  (device)
 *   F      : f32 [H, Lq, r], G : f32 [H, Lk, r], non-negative          (device)
 *   lambda : f32 [H];  out : bf16 [B, H, Lq, 128]                      (device)
 *   ws     : diffattn_fwd_lowrank_workspace_size bytes, 16-byte aligned,
 *            owned by the caller.
 * Head h reads KV head h / (H / Hkv); H / Hkv must be even (heads are
 * computed in pairs that share a KV head).  Requires bf16, D == 128,
 * 1 <= r <= 16 and B * H <= 65535.  The causal mask is the library's
 * bottom-right one.  Negative factors are not checked; they give a result
 * that is not a map. */
DIFFATTN_API int diffattn_fwd_lowrank(const void* q, const void* k, const void* v, const float* F, const float* G,
                                      const float* lambda, void* out, diffattn_dtype dtype, int B, int H, int Hkv,
                                      int Lq, int Lk, int D, int r, int causal, void* ws, size_t ws_bytes,
                                      void* stream);

/* Gradients of λ = exp(lq1.lk1) - exp(lq2.lk2) + λ_init with respect to its
 * parameter vectors ([heads, dim] f32 each), given dlambda [heads]: fp64
 * inside, f32 out.                                                 (device) */
DIFFATTN_API int diffattn_lambda_backward(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                                          const float* dlambda, int heads, int dim, float* dlq1, float* dlk1,
                                          float* dlq2, float* dlk2, void* stream);

/* Workspace, in bytes, that diffattn_decode_v2_paged needs on the current
 * device for B sequences over Hkv KV heads (independent of the lengths and the
 * page size).  0 for invalid sizes. */
DIFFATTN_API size_t diffattn_decode_paged_workspace_size(int B, int Hkv);

/* Paged, variable-length single-token V2 decode (serving layout).  Same
 * operation as diffattn_decode_v2, each sequence against its own cache.
 * The tutorial ("差分注意力", section V1 到 V2 的 diff) names serving engines
 * such as vLLM and SGLang as the integration target but gives no layout; the
 * layout below is the common token-major page pool.
 *   q           : [B, Hq, 128] bf16                  (device)
 *   k_pages,
 *   v_pages     : [num_pages, page_size, Hkv, 128] bf16: page p holds
 *                 page_size consecutive tokens of one sequence, every KV head
 *                 of a token side by side                           (device)
 *   block_table : int32 [B, max_pages]; row b lists sequence b's page ids in
 *                 token order                                       (device)
 *   seq_lens    : int32 [B]; sequence b is its first seq_lens[b] tokens.
 *                 Values are clamped to [0, max_pages * page_size]; only the
 *                 first ceil(seq_lens[b] / page_size) entries of row b are
 *                 read, and a page id outside [0, num_pages) reads zeros.
 *                 A length of 0 gives a zero output.                (device)
 *   lambda      : f32 [Hq/2];  out : [B, Hq/2, 128] bf16            (device)
 *   ws          : device workspace of diffattn_decode_paged_workspace_size
 *                 bytes, 16-byte aligned, owned by the caller.  The call also
 *                 leaves the per-sequence block prefix there.
 * Requires bf16, Hq even, Hq % Hkv == 0, Hq/Hkv even and <= 8, page_size in
 * {16, 32, 64, 128, 256}, 1 <= B <= 2048, and B * Hkv * max_pages *
 * page_size / 64 < 2^31.  Rows of a page past a sequence's length are never
 * used, whatever they hold (they may be uninitialised). */
DIFFATTN_API int diffattn_decode_v2_paged(const void* q, const void* k_pages, const void* v_pages,
                                          const int* block_table, const int* seq_lens, const float* lambda,
                                          void* out, diffattn_dtype dtype, int B, int Hq, int Hkv,
                                          int num_pages, int page_size, int max_pages, void* ws,
                                          size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DIFFATTN_H_ */
