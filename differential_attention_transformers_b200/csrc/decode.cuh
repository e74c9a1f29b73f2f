// decode.cuh -- single-token differential attention decode over a KV cache.
//
// HBM-bound: every cached K and V element is read exactly once for all query
// heads of its KV group and for both maps ("差分注意力" tutorial, section V1
// 到 V2 的 diff: V2 doubles the Q heads over the same KV heads so that one KV
// load serves more queries; V1 is charged with loading the V cache twice,
// which the fused V1 mode here avoids by reading K1, K2 and V once).
//
// Split-KV: the (batch, KV head, 64-key block) space is cut into equal
// contiguous ranges, one per CTA (grid = a multiple of the SM count), so every
// CTA streams the same number of bytes.  A CTA emits one partial record per
// (batch, KV head) segment of its range: for each of the 8 query columns the
// running max m (log2 units), the sum l and the unnormalised output O[128].
// The combine kernel merges the records of each query head (log-sum-exp) and
// applies O = O1/l1 - lambda * O2/l2.
//
// Paged, variable-length mode (V2): the caches are a pool of token-major pages
// [num_pages, page_size, Hkv, 128] addressed through a block table, and each
// sequence has its own length.  Every CTA first builds, in shared memory, the
// prefix of 64-key blocks over the sequences (block counts times Hkv), so the
// same equal split of the flattened block space applies; a CTA's record for
// segment (b, g) goes to slot CTA + b*Hkv + g, which is unique along the
// staircase of CTA ranges and bounded by grid + B*Hkv.  Tiles come in by a 4-D
// tensor map over the pool (one box per page part of the block).  Cache rows
// past a sequence's length are masked and their V rows zeroed in shared memory
// before the PV product, since a page's unused rows may hold anything.
//
// Inner product per 16-key slice and warp, on mma.sync m16n8k16 (bf16, f32
// accumulate) with the keys as M so that the 8 query columns fill N = 8:
//   S^T[16 keys x 8 cols]  = K[16 x 128] . Qcols^T[128 x 8]
//   O^T[128 x 8]          += V^T[128 x 16] . P^T[16 x 8]
// P^T goes from the C-fragment layout to the B-fragment layout with
// movmatrix.trans.  Query columns: V2 = the G <= 8 Q heads of the group
// (pair p = columns 2p, 2p+1); V1 = columns 0..3 map 1 of the group's heads
// and 4..7 map 2, against K = [K1 | K2] (block-diagonal query operand).
#pragma once

#include "common.cuh"

namespace da {

constexpr int DEC_KB = 64;                  // keys per block (one pipeline stage)
constexpr int DEC_CONSUMERS = 4;            // consumer warps, 16 keys of each block each
constexpr int DEC_THREADS = 32 * (DEC_CONSUMERS + 1);
constexpr int DEC_REC = 8 * 2 + 8 * 128;    // floats per partial record: m[8], l[8], O[8][128]
constexpr int DEC_TILE_BYTES = DEC_KB * 128 * 2;  // one 64-key x 128-wide bf16 tile (two 8 KB boxes)
constexpr int DEC_MAXB = 2048;              // paged mode: most sequences per launch

struct DecodeArgs {
  const __nv_bfloat16* q1;  // V2: q [B,Hq,128]; V1: q1 [B,H,64]
  const __nv_bfloat16* q2;  // V1: q2 [B,H,64]; V2: unused
  float* ws;                // partial records
  int B, Hq, Hkv, T;        // Hq: V2 Q heads, V1 heads
  int v1;                   // layout
  int maps;                 // bit0: map 1 columns, bit1: map 2 columns (V1 unfused passes)
  int grid;                 // CTAs
  int maxseg;               // partial slots per CTA
  long long nblk;           // 64-key blocks per (batch, KV head)
  long long total;          // B * Hkv * nblk
  float scale_log2;         // log2(e) / sqrt(d)
  Watch watch;
  // paged mode
  const int* block_table;   // [B, max_pages] page ids
  const int* seq_lens;      // [B]
  int* cu_out;              // [B+1] block prefix, written by CTA 0 for the combine
  int max_pages, page_size, page_shift;
};

__host__ __device__ __forceinline__ long long dec_blk_start(long long i, long long total, int grid) {
  return i * total / grid;
}

// The CTA whose range [dec_blk_start(i), dec_blk_start(i + 1)) holds block x,
// 0 <= x < total: the largest i with i * total / grid <= x, i.e. with
// i * total < (x + 1) * grid.  Its range is never empty.
__host__ __device__ __forceinline__ long long dec_owner(long long x, long long total, int grid) {
  return ((x + 1) * grid - 1) / total;
}

template <int NST, bool PAGED = false>
struct DecSmem {
  alignas(1024) uint8_t k[NST][DEC_TILE_BYTES];
  alignas(1024) uint8_t v[NST][DEC_TILE_BYTES];
  float mo[DEC_CONSUMERS][8][128];
  float mm[DEC_CONSUMERS][8];
  float ml[DEC_CONSUMERS][8];
  alignas(8) uint64_t full[NST];
  uint64_t empty[NST];
  int abort_flag;
  // paged mode: flattened block offset of each sequence (cu[B] = total) and its length
  int cu[PAGED ? DEC_MAXB + 1 : 1];
  int len[PAGED ? DEC_MAXB : 1];
  int part[PAGED ? DEC_THREADS : 1];
};

// Paged mode: the sequence holding flattened block x (largest b with
// cu[b] <= x; empty sequences have cu[b] == cu[b+1] and are skipped).
__device__ __forceinline__ int dec_find_seq(const int* cu, int B, long long x) {
  int lo = 0, hi = B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= x) lo = mid;
    else hi = mid;
  }
  return lo;
}

// Byte offset of element (row, 16-byte chunk) inside a 128-byte-swizzled box
// of 128-byte rows (TMA SWIZZLE_128B, box base 1024-byte aligned).
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ bool bar_any(bool pred) {
  // Barrier over the consumer warps (named barrier 1) with an OR reduction,
  // so that all of them take the same abort decision.
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(DEC_CONSUMERS * 32)
      : "memory");
  return r != 0;
}

template <int NST, bool PAGED = false>
__global__ void __launch_bounds__(DEC_THREADS)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK1, const __grid_constant__ CUtensorMap tmK2,
                    const __grid_constant__ CUtensorMap tmV, DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  DecSmem<NST, PAGED>& S = *reinterpret_cast<DecSmem<NST, PAGED>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(smem_u32(&S.full[i]), 1);
      mbar_init(smem_u32(&S.empty[i]), DEC_CONSUMERS);
    }
    S.abort_flag = 0;
    mbar_fence_init();
  }
  long long total = a.total;
  if constexpr (PAGED) {
    // Block prefix over the sequences: lengths clamped to [0, max_pages * page_size].
    const int per = (a.B + DEC_THREADS - 1) / DEC_THREADS;
    const int b0 = min(a.B, (int)threadIdx.x * per), b1 = min(a.B, b0 + per);
    const int cap = a.max_pages * a.page_size;
    int sum = 0;
    for (int b = b0; b < b1; ++b) {
      const int n = min(max(a.seq_lens[b], 0), cap);
      S.len[b] = n;
      sum += ((n + DEC_KB - 1) / DEC_KB) * a.Hkv;
    }
    S.part[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
      int run = 0;
      for (int i = 0; i < DEC_THREADS; ++i) {
        const int v = S.part[i];
        S.part[i] = run;
        run += v;
      }
      S.cu[a.B] = run;
    }
    __syncthreads();
    int run = S.part[threadIdx.x];
    for (int b = b0; b < b1; ++b) {
      S.cu[b] = run;
      run += ((S.len[b] + DEC_KB - 1) / DEC_KB) * a.Hkv;
    }
    __syncthreads();
    if (blockIdx.x == 0)
      for (int i = threadIdx.x; i <= a.B; i += DEC_THREADS) a.cu_out[i] = S.cu[i];
    total = S.cu[a.B];
  }
  __syncthreads();

  const long long lo = dec_blk_start(blockIdx.x, total, a.grid);
  const long long hi = dec_blk_start(blockIdx.x + 1, total, a.grid);
  const bool load_k2 = a.v1 ? (a.maps & 2) != 0 : true;
  const bool load_k1 = a.v1 ? (a.maps & 1) != 0 : true;

  if (warp == DEC_CONSUMERS) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      tma_prefetch_desc(&tmK1);
      tma_prefetch_desc(&tmV);
      if (a.v1) tma_prefetch_desc(&tmK2);
      long long issued_last[NST];
      for (int i = 0; i < NST; ++i) issued_last[i] = -1;
      bool ok = true;
      // Paged mode: where block x lies -- its KV head, first key and page
      // ids.  The sequence index only moves forward as x does, and the page
      // ids of block x + 1 are read before the wait for block x's stage, so
      // the block-table reads are in flight while this thread waits.
      struct PagedBlk {
        int pg, pkey0, pparts, pages[4];
      };
      int bcur = PAGED ? dec_find_seq(S.cu, a.B, lo) : 0;
      auto locate = [&](long long x) {
        PagedBlk r{0, 0, 1, {0, 0, 0, 0}};
        if constexpr (PAGED) {
          while (S.cu[bcur + 1] <= x) ++bcur;   // skips empty sequences; x < cu[B]
          const int b = bcur;
          const int nb = (S.cu[b + 1] - S.cu[b]) / a.Hkv;
          const int within = (int)(x - S.cu[b]);
          r.pg = within / nb;
          r.pkey0 = (within % nb) * DEC_KB;
          const int* row = a.block_table + (size_t)b * a.max_pages + (r.pkey0 >> a.page_shift);
          if (a.page_size >= DEC_KB) {
            r.pages[0] = row[0];
          } else {
            // page parts of the block that hold a key of the sequence (>= 1);
            // parts wholly past it are not loaded (masked, V rows zeroed)
            r.pparts = min(DEC_KB, S.len[b] - r.pkey0 + a.page_size - 1) / a.page_size;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (i < r.pparts) r.pages[i] = row[i];
          }
        }
        return r;
      };
      PagedBlk nxt{0, 0, 1, {0, 0, 0, 0}};
      if (PAGED && lo < hi) nxt = locate(lo);
      for (long long x = lo; x < hi; ++x) {
        const long long it = x - lo;
        const int st = (int)(it % NST);
        const long long use = it / NST;
        const PagedBlk cur = nxt;
        if (PAGED && x + 1 < hi) nxt = locate(x + 1);
        const int pg = cur.pg, pkey0 = cur.pkey0, pparts = cur.pparts;
        const int pages[4] = {cur.pages[0], cur.pages[1], cur.pages[2], cur.pages[3]};
        if (use > 0 && !wait_bar(smem_u32(&S.empty[st]), (uint32_t)((use - 1) & 1), abort_flag, a.watch)) {
          ok = false;
          break;
        }
        const uint32_t fb = smem_u32(&S.full[st]);
        const uint32_t kd = smem_u32(S.k[st]), vd = smem_u32(S.v[st]);
        if constexpr (PAGED) {
          if (a.page_size >= DEC_KB) {
            const int y = pkey0 & (a.page_size - 1);
            mbar_expect_tx(fb, 2 * DEC_TILE_BYTES);
            tma_load_4d(kd, &tmK1, fb, 0, pg, y, pages[0]);
            tma_load_4d(kd + DEC_TILE_BYTES / 2, &tmK1, fb, 64, pg, y, pages[0]);
            tma_load_4d(vd, &tmV, fb, 0, pg, y, pages[0]);
            tma_load_4d(vd + DEC_TILE_BYTES / 2, &tmV, fb, 64, pg, y, pages[0]);
          } else {
            const int ps = a.page_size;
            mbar_expect_tx(fb, (uint32_t)(pparts * ps * 128 * 4));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (i >= pparts) break;
              const uint32_t off = (uint32_t)(i * ps * 128);
              tma_load_4d(kd + off, &tmK1, fb, 0, pg, 0, pages[i]);
              tma_load_4d(kd + DEC_TILE_BYTES / 2 + off, &tmK1, fb, 64, pg, 0, pages[i]);
              tma_load_4d(vd + off, &tmV, fb, 0, pg, 0, pages[i]);
              tma_load_4d(vd + DEC_TILE_BYTES / 2 + off, &tmV, fb, 64, pg, 0, pages[i]);
            }
          }
          issued_last[st] = use;
          continue;
        }
        const long long bg = x / a.nblk;
        const int key0 = (int)((x % a.nblk) * DEC_KB);
        uint32_t bytes = DEC_TILE_BYTES;  // V
        if (a.v1) bytes += (load_k1 ? DEC_TILE_BYTES / 2 : 0) + (load_k2 ? DEC_TILE_BYTES / 2 : 0);
        else bytes += DEC_TILE_BYTES;
        mbar_expect_tx(fb, bytes);
        if (a.v1) {
          if (load_k1) tma_load_3d(kd, &tmK1, fb, 0, key0, (int)bg);
          if (load_k2) tma_load_3d(kd + DEC_TILE_BYTES / 2, &tmK2, fb, 0, key0, (int)bg);
        } else {
          tma_load_3d(kd, &tmK1, fb, 0, key0, (int)bg);
          tma_load_3d(kd + DEC_TILE_BYTES / 2, &tmK1, fb, 64, key0, (int)bg);
        }
        tma_load_3d(vd, &tmV, fb, 0, key0, (int)bg);
        tma_load_3d(vd + DEC_TILE_BYTES / 2, &tmV, fb, 64, key0, (int)bg);
        issued_last[st] = use;
      }
      (void)ok;
      // Every copy issued must have landed before the CTA may exit.
      for (int i = 0; i < NST; ++i)
        if (issued_last[i] >= 0) drain_bar(smem_u32(&S.full[i]), (uint32_t)(issued_last[i] & 1), a.watch.status);
    }
    return;
  }

  // -------------------------------------------------------------- consumers --
  const int w = warp;                 // 16-key slice of each block
  const int col0 = 2 * (lane & 3);    // this thread's two query columns
  const int grp = a.v1 ? a.Hq / a.Hkv : a.Hq / a.Hkv;
  const int seg_first_bg = PAGED ? 0 : (int)(lo / a.nblk);
  // V1 single-map passes load only one K half: skip the other half's k-steps.
  const int kk_lo = (a.v1 && !load_k1) ? 4 : 0;
  const int kk_hi = (a.v1 && !load_k2) ? 4 : 8;
  // The segment (b, g) holding block xx, its first block and its end within
  // this CTA's range.
  struct Seg {
    long long bg, x0, end;
    int b, g, len;
  };
  auto seg_at = [&](long long xx) {
    Seg sg;
    if constexpr (PAGED) {
      sg.b = dec_find_seq(S.cu, a.B, xx);
      const int nb = (S.cu[sg.b + 1] - S.cu[sg.b]) / a.Hkv;
      sg.g = (int)(xx - S.cu[sg.b]) / nb;
      sg.bg = (long long)sg.b * a.Hkv + sg.g;
      sg.x0 = S.cu[sg.b] + (long long)sg.g * nb;
      sg.end = min(hi, sg.x0 + nb);
      sg.len = S.len[sg.b];
    } else {
      sg.bg = xx / a.nblk;
      sg.x0 = sg.bg * a.nblk;
      sg.end = min(hi, (sg.bg + 1) * a.nblk);
      sg.b = (int)(sg.bg / a.Hkv);
      sg.g = (int)(sg.bg % a.Hkv);
      sg.len = a.T;
    }
    return sg;
  };
  // query operand (B fragments) of segment (b, g) for the 8 columns: n = lane / 4
  auto load_q = [&](int b, int g, uint32_t (&q)[8][2]) {
    const int n = lane >> 2;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t v0 = 0u, v1r = 0u;
      const int dim = 16 * (kk & 3) + 2 * (lane & 3);
      if (a.v1) {
        // columns 0..3: map 1 (dims of K1 = k-steps 0..3); 4..7: map 2 (k-steps 4..7)
        const bool m2 = n >= 4;
        const int hl = n & 3;
        const bool active = (kk >= 4) == m2 && hl < grp && (m2 ? (a.maps & 2) : (a.maps & 1));
        if (active) {
          const __nv_bfloat16* qp = (m2 ? a.q2 : a.q1) + ((size_t)b * a.Hq + g * grp + hl) * 64;
          v0 = *reinterpret_cast<const uint32_t*>(qp + dim);
          v1r = *reinterpret_cast<const uint32_t*>(qp + dim + 8);
        }
      } else if (n < grp) {
        const __nv_bfloat16* qp = a.q1 + ((size_t)b * a.Hq + g * grp + n) * 128 + 64 * (kk >> 2);
        v0 = *reinterpret_cast<const uint32_t*>(qp + dim);
        v1r = *reinterpret_cast<const uint32_t*>(qp + dim + 8);
      }
      q[kk][0] = v0;
      q[kk][1] = v1r;
    }
  };

  bool aborted = false;
  long long x = lo;
  Seg cur{};
  uint32_t qb[8][2];
  if (x < hi) {
    cur = seg_at(x);
    load_q(cur.b, cur.g, qb);
  }
  while (x < hi) {
    const long long bg = cur.bg, seg_end = cur.end, seg_x0 = cur.x0;
    const int len = cur.len;
    // The next segment's queries are loaded now, while this segment's
    // blocks stream, so they are in registers when it starts.
    const bool more = seg_end < hi;
    Seg nxt = cur;
    uint32_t qn[8][2];
    if (more) {
      nxt = seg_at(seg_end);
      load_q(nxt.b, nxt.g, qn);
    }

    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

    for (; x < seg_end; ++x) {
      const long long it = x - lo;
      const int st = (int)(it % NST);
      // a stage already full costs one test and one vote; otherwise lane 0 waits
      const uint32_t fbar = smem_u32(&S.full[st]), fpar = (uint32_t)((it / NST) & 1);
      bool ok = __all_sync(0xffffffffu, mbar_test(fbar, fpar));
      if (!ok) {
        if (lane == 0) ok = wait_bar(fbar, fpar, abort_flag, a.watch);
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
      if (!ok) { aborted = true; break; }

      const uint32_t kb = smem_u32(S.k[st]), vb = smem_u32(S.v[st]);
      const int r0 = 16 * w;
      // S^T = K . Q^T
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if (kk < kk_lo || kk >= kk_hi) continue;
        const int row = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int chunk = 2 * (kk & 3) + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kb + (kk >> 2) * (DEC_TILE_BYTES / 2) + swz(row, chunk), a0, a1, a2, a3);
        mma16816(s, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
      }
      // mask the ragged tail of the cache
      const int blk_key0 = (int)(x - seg_x0) * DEC_KB;
      const int key_lo = blk_key0 + r0 + (lane >> 2);
      const bool v_lo = key_lo < len, v_hi = key_lo + 8 < len;
      // Paged mode: a block that ends past the sequence may hold anything in
      // its tail rows (unused page rows, or rows of parts not loaded); zero this
      // warp's V rows there so that P = 0 meets finite values.
      const bool sanitize = PAGED && blk_key0 + DEC_KB > len;
      if (sanitize) {
        const int rr = r0 + (lane & 15);
        if (blk_key0 + rr >= len) {
          uint4* vrow = reinterpret_cast<uint4*>(S.v[st] + (lane >> 4) * (DEC_TILE_BYTES / 2) + rr * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) vrow[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
      float xs[4];
      xs[0] = v_lo ? s[0] * a.scale_log2 : -INFINITY;
      xs[1] = v_lo ? s[1] * a.scale_log2 : -INFINITY;
      xs[2] = v_hi ? s[2] * a.scale_log2 : -INFINITY;
      xs[3] = v_hi ? s[3] * a.scale_log2 : -INFINITY;
      float mx0 = fmaxf(xs[0], xs[2]), mx1 = fmaxf(xs[1], xs[3]);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
      const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = ex2(m_run[0] - mu0), al1 = ex2(m_run[1] - mu1);
      m_run[0] = mn0;
      m_run[1] = mn1;
      const float p0 = ex2(xs[0] - mu0), p1 = ex2(xs[1] - mu1);
      const float p2 = ex2(xs[2] - mu0), p3 = ex2(xs[3] - mu1);
      l_run[0] = l_run[0] * al0 + p0 + p2;
      l_run[1] = l_run[1] * al1 + p1 + p3;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[i][0] *= al0; acc[i][2] *= al0;
        acc[i][1] *= al1; acc[i][3] *= al1;
      }
      // P = P_hi + P_lo in bf16 (see the prefill kernel): residual MMAs keep
      // the map difference accurate when lambda is near 1.
      const uint32_t h01 = pack_bf16(p0, p1), h23 = pack_bf16(p2, p3);
      const uint32_t pb0 = movm_t(h01);
      const uint32_t pb1 = movm_t(h23);
      const uint32_t pr0 = movm_t(pack_bf16(p0 - __uint_as_float(h01 << 16), p1 - __uint_as_float(h01 & 0xFFFF0000u)));
      const uint32_t pr1 = movm_t(pack_bf16(p2 - __uint_as_float(h23 << 16), p3 - __uint_as_float(h23 & 0xFFFF0000u)));
      // O^T += V^T . P^T
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int mi = lane >> 3;
        const int row = r0 + (lane & 7) + (mi >> 1) * 8;
        const int chunk = 2 * (mt & 3) + (mi & 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vb + (mt >> 2) * (DEC_TILE_BYTES / 2) + swz(row, chunk), a0, a1, a2, a3);
        mma16816(acc[mt], a0, a1, a2, a3, pb0, pb1);
        mma16816(acc[mt], a0, a1, a2, a3, pr0, pr1);
      }
      // generic-proxy writes to the stage must be ordered before the next
      // copy into it (async proxy)
      if (sanitize) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.empty[st]));
    }

    // ---- merge the four warps' states of this segment into one record ----
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], o);
      l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], o);
    }
    if (lane < 4) {
      S.mm[w][col0] = m_run[0]; S.mm[w][col0 + 1] = m_run[1];
      S.ml[w][col0] = l_run[0]; S.ml[w][col0 + 1] = l_run[1];
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int dv = 16 * mt + (lane >> 2);
      S.mo[w][col0][dv] = acc[mt][0];
      S.mo[w][col0 + 1][dv] = acc[mt][1];
      S.mo[w][col0][dv + 8] = acc[mt][2];
      S.mo[w][col0 + 1][dv + 8] = acc[mt][3];
    }
    if (bar_any(aborted || *abort_flag)) break;
    {
      const int t = threadIdx.x;  // 0..127: output dv index, all 8 columns
      float* rec = PAGED ? a.ws + ((size_t)blockIdx.x + (size_t)bg) * DEC_REC
                         : a.ws + ((size_t)blockIdx.x * a.maxseg + (size_t)(bg - seg_first_bg)) * DEC_REC;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < DEC_CONSUMERS; ++ww) M = fmaxf(M, S.mm[ww][c]);
        const float Mu = M == -INFINITY ? 0.f : M;
        float o = 0.f, l = 0.f;
#pragma unroll
        for (int ww = 0; ww < DEC_CONSUMERS; ++ww) {
          const float f = ex2(S.mm[ww][c] - Mu);
          o += S.mo[ww][c][t] * f;
          l += S.ml[ww][c] * f;
        }
        rec[16 + c * 128 + t] = o;
        if (t == 0) { rec[c] = M; rec[8 + c] = l; }
      }
    }
    if (bar_any(false)) break;  // records read from smem before the next segment overwrites it
    if (more) {
      cur = nxt;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        qb[kk][0] = qn[kk][0];
        qb[kk][1] = qn[kk][1];
      }
    }
  }
}

struct CombineArgs {
  const float* ws;
  const float* lambda;
  __nv_bfloat16* out;  // V2: [B, Hq/2, 128]; V1: [B, H, 128]
  int B, Hq, Hkv, v1;
  int grid, maxseg;
  long long nblk, total;
  int two_pass;        // V1 unfused: map 2 records live in a second workspace half
  size_t half_floats;  // offset of the second half
  const int* cu;       // paged mode: block prefix written by the split kernel (null otherwise)
};

// One CTA (128 threads = the value width) per (batch, KV head): the output
// heads of a KV head share one walk over the split CTAs' records.  Each
// output keeps the order of operations of a walk of its own, so the result
// does not depend on how many heads share it.
__global__ void __launch_bounds__(128) decode_combine_kernel(CombineArgs a) {
  constexpr int MAXO = 4;   // output heads of a KV head: V2 (8 Q columns) / 2, V1 (4 + 4 columns)
  const int t = threadIdx.x;
  const int Hout = a.v1 ? a.Hq : a.Hq / 2;
  const int grp = a.Hq / a.Hkv;
  const int opg = a.v1 ? grp : grp / 2;
  const int b = blockIdx.x / a.Hkv, g = blockIdx.x % a.Hkv;
  const long long bg = (long long)b * a.Hkv + g;
  long long x0, x1, total = a.total;
  if (a.cu) {   // paged: this sequence's blocks per KV head from the prefix
    const int nb = (a.cu[b + 1] - a.cu[b]) / a.Hkv;
    x0 = a.cu[b] + (long long)g * nb;
    x1 = x0 + nb;
    total = a.cu[a.B];
  } else {
    x0 = bg * a.nblk;
    x1 = x0 + a.nblk;
  }
  // query column of output head oh and map mp: V2 pair oh = columns 2 oh,
  // 2 oh + 1; V1 head oh = column oh (map 1) and 4 + oh (map 2)
  auto col = [&](int oh, int mp) { return a.v1 ? (mp ? 4 + oh : oh) : 2 * oh + mp; };

  // The CTAs whose ranges overlap [x0, x1), in ascending order: start at the
  // owner of x0, then jump to the owner of the block after each range.  Only
  // CTAs that wrote a record for this segment are visited (with short caches
  // most CTAs of the grid have an empty range and none of them is touched).
  // Two walks: the maxima of both maps first, then the scaled sums, so every
  // record is scaled by its exact distance to the global maximum.
  auto record = [&](long long i, long long s, int mp) -> const float* {
    const float* base = a.ws + ((a.two_pass && mp == 1) ? a.half_floats : 0);
    return a.cu ? base + ((size_t)i + (size_t)bg) * DEC_REC
                : base + ((size_t)i * a.maxseg + (size_t)(bg - s / a.nblk)) * DEC_REC;
  };
  float M[MAXO][2];
#pragma unroll
  for (int oh = 0; oh < MAXO; ++oh) M[oh][0] = M[oh][1] = -INFINITY;
  for (long long x = x0; x < x1;) {
    const long long i = dec_owner(x, total, a.grid);
    const long long s = dec_blk_start(i, total, a.grid), e = dec_blk_start(i + 1, total, a.grid);
#pragma unroll
    for (int oh = 0; oh < MAXO; ++oh)
      if (oh < opg) {
#pragma unroll
        for (int mp = 0; mp < 2; ++mp) M[oh][mp] = fmaxf(M[oh][mp], record(i, s, mp)[col(oh, mp)]);
      }
    x = e;
  }
  float o[MAXO][2], l[MAXO][2];
#pragma unroll
  for (int oh = 0; oh < MAXO; ++oh) o[oh][0] = o[oh][1] = l[oh][0] = l[oh][1] = 0.f;
  for (long long x = x0; x < x1;) {
    const long long i = dec_owner(x, total, a.grid);
    const long long s = dec_blk_start(i, total, a.grid), e = dec_blk_start(i + 1, total, a.grid);
#pragma unroll
    for (int oh = 0; oh < MAXO; ++oh)
      if (oh < opg) {
#pragma unroll
        for (int mp = 0; mp < 2; ++mp) {
          const int c = col(oh, mp);
          const float* rec = record(i, s, mp);
          const float f = ex2(rec[c] - (M[oh][mp] == -INFINITY ? 0.f : M[oh][mp]));
          o[oh][mp] += rec[16 + c * 128 + t] * f;
          l[oh][mp] += rec[8 + c] * f;
        }
      }
    x = e;
  }
#pragma unroll
  for (int oh = 0; oh < MAXO; ++oh)
    if (oh < opg) {
      const int h = g * opg + oh;
      const float r0 = l[oh][0] > 0.f ? o[oh][0] / l[oh][0] : 0.f;
      const float r1 = l[oh][1] > 0.f ? o[oh][1] / l[oh][1] : 0.f;
      const float lam = a.lambda[h];
      a.out[((size_t)b * Hout + h) * 128 + t] = __float2bfloat16_rn(__fsub_rn(r0, __fmul_rn(lam, r1)));
    }
}

}  // namespace da
