// Parameter-free MoBA gate on the tensor cores: scores s = <q, Kbar[b]> for the strictly
// earlier blocks of the query's sequence, forced own block, top-(k-1) past blocks by
// descending score with ties to the lower block index.  (MoBA README, "Parameter-less
// Gating Mechanism" and the FAQ answer of GitHub issue #27: the own block is always taken
// and is not a candidate, k-1 more blocks come from earlier blocks; youleyou.com,
// "Kimi发布MoBA突破性实现无限上下文", section "PyTorch实现关键要点": score by the product of the
// query with the pooled keys, mask future blocks, top-k.)
//
// Scores.  The candidate blocks 0..i-1 of a 128-token query tile are processed in chunks of
// up to 64: the chunk's pooled keys, split into bf16 hi + lo parts (Kbar = hi + lo +
// O(2^-17 |Kbar|)), are staged by TMA and S = Q hi^T + Q lo^T accumulates in fp32 TMEM
// (double-buffered).  Thread r reads row r of S from TMEM and keeps a running top-(k-1) list
// in registers.
//
// Two kernels.  gate_tc_kernel takes 128 tokens of one head per CTA, three CTAs per SM.
// gate_group_kernel, for the exact selection (top_k > 5) of KV groups of a multiple of four
// query heads, is persistent, one CTA per SM: an item is 128 tokens x four query heads of one
// KV group, so a chunk of pooled keys is staged once for 512 rows, the next two chunks (of
// this item or the next ones) are in flight while the current one is multiplied and scanned,
// and the next item's Q tiles load as soon as the current item's MMAs are done.
//
// Selection cost.  With at most four blocks to choose (top_k <= 5) and more than one chunk of
// candidates (the set-up below does not pay for itself on one chunk), a score is not inserted
// into the running list one by one.  Each score becomes a key in [1, 2): the score scaled by
// 0.49 / B, where B = |q| max_b |Kbar[b]| bounds every candidate's |s| (Cauchy-Schwarz), is
// rounded onto the grid 2^-18 by one fma against 48 (whose ulp is 2^-18), moved to 1.5 + that
// value, and the low five mantissa bits, free on that grid, take 31 - (column in its group of
// 32).  Keys then compare as plain floats: a larger key is a higher score, and among scores
// that round to the same grid point, the lower block.  A min/max network takes the group's
// top keys and only those are decoded and merged into the running list.  Scores are thus
// ordered with a resolution of 2^-18 B / 0.49, the order of the hi/lo error of the scores
// themselves (2^-18 sum_d |q_d| |Kbar_d| <= 2^-18 B); exact ties still go to the lower block.
#include <cudaTypedefs.h>
#include <float.h>

#include "moba_internal.cuh"
#include "sm100.cuh"

namespace moba {

namespace {

constexpr int kRows = 128;  // query rows per tile
constexpr int kCand = 64;   // candidate blocks per chunk

__device__ __forceinline__ bool ranks_before(float sa, int32_t ba, float sb, int32_t bb) {
  return sa > sb || (sa == sb && ba < bb);
}

// Running top-m of one query row over candidates that arrive in ascending block index.
// kMaxM: compile-time capacity (>= m), so the lists live in registers.  In a list the first
// kMaxM - m slots hold sentinels that rank before every score and are never displaced, so
// the m live slots are the last m and the current m-th best is always the last slot.
// kQuant: quantized keys + min/max network (kMaxM <= 4 only), else exact insertion.
template <int kMaxM, bool kQuant_ = (kMaxM <= 4)>
struct RowTopK {
  static constexpr bool kQuant = kQuant_;
  static_assert(!kQuant || kMaxM <= 4, "the quantized form keeps at most four blocks");
  // the exact form keeps kLists lists; column x of a group goes to list x % kLists, so
  // kLists insertion chains run side by side
  static constexpr int kLists = kQuant ? 1 : (kMaxM <= 4 ? 4 : (kMaxM <= 8 ? 2 : 1));
  float ls[kLists][kMaxM];
  int32_t lb[kLists][kMaxM];

  __device__ __forceinline__ void init(int m) {
#pragma unroll
    for (int j = 0; j < kLists; ++j)
#pragma unroll
      for (int q = 0; q < kMaxM; ++q) {
        const bool live = q >= kMaxM - m;
        // quantized keys of real candidates are >= 1, exact scores are > -FLT_MAX
        ls[j][q] = live ? (kQuant ? 0.f : -FLT_MAX) : FLT_MAX;
        lb[j][q] = live ? INT32_MAX : -1;
      }
  }

  // A new candidate ranks after every listed entry whose score is >= its own (ties go to
  // the lower index, which arrived first) and before the rest: the list shifts down by one
  // from that position.  A score at or below the last slot leaves the list unchanged.
  __device__ __forceinline__ static void insert(float (&l)[kMaxM], int32_t (&b)[kMaxM], float sc, int32_t blk) {
    bool ge[kMaxM];
#pragma unroll
    for (int q = 0; q < kMaxM; ++q) ge[q] = l[q] >= sc;
#pragma unroll
    for (int q = kMaxM - 1; q >= 1; --q) {
      l[q] = ge[q] ? l[q] : (ge[q - 1] ? sc : l[q - 1]);
      b[q] = ge[q] ? b[q] : (ge[q - 1] ? blk : b[q - 1]);
    }
    l[0] = ge[0] ? l[0] : sc;
    b[0] = ge[0] ? b[0] : blk;
  }

  // The 32 scores (fp32 bits) of candidate blocks b0 .. b0 + 31; blocks >= i are not
  // candidates.  scl: the row's key scale (quantized form only).
  __device__ __forceinline__ void scan(const uint32_t (&v)[32], int32_t b0, int i, float scl) {
    if constexpr (kQuant) {
      float key[32];
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        // fl(s * scl + 48) is 48 + s * scl rounded to the grid 2^-18; minus 46.5 moves it to
        // [1.01, 1.99] exactly, where the grid leaves five mantissa bits for the code.
        float t0, t1;
        fma2(t0, t1, __uint_as_float(v[x]), __uint_as_float(v[x + 1]), scl, scl, 48.f, 48.f);
        add2(t0, t1, t0, t1, -46.5f, -46.5f);
        add2(key[x], key[x + 1], t0, t1, (float)(31 - x) * 0x1p-23f, (float)(30 - x) * 0x1p-23f);
      }
      const int nv = i - b0;  // candidate columns in this group (the same for the whole tile)
      if (nv < 32) {
#pragma unroll
        for (int x = 0; x < 32; ++x) key[x] = x < nv ? key[x] : 0.f;
      }
      float top[kMaxM];
      if constexpr (kMaxM == 2) {
        // Tournament: sorted pairs, then the top 2 of two top-2 lists is
        // (max of the heads, max of the smaller head and both tails).
        float hd[16], tl[16];
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          hd[p] = fmaxf(key[2 * p], key[2 * p + 1]);
          tl[p] = fminf(key[2 * p], key[2 * p + 1]);
        }
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
          for (int p = 0; p < w; ++p) {
            const float H = fmaxf(hd[2 * p], hd[2 * p + 1]);
            tl[p] = max3(fminf(hd[2 * p], hd[2 * p + 1]), tl[2 * p], tl[2 * p + 1]);
            hd[p] = H;
          }
        top[0] = hd[0];
        top[1] = tl[0];
      } else {
        // Insertion network: each key passes down the sorted list, keeping the larger.
#pragma unroll
        for (int q = 0; q < kMaxM; ++q) top[q] = 0.f;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          float k = key[x];
#pragma unroll
          for (int q = 0; q < kMaxM - 1; ++q) {
            const float hi = fmaxf(top[q], k);
            k = fminf(top[q], k);
            top[q] = hi;
          }
          top[kMaxM - 1] = fmaxf(top[kMaxM - 1], k);
        }
      }
      // The group's best keys, best first, into the running list (grid value + block); an
      // equal grid value from a later group ranks after the listed one (lower block).
#pragma unroll
      for (int q = 0; q < kMaxM; ++q) {
        const uint32_t bits = __float_as_uint(top[q]);
        insert(ls[0], lb[0], __uint_as_float(bits & ~31u), b0 + 31 - (int32_t)(bits & 31u));
      }
    } else {
      // Exact scores; columns at or past the query block score -FLT_MAX, which never enters
      // a list.  Short lists take every score without a branch; longer ones skip a score at
      // or below their last slot.
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int32_t b = b0 + x;
        const float sc = b < i ? __uint_as_float(v[x]) : -FLT_MAX;
        if constexpr (kMaxM <= 4) {
          insert(ls[x % kLists], lb[x % kLists], sc, b);
        } else {
          if (sc > ls[x % kLists][kMaxM - 1]) insert(ls[x % kLists], lb[x % kLists], sc, b);
        }
      }
    }
  }

  // Own block in slot 0, the m chosen blocks by descending score, -1 padding.
  __device__ __forceinline__ void write(int32_t* out, int i, int m, int k) {
    // fold lists 1.. into list 0 (their entries are not in index order: full comparison)
#pragma unroll
    for (int j = 1; j < kLists; ++j)
#pragma unroll
      for (int p = 0; p < kMaxM; ++p) {
        if (p < kMaxM - m) continue;
        float sc = ls[j][p];
        int32_t cb = lb[j][p];
#pragma unroll
        for (int q = 0; q < kMaxM; ++q) {
          const bool take = ranks_before(sc, cb, ls[0][q], lb[0][q]);
          const float os = ls[0][q];
          const int32_t ob = lb[0][q];
          ls[0][q] = take ? sc : os;
          lb[0][q] = take ? cb : ob;
          sc = take ? os : sc;
          cb = take ? ob : cb;
        }
      }
    out[0] = i;
#pragma unroll
    for (int q = 0; q < kMaxM; ++q)
      if (q >= kMaxM - m) out[1 + q - (kMaxM - m)] = lb[0][q];
    for (int q = 1 + m; q < k; ++q) out[q] = -1;
  }
};

// Key scale of the quantized form for one row: 0.49 / B, B = |q| sqrt(kmax2), where kmax2 is
// the largest squared norm of the row's candidate pooled keys and q is row r of a staged
// [128 x D] tile (rows 128-byte swizzled: the sum of squares does not depend on the order in
// which the row's 16-byte pieces are read).  |s| <= B for every candidate, so s * scale lies
// in [-0.49, 0.49] (up to the scores' own rounding); B == 0, or a non-finite B, gives scale 0,
// which leaves every key at 1.5 + code: the lowest blocks.
template <int D>
__device__ __forceinline__ float key_scale(const uint8_t* qtile, int r, float kmax2) {
  const uint8_t* qrow = qtile + r * 128;
  float qn = 0.f;
#pragma unroll
  for (int hh = 0; hh < D / 64; ++hh)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 u = *reinterpret_cast<const uint4*>(qrow + hh * kRows * 128 + j * 16);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(w4[e] << 16), hi = __uint_as_float(w4[e] & 0xffff0000u);
        qn = fmaf(lo, lo, qn);
        qn = fmaf(hi, hi, qn);
      }
    }
  const float bound = sqrtf(qn) * sqrtf(kmax2);
  return (bound > 1e-30f && bound <= FLT_MAX) ? 0.49f / bound : 0.f;
}

// The MMAs of one chunk for one 128-row Q tile: S = Q hi^T + Q lo^T into n TMEM columns.
template <int D>
__device__ __forceinline__ void issue_chunk_mma(uint32_t tmem_s, uint32_t sQ, uint32_t sHi, uint32_t sLo, int n) {
  const uint32_t idesc = idesc_bf16(kRows, n, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t koff = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
    const uint32_t boff = (kk >> 2) * (kCand * 128) + (kk & 3) * 32;
    const uint64_t ad = sdesc_sw128(sQ + koff, 16, 1024);
    mma_bf16_ss_warp(tmem_s, ad, sdesc_sw128(sHi + boff, 16, 1024), idesc, kk > 0 ? 1u : 0u);
    mma_bf16_ss_warp(tmem_s, ad, sdesc_sw128(sLo + boff, 16, 1024), idesc, 1u);
  }
}

// TMEM columns [t0, t0 + 32 * ngrp) of this thread's row, 32 at a time, through scan(v, g).
// kAhead: the next group's load is in flight while the current group is scanned (32 more
// registers; the group kernel's 16 epilogue warps hide the load latency without it).
template <bool kAhead = true, typename Scan>
__device__ __forceinline__ void scan_tmem(uint32_t t0, int ngrp, Scan&& scan) {
  if constexpr (!kAhead) {
    for (int gi = 0; gi < ngrp; ++gi) {
      uint32_t v[32];
      tmem_ld32(t0 + gi * 32, v);
      tmem_wait_ld(v);
      scan(v, gi);
    }
    return;
  }
  uint32_t va[32], vb[32];
  tmem_ld32(t0, va);
  tmem_wait_ld(va);
  for (int gi = 0; gi < ngrp; gi += 2) {
    if (gi + 1 < ngrp) tmem_ld32(t0 + (gi + 1) * 32, vb);
    scan(va, gi);
    if (gi + 1 < ngrp) {
      tmem_wait_ld(vb);
      if (gi + 2 < ngrp) tmem_ld32(t0 + (gi + 2) * 32, va);
      scan(vb, gi + 1);
      if (gi + 2 < ngrp) tmem_wait_ld(va);
    }
  }
}

// ============================================================================ per head
constexpr int kThreads = 160;  // warps 0-3 epilogue, warp 4 TMA + MMA (whole warp)

template <int D>
struct GLayout {
  static constexpr int kQ = 0;                      // [128 x D] bf16
  static constexpr int kHi = kQ + kRows * D * 2;    // [kCand x D] bf16
  static constexpr int kLo = kHi + kCand * D * 2;   // [kCand x D] bf16
  static constexpr int kBar = kLo + kCand * D * 2;
  static constexpr int kAlloc = kBar + 128 + 1024;
  static constexpr uint32_t kTmemCols = 2 * kCand;  // double-buffered S
};

enum GBar { kFull = 0, kQFull, kKFree, kTFull0, kTFull1, kTFree0, kTFree1, kGDone, kGNumBars };

// One CTA per 128 tokens of one query head inside one query block i, three CTAs per SM;
// one chunk buffer (the next chunk loads once the current chunk's MMAs have read it).
template <int D, int kMaxM>
__global__ void __launch_bounds__(kThreads, 3)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmHi,
                   const __grid_constant__ CUtensorMap tmLo, Geom g, const float* __restrict__ kn2,
                   int32_t* __restrict__ sel) {
  using L = GLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kGNumBars * 8);
  float* red = reinterpret_cast<float*>(smem + L::kBar + kGNumBars * 8 + 16);  // [4]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int per_blk = g.bs / kRows;
  const int i = blockIdx.x / per_blk;  // query block (local to the sequence)
  const int qt = blockIdx.x - i * per_blk;
  const int s = blockIdx.y, h = blockIdx.z, gk = h / g.G;
  const int32_t ts = seq_start(g, s), te = seq_end(g, s);
  const int32_t q0 = ts + i * g.bs + qt * kRows;
  if (q0 >= te) return;
  const int nrows = min(kRows, te - q0);
  const int m = min(g.k - 1, i);  // past blocks to choose
  if (m == 0) {  // nothing to score: own block only
    for (int r = tid; r < nrows; r += kThreads) {
      int32_t* out = sel + ((int64_t)(q0 + r) * g.Hq + h) * g.k;
      out[0] = i;
      for (int q = 1; q < g.k; ++q) out[q] = -1;
    }
    return;
  }
  const int nch = (i + kCand - 1) / kCand;

  if (warp == 4) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    mbar_init(&bars[kFull], 1);
    mbar_init(&bars[kQFull], 1);
    mbar_init(&bars[kKFree], 1);
    mbar_init(&bars[kTFull0], 1);
    mbar_init(&bars[kTFull1], 1);
    mbar_init(&bars[kTFree0], kRows);
    mbar_init(&bars[kTFree1], kRows);
    mbar_init(&bars[kGDone], 1);
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t kb_row0 = (int64_t)s * g.MB;  // first pooled-key row of this sequence
  bool ok = true;

  if (warp < 4) {
    // ========================================================= epilogue: running top-m
    const int r = tid;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // One selection form for the whole row: scan(tk, scl) walks the chunks.
    auto select = [&](auto& tk, float scl) {
      tk.init(m);
      for (int c = 0; c < nch && ok; ++c) {
        const int buf = c & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kTFull0 + buf], (c >> 1) & 1, g.err));
        if (!ok) break;
        tc_fence_after();
        const int c0 = c * kCand;
        scan_tmem(tmem + lane_off + buf * kCand, (min(kCand, i - c0) + 31) / 32,
                  [&](const uint32_t (&v)[32], int gi) { tk.scan(v, c0 + gi * 32, i, scl); });
        tc_fence_before();
        mbar_arrive(&bars[kTFree0 + buf]);
      }
      if (ok && r < nrows) tk.write(sel + ((int64_t)(q0 + r) * g.Hq + h) * g.k, i, m, g.k);
    };
    // Quantized keys pay a per-row set-up (the key scale) that a single chunk of candidates
    // does not repay: rows with at most kCand candidates take the exact insertion.
    bool quant = false;
    if constexpr (kMaxM <= 4) quant = i > kCand;  // the same for the whole CTA
    if (quant) {
      if constexpr (kMaxM <= 4) {
        // the candidates' largest squared norm, by all 128 threads
        const float* kn = kn2 + ((int64_t)s * g.Hkv + gk) * g.MB;
        float kmax = 0.f;
        for (int b = r; b < i; b += kRows) kmax = fmaxf(kmax, kn[b]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        if (lane == 0) red[warp] = kmax;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        kmax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kQFull], 0, g.err));
        const float scl = ok ? key_scale<D>(smem + L::kQ, r, kmax) : 0.f;
        RowTopK<kMaxM, true> tk;
        select(tk, scl);
      }
    } else {
      RowTopK<kMaxM, false> tk;
      select(tk, 0.f);
    }
  } else {
    // ========================================================= TMA + MMA issuer (warp 4)
    // The whole warp runs this loop: lane 0 issues the TMA copies, one elected lane the MMAs.
    auto load_chunk = [&](int c, bool with_q) {
      if (lane != 0) return;
      if (with_q) {
        mbar_expect_tx(&bars[kQFull], kRows * D * 2);
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(smem + L::kQ + hh * kRows * 128, &tmQ, &bars[kQFull], hh * 64, h, q0);
      }
      // one box of kCand rows (rows past the candidates load too, and are never scanned)
      mbar_expect_tx(&bars[kFull], (uint32_t)(2 * kCand * D * 2));
      const int row = (int)(kb_row0 + c * kCand);
      for (int hh = 0; hh < D / 64; ++hh) {
        tma_load_3d(smem + L::kHi + hh * kCand * 128, &tmHi, &bars[kFull], hh * 64, gk, row);
        tma_load_3d(smem + L::kLo + hh * kCand * 128, &tmLo, &bars[kFull], hh * 64, gk, row);
      }
    };
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmHi);
      prefetch_tmap(&tmLo);
    }
    load_chunk(0, true);
    __syncwarp();
    for (int c = 0; c < nch && ok; ++c) {
      const int buf = c & 1;
      ok = mbar_wait_warp(&bars[kFull], c & 1, g.err);
      if (ok && c == 0) ok = mbar_wait_warp(&bars[kQFull], 0, g.err);
      if (ok && c >= 2) ok = mbar_wait_warp(&bars[kTFree0 + buf], ((c >> 1) - 1) & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      const int ncand = min(kCand, i - c * kCand);
      issue_chunk_mma<D>(tmem + buf * kCand, smem_u32(smem + L::kQ), smem_u32(smem + L::kHi),
                         smem_u32(smem + L::kLo), (ncand + 15) & ~15);
      mma_commit_warp(&bars[kTFull0 + buf]);
      if (c + 1 < nch) {  // the buffer takes the next chunk once these MMAs have read it
        mma_commit_warp(&bars[kKFree]);
        ok = mbar_wait_warp(&bars[kKFree], c & 1, g.err);
        if (!ok) break;
        load_chunk(c + 1, false);
        __syncwarp();
      }
    }
    mma_commit_warp(&bars[kGDone]);
    mbar_wait_warp(&bars[kGDone], 0, g.err);
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ============================================================================ KV group
constexpr int kGrpHeads = 4;                            // query heads per item
constexpr int kGrpEpiWarps = 4 * kGrpHeads;             // four warps (128 rows) per head
constexpr int kGrpThreads = (kGrpEpiWarps + 1) * 32;    // + the TMA/MMA warp
constexpr uint32_t kGrpTmemCols = 512;                  // kGrpHeads x 2 buffers x kCand

template <int D>
struct GrpLayout {
  static constexpr int kQTile = kRows * D * 2;          // [128 x D] bf16
  static constexpr int kChunk = 2 * kCand * D * 2;      // hi [kCand x D] + lo [kCand x D] bf16
  static constexpr int kBufs = 3;                       // chunk buffers: two copies ahead
  static constexpr int kQ = 0;                          // kGrpHeads tiles
  static constexpr int kBuf0 = kQ + kGrpHeads * kQTile;
  static constexpr int kBar = kBuf0 + kBufs * kChunk;
  static constexpr int kBytes = kBar + 256;
  // At least half of an SM's shared memory, so that no second CTA of this kernel shares
  // the SM: each holds all 512 TMEM columns for its whole (persistent) life.
  static constexpr int kAlloc = kBytes + 1024 > 116 * 1024 ? kBytes + 1024 : 116 * 1024;
  __host__ __device__ static constexpr int hi(int b) { return kBuf0 + b * kChunk; }
  __host__ __device__ static constexpr int lo(int b) { return kBuf0 + b * kChunk + kCand * D * 2; }
};

enum GrpBar {
  pFull0 = 0, pFull1, pFull2, pKFree0, pKFree1, pKFree2, pTFull0, pTFull1, pTFree0, pTFree1, pQFull, pQFree,
  pQRead, pDone, pNumBars
};
static_assert(pNumBars * 8 + 16 <= 256, "barrier area");

// Item = (query block i, sequence, 128-token tile, KV head, group of up to four of its query
// heads); items run in descending block index, so the heaviest (most candidates) go first.
struct GItem {
  int s, i, gk, h0, nh, m, nch, nrows;
  int32_t q0;
  bool valid;
};

__device__ __forceinline__ GItem item_geom(const Geom& g, int64_t id, int nhg) {
  const int per_blk = g.bs / kRows;
  const int64_t nhk = (int64_t)g.Hkv * nhg;
  GItem it;
  const int hk = (int)(id % nhk);
  id /= nhk;
  const int qt = (int)(id % per_blk);
  id /= per_blk;
  it.s = (int)(id % g.num_seqs);
  it.i = g.MB - 1 - (int)(id / g.num_seqs);
  it.gk = hk / nhg;
  const int hg = hk - it.gk * nhg;
  it.h0 = it.gk * g.G + hg * kGrpHeads;
  it.nh = min(kGrpHeads, g.G - hg * kGrpHeads);
  const int32_t ts = seq_start(g, it.s), te = seq_end(g, it.s);
  it.q0 = ts + it.i * g.bs + qt * kRows;
  it.valid = it.q0 < te;
  it.nrows = it.valid ? min(kRows, te - it.q0) : 0;
  it.m = min(g.k - 1, it.i);
  it.nch = it.m == 0 ? 0 : (it.i + kCand - 1) / kCand;
  return it;
}

template <int D, int kMaxM>
__global__ void __launch_bounds__(kGrpThreads, 1)
    gate_group_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmHi,
                      const __grid_constant__ CUtensorMap tmLo, Geom g, int32_t* __restrict__ sel, int64_t nitems,
                      int nhg) {
  static_assert(!RowTopK<kMaxM>::kQuant, "the group kernel runs the exact selection");
  using L = GrpLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + pNumBars * 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == kGrpEpiWarps) {
    tmem_alloc(tmem_slot, kGrpTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    for (int b = 0; b < L::kBufs; ++b) {
      mbar_init(&bars[pFull0 + b], 1);
      mbar_init(&bars[pKFree0 + b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[pTFull0 + b], 1);
      mbar_init(&bars[pTFree0 + b], kGrpEpiWarps * 32);
    }
    mbar_init(&bars[pQFull], 1);
    mbar_init(&bars[pQFree], 1);
    mbar_init(&bars[pQRead], kGrpEpiWarps * 32);
    mbar_init(&bars[pDone], 1);
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp < kGrpEpiWarps) {
    // ========================================================= epilogue: running top-m
    // Warp w takes rows 32 (w % 4) .. + 31 (its TMEM lanes) of head slot w / 4.  Every
    // epilogue thread arrives on every barrier, whether or not its head slot is in use.
    const int hs = warp >> 2, r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t gc = 0, qi = 0;  // chunks and Q items done
    for (int64_t id = blockIdx.x; id < nitems && ok; id += gridDim.x) {
      const GItem it = item_geom(g, id, nhg);
      if (!it.valid) continue;
      const bool mine = hs < it.nh && r < it.nrows;
      int32_t* out = sel + ((int64_t)(it.q0 + r) * g.Hq + it.h0 + hs) * g.k;
      if (it.nch == 0) {  // nothing to score: own block only
        if (mine) {
          out[0] = it.i;
          for (int q = 1; q < g.k; ++q) out[q] = -1;
        }
        continue;
      }
      // no Q reads here, but the arrival below must not run ahead of this item's Q load: the
      // producer waits for each item's arrivals before it loads the next item's Q
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[pQFull], qi & 1, g.err));
      if (!ok) break;
      mbar_arrive(&bars[pQRead]);  // this item's Q tiles may be replaced once its MMAs are done too
      RowTopK<kMaxM> tk;
      tk.init(it.m);
      for (int c = 0; c < it.nch && ok; ++c, ++gc) {
        const int tb = gc & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[pTFull0 + tb], (gc >> 1) & 1, g.err));
        if (!ok) break;
        tc_fence_after();
        if (hs < it.nh) {
          const int c0 = c * kCand;
          scan_tmem<false>(tmem + lane_off + (uint32_t)((hs * 2 + tb) * kCand), (min(kCand, it.i - c0) + 31) / 32,
                    [&](const uint32_t (&v)[32], int gi) { tk.scan(v, c0 + gi * 32, it.i, 0.f); });
        }
        tc_fence_before();
        mbar_arrive(&bars[pTFree0 + tb]);
      }
      if (ok && mine) tk.write(out, it.i, it.m, g.k);
      ++qi;
    }
  } else {
    // ========================================================= TMA + MMA issuer
    // The whole warp runs this loop: lane 0 issues the TMA copies, one elected lane the MMAs.
    // Chunks are numbered across the CTA's items (gc); chunk gc uses key buffer gc % 3 and
    // TMEM buffer gc & 1.  The copies run two chunks ahead of the MMAs (across item
    // boundaries), so the next two chunks are in flight while the current one is multiplied.
    auto next_item = [&](int64_t id, GItem& it) -> int64_t {  // first item from id on with work
      for (; id < nitems; id += gridDim.x) {
        it = item_geom(g, id, nhg);
        if (it.valid && it.nch > 0) return id;
      }
      return nitems;
    };
    auto load_q = [&](const GItem& it) {
      if (lane != 0) return;
      mbar_expect_tx(&bars[pQFull], (uint32_t)(it.nh * L::kQTile));
      for (int hs = 0; hs < it.nh; ++hs)
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(smem + L::kQ + hs * L::kQTile + hh * kRows * 128, &tmQ, &bars[pQFull], hh * 64, it.h0 + hs,
                      it.q0);
    };
    // the copy cursor: the next chunk to load (item lid, chunk lc) and its number gl
    GItem lit;
    int64_t lid = next_item(blockIdx.x, lit);
    int lc = 0;
    uint32_t gl = 0;
    auto load_next = [&]() -> bool {
      if (lid >= nitems) return false;
      const int b = (int)(gl % L::kBufs);
      // the buffer was last read by chunk gl - 3's MMAs
      if (gl >= (uint32_t)L::kBufs && !mbar_wait_warp(&bars[pKFree0 + b], (gl / L::kBufs - 1) & 1, g.err))
        return false;
      if (lane == 0) {
        // one box of kCand rows (rows past the candidates load too, and are never scanned)
        mbar_expect_tx(&bars[pFull0 + b], (uint32_t)L::kChunk);
        const int row = (int)((int64_t)lit.s * g.MB + lc * kCand);
        for (int hh = 0; hh < D / 64; ++hh) {
          tma_load_3d(smem + L::hi(b) + hh * kCand * 128, &tmHi, &bars[pFull0 + b], hh * 64, lit.gk, row);
          tma_load_3d(smem + L::lo(b) + hh * kCand * 128, &tmLo, &bars[pFull0 + b], hh * 64, lit.gk, row);
        }
      }
      __syncwarp();
      ++gl;
      if (++lc == lit.nch) {
        lid = next_item(lid + gridDim.x, lit);
        lc = 0;
      }
      return true;
    };
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmHi);
      prefetch_tmap(&tmLo);
    }
    GItem cur;
    int64_t id = next_item(blockIdx.x, cur);
    if (id < nitems) load_q(cur);
    __syncwarp();
    for (int q = 0; q < L::kBufs - 1; ++q) load_next();
    uint32_t gc = 0, qi = 0;
    const uint32_t idesc = idesc_bf16(kRows, kCand, false, false);
    while (id < nitems && ok) {
      GItem nxt = cur;
      int64_t nid = id;
      for (int c = 0; c < cur.nch && ok; ++c, ++gc) {
        const int b = (int)(gc % L::kBufs), tb = gc & 1;
        ok = mbar_wait_warp(&bars[pFull0 + b], (gc / L::kBufs) & 1, g.err);
        if (ok && c == 0) ok = mbar_wait_warp(&bars[pQFull], qi & 1, g.err);
        if (ok && gc >= 2) ok = mbar_wait_warp(&bars[pTFree0 + tb], ((gc >> 1) - 1) & 1, g.err);
        if (!ok) break;
        tc_fence_after();
        // N = 64 columns whatever the chunk's candidate count: columns past the candidates
        // (rows the copy brought in beyond them) are computed and never scanned
        const uint32_t sHi = smem_u32(smem + L::hi(b)), sLo = smem_u32(smem + L::lo(b));
        for (int hs = 0; hs < cur.nh; ++hs) {
          const uint32_t sQ = smem_u32(smem + L::kQ + hs * L::kQTile);
          const uint32_t td = tmem + (uint32_t)((hs * 2 + tb) * kCand);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
            const uint32_t boff = (kk >> 2) * (kCand * 128) + (kk & 3) * 32;
            const uint32_t ad = sdesc_lo(sQ + koff, 16);
            mma_ss_lo(td, ad, sdesc_lo(sHi + boff, 16), idesc, kk > 0 ? 1u : 0u);
            mma_ss_lo(td, ad, sdesc_lo(sLo + boff, 16), idesc, 1u);
          }
        }
        mma_commit_warp(&bars[pTFull0 + tb]);
        mma_commit_warp(&bars[pKFree0 + b]);
        const bool last = c + 1 == cur.nch;
        if (last) mma_commit_warp(&bars[pQFree]);
        // keep the copies two chunks ahead
        while (ok && gl <= gc + 2 && lid < nitems) ok = load_next();
        if (last) {
          nid = next_item(id + gridDim.x, nxt);
          if (ok && nid < nitems) {
            // the next item's Q tiles replace these once this item's MMAs and reads are done
            ok = mbar_wait_warp(&bars[pQFree], qi & 1, g.err) && mbar_wait_warp(&bars[pQRead], qi & 1, g.err);
            if (ok) load_q(nxt);
            __syncwarp();
          }
        }
      }
      ++qi;
      id = nid;
      cur = nxt;
    }
    mma_commit_warp(&bars[pDone]);
    mbar_wait_warp(&bars[pDone], 0, g.err);
  }
  __syncthreads();
  if (warp == kGrpEpiWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, kGrpTmemCols);
  }
}

// Kbar (fp32) -> bf16 hi = rn(x), lo = rn(x - hi), and each pooled key's squared norm.  One
// warp per (sequence, block, KV head) row of Kbar [num_seqs, MB, Hkv, D]; the norms go to
// kn2 [num_seqs, Hkv, MB], contiguous over the blocks that one gate item scans.
__global__ void kbar_split_kernel(const float* __restrict__ kbar, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo, float* __restrict__ kn2, Geom g) {
  const int lane = threadIdx.x & 31;
  const int64_t nrow = (int64_t)g.num_seqs * g.MB * g.Hkv;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < nrow; row += wstride) {
    const int64_t base = row * g.D;
    float ss = 0.f;
    for (int d = lane; d < g.D; d += 32) {
      const float x = kbar[base + d];
      const __nv_bfloat16 xh = __float2bfloat16_rn(x);
      hi[base + d] = xh;
      lo[base + d] = __float2bfloat16_rn(x - __bfloat162float(xh));
      ss = fmaf(x, x, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) {
      const int64_t hk = row % g.Hkv, sb = row / g.Hkv;  // sb = s * MB + b
      const int64_t s = sb / g.MB, b = sb - s * g.MB;
      kn2[(s * g.Hkv + hk) * g.MB + b] = ss;
    }
  }
}

template <int D, int kMaxM>
cudaError_t launch_group(const Geom& g, const CUtensorMap& tq, const CUtensorMap& th, const CUtensorMap& tl,
                         int32_t* sel, cudaStream_t st) {
  const int nhg = g.G / kGrpHeads;
  const int64_t nitems = (int64_t)g.MB * g.num_seqs * (g.bs / kRows) * g.Hkv * nhg;
  if (nitems == 0) return cudaSuccess;
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int smem = GrpLayout<D>::kAlloc;
  e = cudaFuncSetAttribute(gate_group_kernel<D, kMaxM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(nitems < nsm ? nitems : nsm);
  gate_group_kernel<D, kMaxM><<<grid, kGrpThreads, smem, st>>>(tq, th, tl, g, sel, nitems, nhg);
  return cudaGetLastError();
}

template <int D, int kMaxM>
cudaError_t launch_gate_d(const Geom& g, const __nv_bfloat16* Q, int32_t* sel, const Work& w, cudaStream_t st) {
  CUtensorMap tq, th, tl;
  cudaError_t e = make_rows_map(&tq, Q, (uint64_t)g.T, g.Hq, D, kRows);
  if (e != cudaSuccess) return e;
  const uint64_t nb = (uint64_t)g.num_seqs * g.MB;
  e = make_rows_map(&th, w.kbar_hi, nb, g.Hkv, D, kCand);
  if (e != cudaSuccess) return e;
  e = make_rows_map(&tl, w.kbar_lo, nb, g.Hkv, D, kCand);
  if (e != cudaSuccess) return e;
  // The exact selection (more than four blocks to choose) of query heads in KV groups of a
  // multiple of four runs on the group kernel: measured 3.7 -> 2.9 ms on the varlen workload
  // (top_k 12).  The quantized selection stays on the per-head kernel, which measured faster
  // wherever items have many chunks (8.4 against 10.3 ms at 1M, 59 against 78 ms at 10M).
  if constexpr (!RowTopK<kMaxM>::kQuant) {
    if (g.G % kGrpHeads == 0) return launch_group<D, kMaxM>(g, tq, th, tl, sel, st);
  }
  const int smem = GLayout<D>::kAlloc;
  e = cudaFuncSetAttribute(gate_tc_kernel<D, kMaxM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(g.MB * (g.bs / kRows)), (unsigned)g.num_seqs, (unsigned)g.Hq);
  gate_tc_kernel<D, kMaxM><<<grid, kThreads, smem, st>>>(tq, th, tl, g, w.kbar_n2, sel);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate(const Geom& g, const __nv_bfloat16* Q, const float* Kbar, int32_t* sel, const Work& w,
                        cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  const int64_t nrow = (int64_t)g.num_seqs * g.MB * g.Hkv;
  if (nrow > 0) {
    const int64_t want = (nrow + 7) / 8;  // eight rows (warps) per block
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    kbar_split_kernel<<<blocks, 256, 0, st>>>(Kbar, w.kbar_hi, w.kbar_lo, w.kbar_n2, g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int m = g.k - 1;
  if (g.D == 64) {
    if (m <= 2) return launch_gate_d<64, 2>(g, Q, sel, w, st);
    if (m <= 4) return launch_gate_d<64, 4>(g, Q, sel, w, st);
    if (m <= 8) return launch_gate_d<64, 8>(g, Q, sel, w, st);
    return launch_gate_d<64, kMaxTopK - 1>(g, Q, sel, w, st);
  }
  if (m <= 2) return launch_gate_d<128, 2>(g, Q, sel, w, st);
  if (m <= 4) return launch_gate_d<128, 4>(g, Q, sel, w, st);
  if (m <= 8) return launch_gate_d<128, 8>(g, Q, sel, w, st);
  return launch_gate_d<128, kMaxTopK - 1>(g, Q, sel, w, st);
}

}  // namespace moba
