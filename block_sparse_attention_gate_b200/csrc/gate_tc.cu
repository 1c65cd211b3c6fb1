// Parameter-free MoBA gate on the tensor cores: scores s = <q, Kbar[b]> for the strictly
// earlier blocks of the query's sequence, forced own block, top-(k-1) past blocks by
// descending score with ties to the lower block index.  (MoBA README, "Parameter-less
// Gating Mechanism" and the FAQ answer of GitHub issue #27: the own block is always taken
// and is not a candidate, k-1 more blocks come from earlier blocks; youleyou.com,
// "Kimi发布MoBA突破性实现无限上下文", section "PyTorch实现关键要点": score by the product of the
// query with the pooled keys, mask future blocks, top-k.)
//
// A CTA takes 128 consecutive tokens of one query head inside one query block i.  The
// candidate blocks 0..i-1 are processed in chunks of up to 64: the chunk's pooled keys,
// split into bf16 hi + lo parts (Kbar = hi + lo + O(2^-17 |Kbar|)), are staged by TMA and
// S = Q hi^T + Q lo^T accumulates in fp32 TMEM (double-buffered).  Thread r reads row r
// of S from TMEM and keeps a running top-(k-1) list in registers.
//
// Selection cost.  With at most four blocks to choose (top_k <= 5) a score is not inserted
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

constexpr int kThreads = 160;     // warps 0-3 epilogue, warp 4 TMA + MMA (whole warp)
constexpr int kRows = 128;        // query rows per CTA
// Candidate blocks per chunk and chunk buffers: one buffer of 64 keeps three CTAs per SM,
// which measured faster at 1M than two buffers (two CTAs per SM) or chunks of 32.
constexpr int kGateCand = 64;
constexpr int kGateBufs = 1;

// Shared memory: the Q tile and kBufs buffers of a chunk's pooled keys (hi then lo).
template <int D, int kCand, int kBufs>
struct GLayout {
  static constexpr int kQ = 0;                           // [128 x D] bf16
  static constexpr int kChunk = 2 * kCand * D * 2;       // hi [kCand x D] + lo [kCand x D] bf16
  static constexpr int kBuf0 = kQ + kRows * D * 2;
  static constexpr int kBar = kBuf0 + kBufs * kChunk;
  static constexpr int kAlloc = kBar + 128 + 1024;
  static constexpr uint32_t kTmemCols = 2 * kCand;       // double-buffered S
  __host__ __device__ static constexpr int hi(int b) { return kBuf0 + b * kChunk; }
  __host__ __device__ static constexpr int lo(int b) { return kBuf0 + b * kChunk + kCand * D * 2; }
};

enum GBar { kFull0 = 0, kFull1, kQFull, kKFree0, kKFree1, kTFull0, kTFull1, kTFree0, kTFree1, kGDone, kGNumBars };

__device__ __forceinline__ bool ranks_before(float sa, int32_t ba, float sb, int32_t bb) {
  return sa > sb || (sa == sb && ba < bb);
}

// kMaxM: compile-time capacity of the running top lists (>= top_k - 1), so the lists live
// in registers; kLists of them take interleaved candidates to shorten the dependency chain.
template <int D, int kMaxM, int kCand, int kBufs, int kLists = (kMaxM <= 8 ? 2 : 1)>
__global__ void __launch_bounds__(kThreads, kBufs == 1 ? 3 : 2)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmHi,
                   const __grid_constant__ CUtensorMap tmLo, Geom g, const float* __restrict__ kn2,
                   int32_t* __restrict__ sel) {
  using L = GLayout<D, kCand, kBufs>;
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
    mbar_init(&bars[kFull0], 1);
    mbar_init(&bars[kFull1], 1);
    mbar_init(&bars[kQFull], 1);
    mbar_init(&bars[kKFree0], 1);
    mbar_init(&bars[kKFree1], 1);
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
    // Chunk loop shared by both selection forms: scan(v, b0) takes the 32 scores of row r for
    // candidate blocks b0 .. b0 + 31 (columns at or past the query block i are not candidates).
    auto run_chunks = [&](auto&& scan) {
      for (int c = 0; c < nch && ok; ++c) {
        const int buf = c & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kTFull0 + buf], (c >> 1) & 1, g.err));
        if (!ok) break;
        tc_fence_after();
        const int c0 = c * kCand;
        const int ngrp = (min(kCand, i - c0) + 31) / 32;
        const uint32_t t0 = tmem + lane_off + buf * kCand;
        // The next group's TMEM load is in flight while the current group is scanned.
        uint32_t va[32], vb[32];
        tmem_ld32(t0, va);
        tmem_wait_ld(va);
        for (int gi = 0; gi < ngrp; gi += 2) {
          if (gi + 1 < ngrp) tmem_ld32(t0 + (gi + 1) * 32, vb);
          scan(va, c0 + gi * 32);
          if (gi + 1 < ngrp) {
            tmem_wait_ld(vb);
            if (gi + 2 < ngrp) tmem_ld32(t0 + (gi + 2) * 32, va);
            scan(vb, c0 + (gi + 1) * 32);
            if (gi + 2 < ngrp) tmem_wait_ld(va);
          }
        }
        tc_fence_before();
        mbar_arrive(&bars[kTFree0 + buf]);
      }
    };
    // Candidates reach a list in ascending block index, so a new one ranks after every
    // listed entry whose score is >= its own (ties go to the lower index) and before the
    // rest: the list shifts down by one from that position.  A score at or below the last
    // slot leaves the list unchanged, so the update needs no branch.  In a list, the first
    // kMaxM - m slots hold sentinels that rank before every score and are never displaced,
    // so the m live slots are the last m and the current m-th best is always the last slot.
    auto insert = [&](float (&ls)[kMaxM], int32_t (&lb)[kMaxM], float sc, int32_t b) {
      bool ge[kMaxM];
#pragma unroll
      for (int q = 0; q < kMaxM; ++q) ge[q] = ls[q] >= sc;
#pragma unroll
      for (int q = kMaxM - 1; q >= 1; --q) {
        ls[q] = ge[q] ? ls[q] : (ge[q - 1] ? sc : ls[q - 1]);
        lb[q] = ge[q] ? lb[q] : (ge[q - 1] ? b : lb[q - 1]);
      }
      ls[0] = ge[0] ? ls[0] : sc;
      lb[0] = ge[0] ? lb[0] : b;
    };
    auto write_out = [&](const int32_t (&lb)[kMaxM]) {
      if (ok && r < nrows) {
        int32_t* out = sel + ((int64_t)(q0 + r) * g.Hq + h) * g.k;
        out[0] = i;
#pragma unroll
        for (int q = 0; q < kMaxM; ++q)
          if (q >= kMaxM - m) out[1 + q - (kMaxM - m)] = lb[q];
        for (int q = 1 + m; q < g.k; ++q) out[q] = -1;
      }
    };

    if constexpr (kMaxM <= 4) {
      // ----------------------------------------------- quantized keys + min/max network
      // B^2 = |q|^2 max_{b<i} |Kbar[b]|^2: the candidates' squared norms by all 128 threads,
      // the query row's from its staged tile (rows are 128-byte swizzled: the sum of squares
      // does not depend on the order in which the row's 16-byte pieces are read).
      const float* kn = kn2 + ((int64_t)s * g.Hkv + gk) * g.MB;
      float kmax = 0.f;
      for (int b = r; b < i; b += kRows) kmax = fmaxf(kmax, kn[b]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      if (lane == 0) red[warp] = kmax;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      kmax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kQFull], 0, g.err));
      float qn = 0.f;
      if (ok) {
        const uint8_t* qrow = smem + L::kQ + r * 128;
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
      }
      // |s| <= B for every candidate, so s * scl lies in [-0.49, 0.49] (up to the scores' own
      // rounding); B == 0 (or a non-finite B) leaves every key at 1.5 + code: lowest blocks.
      const float bound = sqrtf(qn) * sqrtf(kmax);
      const float scl = (bound > 1e-30f && bound <= FLT_MAX) ? 0.49f / bound : 0.f;
      float ls[kMaxM];
      int32_t lb[kMaxM];
#pragma unroll
      for (int q = 0; q < kMaxM; ++q) {
        const bool live = q >= kMaxM - m;
        ls[q] = live ? 0.f : FLT_MAX;  // keys of real candidates are >= 1
        lb[q] = live ? INT32_MAX : -1;
      }
      auto scan_q = [&](const uint32_t (&v)[32], int32_t b0) {
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
        const int nv = i - b0;  // candidate columns in this group (the same for the whole CTA)
        if (nv < 32) {
#pragma unroll
          for (int x = 0; x < 32; ++x) key[x] = x < nv ? key[x] : 0.f;
        }
        float top[kMaxM];
        if constexpr (kMaxM == 2) {
          // Tournament: sorted pairs, then top-2 of two top-2 lists is
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
        // The group's best keys, best first, into the running list (grid value + block);
        // an equal grid value from a later group ranks after the listed one (lower block).
#pragma unroll
        for (int q = 0; q < kMaxM; ++q) {
          const uint32_t bits = __float_as_uint(top[q]);
          insert(ls, lb, __uint_as_float(bits & ~31u), b0 + 31 - (int32_t)(bits & 31u));
        }
      };
      run_chunks(scan_q);
      write_out(lb);
    } else {
      // ----------------------------------------------- exact scores, interleaved lists
      // kLists independent sorted lists (best first) of kMaxM slots each; candidate column x
      // of a 32-column group goes to list x % kLists, so kLists insertion chains run side by
      // side.
      float ts_[kLists][kMaxM];
      int32_t tb_[kLists][kMaxM];
#pragma unroll
      for (int j = 0; j < kLists; ++j)
#pragma unroll
        for (int q = 0; q < kMaxM; ++q) {
          const bool live = q >= kMaxM - m;
          ts_[j][q] = live ? -FLT_MAX : FLT_MAX;
          tb_[j][q] = live ? INT32_MAX : -1;
        }
      // Columns at or past the query block i score -FLT_MAX, which never enters a list; a
      // score at or below a list's last slot skips the insertion.
      auto scan = [&](const uint32_t (&v)[32], int32_t b0) {
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int32_t b = b0 + x;
          const float sc = b < i ? __uint_as_float(v[x]) : -FLT_MAX;
          if (sc > ts_[x % kLists][kMaxM - 1]) insert(ts_[x % kLists], tb_[x % kLists], sc, b);
        }
      };
      run_chunks(scan);
      // Fold lists 1.. into list 0 (entries are no longer in index order: full comparison).
#pragma unroll
      for (int j = 1; j < kLists; ++j)
#pragma unroll
        for (int p = 0; p < kMaxM; ++p) {
          if (p < kMaxM - m) continue;
          float sc = ts_[j][p];
          int32_t cb = tb_[j][p];
#pragma unroll
          for (int q = 0; q < kMaxM; ++q) {
            const bool take = ranks_before(sc, cb, ts_[0][q], tb_[0][q]);
            const float os = ts_[0][q];
            const int32_t ob = tb_[0][q];
            ts_[0][q] = take ? sc : os;
            tb_[0][q] = take ? cb : ob;
            sc = take ? os : sc;
            cb = take ? ob : cb;
          }
        }
      write_out(tb_[0]);
    }
  } else {
    // ========================================================= TMA + MMA issuer (warp 4)
    // The whole warp runs this loop: lane 0 issues the TMA copies, one elected lane the MMAs.
    auto load_chunk = [&](int c, bool with_q) {  // chunk c into buffer c % kBufs
      if (lane != 0) return;
      const int b = c % kBufs;
      if (with_q) {
        mbar_expect_tx(&bars[kQFull], kRows * D * 2);
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(smem + L::kQ + hh * kRows * 128, &tmQ, &bars[kQFull], hh * 64, h, q0);
      }
      // one box of kCand rows (rows past the candidates load too, and are never scanned)
      mbar_expect_tx(&bars[kFull0 + b], (uint32_t)L::kChunk);
      const int row = (int)(kb_row0 + c * kCand);
      for (int hh = 0; hh < D / 64; ++hh) {
        tma_load_3d(smem + L::hi(b) + hh * kCand * 128, &tmHi, &bars[kFull0 + b], hh * 64, gk, row);
        tma_load_3d(smem + L::lo(b) + hh * kCand * 128, &tmLo, &bars[kFull0 + b], hh * 64, gk, row);
      }
    };
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmHi);
      prefetch_tmap(&tmLo);
    }
    for (int c = 0; c < kBufs && c < nch; ++c) load_chunk(c, c == 0);
    __syncwarp();
    const uint32_t sQ = smem_u32(smem + L::kQ);
    for (int c = 0; c < nch && ok; ++c) {
      const int buf = c & 1;        // TMEM buffer
      const int kb = c % kBufs;     // key buffer
      ok = mbar_wait_warp(&bars[kFull0 + kb], (c / kBufs) & 1, g.err);
      if (ok && c == 0) ok = mbar_wait_warp(&bars[kQFull], 0, g.err);
      if (ok && c >= 2) ok = mbar_wait_warp(&bars[kTFree0 + buf], ((c >> 1) - 1) & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      const int ncand = min(kCand, i - c * kCand);
      const int n = (ncand + 15) & ~15;
      const uint32_t idesc = idesc_bf16(kRows, n, false, false);
      const uint32_t sHi = smem_u32(smem + L::hi(kb));
      const uint32_t sLo = smem_u32(smem + L::lo(kb));
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
        const uint32_t boff = (kk >> 2) * (kCand * 128) + (kk & 3) * 32;
        const uint64_t ad = sdesc_sw128(sQ + koff, 16, 1024);
        mma_bf16_ss_warp(tmem + buf * kCand, ad, sdesc_sw128(sHi + boff, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        mma_bf16_ss_warp(tmem + buf * kCand, ad, sdesc_sw128(sLo + boff, 16, 1024), idesc, 1u);
      }
      mma_commit_warp(&bars[kTFull0 + buf]);
      if (c + kBufs < nch) {  // the key buffer takes chunk c + kBufs once these MMAs have read it
        mma_commit_warp(&bars[kKFree0 + kb]);
        ok = mbar_wait_warp(&bars[kKFree0 + kb], (c / kBufs) & 1, g.err);
        if (!ok) break;
        load_chunk(c + kBufs, false);
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

// Kbar (fp32) -> bf16 hi = rn(x), lo = rn(x - hi), and each pooled key's squared norm.  One
// warp per (sequence, block, KV head) row of Kbar [num_seqs, MB, Hkv, D]; the norms go to
// kn2 [num_seqs, Hkv, MB], contiguous over the blocks that one gate CTA scans.
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
cudaError_t launch_gate_d(const Geom& g, const __nv_bfloat16* Q, int32_t* sel, const Work& w, cudaStream_t st) {
  constexpr int kCand = kGateCand, kBufs = kGateBufs;
  CUtensorMap tq, th, tl;
  cudaError_t e = make_rows_map(&tq, Q, (uint64_t)g.T, g.Hq, D, kRows);
  if (e != cudaSuccess) return e;
  const uint64_t nb = (uint64_t)g.num_seqs * g.MB;
  e = make_rows_map(&th, w.kbar_hi, nb, g.Hkv, D, kCand);
  if (e != cudaSuccess) return e;
  e = make_rows_map(&tl, w.kbar_lo, nb, g.Hkv, D, kCand);
  if (e != cudaSuccess) return e;
  const int smem = GLayout<D, kCand, kBufs>::kAlloc;
  e = cudaFuncSetAttribute(gate_tc_kernel<D, kMaxM, kCand, kBufs>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(g.MB * (g.bs / kRows)), (unsigned)g.num_seqs, (unsigned)g.Hq);
  gate_tc_kernel<D, kMaxM, kCand, kBufs><<<grid, kThreads, smem, st>>>(tq, th, tl, g, w.kbar_n2, sel);
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
