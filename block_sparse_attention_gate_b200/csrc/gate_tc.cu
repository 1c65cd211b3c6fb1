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
// of S from TMEM and keeps a sorted running top-(k-1) list in registers.
#include <cudaTypedefs.h>
#include <float.h>

#include "moba_internal.cuh"
#include "sm100.cuh"

namespace moba {


namespace {

constexpr int kThreads = 160;     // warps 0-3 epilogue, warp 4 TMA + MMA (whole warp)
constexpr int kRows = 128;        // query rows per CTA
constexpr int kCand = 64;         // candidate blocks per chunk (three CTAs per SM)
constexpr int kBoxRows = 64;      // candidate rows per TMA box
constexpr uint32_t kTmemCols = 128;

template <int D>
struct GLayout {
  static constexpr int kQ = 0;                       // [128 x D] bf16
  static constexpr int kHi = kQ + kRows * D * 2;     // [kCand x D] bf16
  static constexpr int kLo = kHi + kCand * D * 2;    // [kCand x D] bf16
  static constexpr int kBar = kLo + kCand * D * 2;
  static constexpr int kAlloc = kBar + 128 + 1024;
};

enum GBar { kFull = 0, kKFree, kTFull0, kTFull1, kTFree0, kTFree1, kGDone, kGNumBars };

__device__ __forceinline__ bool ranks_before(float sa, int32_t ba, float sb, int32_t bb) {
  return sa > sb || (sa == sb && ba < bb);
}

// kMaxM: compile-time capacity of the running top lists (>= top_k - 1), so the lists live
// in registers; kLists of them take interleaved candidates to shorten the dependency chain.
template <int D, int kMaxM, int kLists = (kMaxM <= 4 ? 4 : (kMaxM <= 8 ? 2 : 1))>
__global__ void __launch_bounds__(kThreads, 3)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmHi,
                   const __grid_constant__ CUtensorMap tmLo, Geom g, int32_t* __restrict__ sel) {
  using L = GLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kGNumBars * 8);
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
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    mbar_init(&bars[kFull], 1);
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
    // kLists independent sorted lists (best first) of kMaxM slots each; candidate column x
    // of a 32-column group goes to list x % kLists, so kLists insertion chains run side by
    // side.  In each list the first kMaxM - m slots hold sentinels that rank before every
    // score and are never displaced, so the m live slots are the last m and the current
    // m-th best is always the last slot (no runtime indexing).
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
    // Candidates reach a list in ascending block index, so a new one ranks after every
    // listed entry whose score is >= its own (ties go to the lower index) and before the
    // rest: the list shifts down by one from that position.  A score at or below the last
    // slot leaves the list unchanged, so the update needs no branch.
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
    // One 32-column group of S; columns at or past the query block i score -FLT_MAX, which
    // never enters a list.
    auto scan = [&](const uint32_t (&v)[32], int32_t b0) {
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int32_t b = b0 + x;
        const float sc = b < i ? __uint_as_float(v[x]) : -FLT_MAX;
        if constexpr (kMaxM <= 4) {
          insert(ts_[x % kLists], tb_[x % kLists], sc, b);
        } else {
          if (sc > ts_[x % kLists][kMaxM - 1]) insert(ts_[x % kLists], tb_[x % kLists], sc, b);
        }
      }
    };
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
    if (ok && r < nrows) {
      int32_t* out = sel + ((int64_t)(q0 + r) * g.Hq + h) * g.k;
      out[0] = i;
#pragma unroll
      for (int q = 0; q < kMaxM; ++q)
        if (q >= kMaxM - m) out[1 + q - (kMaxM - m)] = tb_[0][q];
      for (int q = 1 + m; q < g.k; ++q) out[q] = -1;
    }
  } else {
    // ========================================================= TMA + MMA issuer (warp 4)
    // The whole warp runs this loop: lane 0 issues the TMA copies, one elected lane the MMAs.
    auto load_chunk = [&](int c, bool with_q) {
      if (lane != 0) return;
      const int c0 = c * kCand;
      const int ncand = min(kCand, i - c0);
      const int nbox = (ncand + kBoxRows - 1) / kBoxRows;
      uint32_t bytes = (uint32_t)nbox * kBoxRows * D * 2 * 2;
      if (with_q) bytes += kRows * D * 2;
      mbar_expect_tx(&bars[kFull], bytes);
      if (with_q)
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(smem + L::kQ + hh * kRows * 128, &tmQ, &bars[kFull], hh * 64, h, q0);
      for (int bx = 0; bx < nbox; ++bx)
        for (int hh = 0; hh < D / 64; ++hh) {
          const int row = (int)(kb_row0 + c0 + bx * kBoxRows);
          const int off = hh * kCand * 128 + bx * kBoxRows * 128;
          tma_load_3d(smem + L::kHi + off, &tmHi, &bars[kFull], hh * 64, gk, row);
          tma_load_3d(smem + L::kLo + off, &tmLo, &bars[kFull], hh * 64, gk, row);
        }
    };
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmHi);
      prefetch_tmap(&tmLo);
    }
    load_chunk(0, true);
    __syncwarp();
    const uint32_t sQ = smem_u32(smem + L::kQ);
    const uint32_t sHi = smem_u32(smem + L::kHi);
    const uint32_t sLo = smem_u32(smem + L::kLo);
    for (int c = 0; c < nch && ok; ++c) {
      const int buf = c & 1;
      ok = mbar_wait_warp(&bars[kFull], c & 1, g.err);
      if (ok && c >= 2) ok = mbar_wait_warp(&bars[kTFree0 + buf], ((c >> 1) - 1) & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      const int ncand = min(kCand, i - c * kCand);
      const int n = (ncand + 15) & ~15;
      const uint32_t idesc = idesc_bf16(kRows, n, false, false);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
        const uint32_t boff = (kk >> 2) * (kCand * 128) + (kk & 3) * 32;
        const uint64_t ad = sdesc_sw128(sQ + koff, 16, 1024);
        mma_bf16_ss_warp(tmem + buf * kCand, ad, sdesc_sw128(sHi + boff, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        mma_bf16_ss_warp(tmem + buf * kCand, ad, sdesc_sw128(sLo + boff, 16, 1024), idesc, 1u);
      }
      mma_commit_warp(&bars[kTFull0 + buf]);
      if (c + 1 < nch) {
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
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Kbar (fp32) -> bf16 hi = rn(x), lo = rn(x - hi).
__global__ void kbar_split_kernel(const float* __restrict__ kbar, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo, int64_t n) {
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
    const float x = kbar[idx];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[idx] = h;
    lo[idx] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
}

template <int D, int kMaxM>
cudaError_t launch_gate_d(const Geom& g, const __nv_bfloat16* Q, int32_t* sel, const Work& w, cudaStream_t st) {
  CUtensorMap tq, th, tl;
  cudaError_t e = make_rows_map(&tq, Q, (uint64_t)g.T, g.Hq, D, kRows);
  if (e != cudaSuccess) return e;
  const uint64_t nb = (uint64_t)g.num_seqs * g.MB;
  e = make_rows_map(&th, w.kbar_hi, nb, g.Hkv, D, kBoxRows);
  if (e != cudaSuccess) return e;
  e = make_rows_map(&tl, w.kbar_lo, nb, g.Hkv, D, kBoxRows);
  if (e != cudaSuccess) return e;
  const int smem = GLayout<D>::kAlloc;
  e = cudaFuncSetAttribute(gate_tc_kernel<D, kMaxM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(g.MB * (g.bs / kRows)), (unsigned)g.num_seqs, (unsigned)g.Hq);
  gate_tc_kernel<D, kMaxM><<<grid, kThreads, smem, st>>>(tq, th, tl, g, sel);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate(const Geom& g, const __nv_bfloat16* Q, const float* Kbar, int32_t* sel, const Work& w,
                        cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  const int64_t n = (int64_t)g.num_seqs * g.MB * g.Hkv * g.D;
  if (n > 0) {
    const int64_t want = (n + 255) / 256;
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    kbar_split_kernel<<<blocks, 256, 0, st>>>(Kbar, w.kbar_hi, w.kbar_lo, n);
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
