// MoBA backward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// MoBA is trained through its block attention (MoBA README, "Trainable Block Sparse
// Attention"); its gate has no parameters ("Parameter-less Gating Mechanism"), so the
// top-k selection is held fixed and the gradient flows through masked softmax attention
// under MoBA's mask (keys of the selected blocks, causal inside the own block).  With the
// forward's LSE known, for a query row p and an attended key j:
//   P = exp(scale <q_p, k_j> - LSE_p),  dP = <dO_p, v_j>,  Dp = <dO_p, O_p>,
//   dS = P (dP - Dp),  dQ_p = scale sum_j dS k_j,  dK_j = scale sum_p dS q_p,
//   dV_j = sum_p P dO_p   (dK, dV summed over the query heads of a KV group).
// The work follows the forward's split (youleyou.com, "Kimi发布MoBA突破性实现无限上下文",
// section "PyTorch实现关键要点": attention over the own block and over the chosen blocks
// separately):
//   bwd_prep_kernel  : Dp = rowsum(dO * O) for every (token, query head).
//   bwd_dq_kernel    : query-row centric, like the forward kernel.  past mode: two tiles of
//                      128 routed rows of one bucket walk the block's keys in 64-key chunks
//                      (S = Q K^T and dP = dO V^T into TMEM, dS in registers written back
//                      as bf16, dQ += dS K accumulated in TMEM) and write one fp32 dQ
//                      partial per routed slot.  own mode: two tiles of 128 tokens walk the
//                      own block causally and add the row's past partials: the final dQ.
//   bwd_dkdv_kernel  : key centric.  A CTA owns 128 keys of one block (one KV head) and
//                      walks every query row that attends them in 64-row sub-tiles: the
//                      bucket's routed rows (the rows that chose the block) and the own
//                      block's later rows of all the group's heads (causal).  S^T = K Q^T
//                      and dP^T = V dO^T go to TMEM (double-buffered), P^T and dS^T come
//                      back as bf16, dV += P^T dO and dK += dS^T Q accumulate in TMEM for
//                      the whole walk, so every dK/dV row is written once, without atomics.
#include <cudaTypedefs.h>
#include <float.h>

#include "moba_internal.cuh"
#include "sm100.cuh"

namespace moba {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ Dp = rowsum(dO * O)
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ O,
                                                       const __nv_bfloat16* __restrict__ dO,
                                                       float* __restrict__ Dp, int64_t rows, int D) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows; row += warps) {
    float acc = 0.f;
    for (int d = lane * 2; d < D; d += 64) {
      const float2 o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(O + row * D + d));
      const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dO + row * D + d));
      acc = fmaf(o.x, g.x, fmaf(o.y, g.y, acc));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) Dp[row] = acc;
  }
}

struct BwdArgs {
  Geom g;
  const __nv_bfloat16* Q;
  const __nv_bfloat16* dO;
  const float* LSE;
  const float* Dp;
  const int32_t* sel;
  const int32_t* counts;
  const int32_t* tile_off;
  const int32_t* tile_bucket;
  const int32_t* rows;
  float* dq_part;       // [R, D] fp32 dQ partial of each routed slot
  __nv_bfloat16* dQ;    // [T, Hq, D]
  __nv_bfloat16* dK;    // [T, Hkv, D]
  __nv_bfloat16* dV;    // [T, Hkv, D]
  int own_head_pairs;
};

// =====================================================================================
// dQ kernel
// =====================================================================================
constexpr int kQThreads = 320;   // warps 0-3 rows of tile 0, 4-7 of tile 1, 8 TMA, 9 MMA
constexpr int kQRows = 128;      // query rows per tile (M), two tiles per CTA
constexpr int kQBN = 64;         // keys per chunk
constexpr uint32_t kQColS = 0;     // S_t at 64 t (dS_t, bf16 pairs, over its first 32 columns)
constexpr uint32_t kQColDP = 128;  // dP_t at 128 + 64 t
constexpr uint32_t kQColDQ = 256;  // dQ_t at 256 + 128 t

template <int D>
struct QLayout {
  static constexpr int kTile = kQRows * D * 2;   // [128 x D] bf16
  static constexpr int kChunk = kQBN * D * 2;    // [64 x D] bf16
  static constexpr int kQ = 0;                   // two tiles
  static constexpr int kDO = kQ + 2 * kTile;     // two tiles
  static constexpr int kK0 = kDO + 2 * kTile;    // two stages
  static constexpr int kV0 = kK0 + 2 * kChunk;   // two stages
  static constexpr int kBar = kV0 + 2 * kChunk;
  static constexpr int kBytes = kBar + 256;
  // at least 120 KB, so one CTA per SM: each CTA holds all 512 TMEM columns
  static constexpr int kAlloc = kBytes + 1024 > 120 * 1024 ? kBytes + 1024 : 120 * 1024;
};

enum QBar { qQFull = 0, qKVFull0, qKVFull1, qKVEmpty0, qKVEmpty1, qSFull0, qSFull1, qPFull0, qPFull1,
            qDQFull0, qDQFull1, qDone, qNumBars };

template <int D, bool kOwn>
__global__ void __launch_bounds__(kQThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, BwdArgs a) {
  using L = QLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + qNumBars * 8);
  const Geom& g = a.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ------------------------------------------------------------- work item
  int gk, s, i_blk = 0, nchunks;
  int32_t key0;
  int32_t row_start[2] = {0, 0};  // past: first routed slot of each tile
  int32_t q0[2] = {0, 0}, hd[2] = {0, 0}, nrows[2] = {0, 0}, tok_off[2] = {0, 0};
  if constexpr (!kOwn) {
    const int32_t tile = (int32_t)blockIdx.x;
    const int32_t total = __ldg(a.tile_off + g.nbk);
    const int64_t lo = __ldg(a.tile_bucket + tile);
    if (tile >= total) return;
    const int32_t b = (int32_t)(lo % g.MB);
    s = (int)((lo / g.MB) % g.num_seqs);
    gk = (int)(lo / ((int64_t)g.MB * g.num_seqs));
    row_start[0] = tile * kPastTileRows;
    row_start[1] = tile * kPastTileRows + kQRows;
    key0 = seq_start(g, s) + b * g.bs;
    nchunks = g.bs / kQBN;
  } else {
    const int per_blk = g.bs / kQRows;
    s = blockIdx.y;
    const int32_t ts = seq_start(g, s), te = seq_end(g, s);
    int last_tile;  // the furthest query tile: keys up to its end
    if (a.own_head_pairs) {
      i_blk = blockIdx.x / per_blk;
      const int qt = blockIdx.x - i_blk * per_blk;
      const int32_t t0 = ts + i_blk * g.bs + qt * kQRows;
      if (t0 >= te) return;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        hd[t] = 2 * blockIdx.z + t;
        q0[t] = t0;
        nrows[t] = min(kQRows, te - t0);
        tok_off[t] = qt * kQRows;
      }
      last_tile = qt;
    } else {
      const int pairs = (per_blk + 1) / 2;
      i_blk = blockIdx.x / pairs;
      const int qp = blockIdx.x - i_blk * pairs;
      const int32_t t0 = ts + i_blk * g.bs + 2 * qp * kQRows;
      if (t0 >= te) return;
      const bool has1 = 2 * qp + 1 < per_blk && t0 + kQRows < te;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        hd[t] = blockIdx.z;
        q0[t] = t0 + t * kQRows;
        nrows[t] = (t == 0 || has1) ? max(0, min(kQRows, te - q0[t])) : 0;
        tok_off[t] = (2 * qp + t) * kQRows;
      }
      last_tile = has1 ? 2 * qp + 1 : 2 * qp;
    }
    gk = hd[0] / g.G;
    key0 = ts + i_blk * g.bs;
    nchunks = (last_tile + 1) * (kQRows / kQBN);
  }

  // ------------------------------------------------------------- early loads (past mode)
  int32_t e = -1;
  if (!kOwn && warp < 8) {
    const int t = warp >> 2, r = tid & (kQRows - 1);
    e = __ldg(a.rows + row_start[t] + r);
    const int64_t qrow = e >= 0 ? e / (g.k - 1) : -1;
    const __nv_bfloat16* srcq = qrow >= 0 ? a.Q + qrow * D : a.Q;
    const __nv_bfloat16* srcg = qrow >= 0 ? a.dO + qrow * D : a.dO;
    const uint32_t nb = qrow >= 0 ? 16u : 0u;
    const uint32_t sQ = smem_u32(smem + L::kQ + t * L::kTile);
    const uint32_t sG = smem_u32(smem + L::kDO + t * L::kTile);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      cp_async_16(sQ + sw128_offset(r, c, kQRows), srcq + c * 8, nb);
      cp_async_16(sG + sw128_offset(r, c, kQRows), srcg + c * 8, nb);
    }
  }

  // ------------------------------------------------------------- setup
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    mbar_init(&bars[qQFull], kOwn ? 1 : 2 * kQRows);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bars[qKVFull0 + q], 1);
      mbar_init(&bars[qKVEmpty0 + q], 1);
      mbar_init(&bars[qSFull0 + q], 1);
      mbar_init(&bars[qPFull0 + q], kQRows);
      mbar_init(&bars[qDQFull0 + q], 1);
    }
    mbar_init(&bars[qDone], 1);
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp < 8) {
    // ========================================================= rows: P, dS, epilogue
    const int t = warp >> 2;
    const int r = tid & (kQRows - 1);
    int64_t qrow = -1;
    if constexpr (kOwn) {
      if (r < nrows[t]) qrow = (int64_t)(q0[t] + r) * g.Hq + hd[t];
    } else {
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(&bars[qQFull]);
      if (e >= 0) qrow = e / (g.k - 1);
    }
    const float lse2 = qrow >= 0 ? __ldg(a.LSE + qrow) * kLog2e : INFINITY;  // +inf: the row is empty
    const float dpv = qrow >= 0 ? __ldg(a.Dp + qrow) : 0.f;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + kQColS + t * kQBN;
    const uint32_t tDP = tmem + lane_off + kQColDP + t * kQBN;
    const uint32_t tDQ = tmem + lane_off + kQColDQ + t * 128;
    const float c2 = g.scale_log2;
    const int row_in_blk = tok_off[t] + r;  // own mode: the row's position inside its block
    for (int j = 0; j < nchunks && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[qSFull0 + t], j & 1, g.err));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[2][32], dv[2][32];
      tmem_ld32(tS, sv[0]);
      tmem_ld32(tS + 32, sv[1]);
      tmem_ld32(tDP, dv[0]);
      tmem_ld32(tDP + 32, dv[1]);
      tmem_wait_ld();
      // own mode: key (j * 64 + x) of the block is visible to the row iff it is <= its position
      const int lim = kOwn ? min(kQBN, max(0, row_in_blk - j * kQBN + 1)) : kQBN;
      uint32_t pk[32];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const int c = h2 * 32 + x;
          float p0 = ex2(fmaf(__uint_as_float(sv[h2][x]), c2, -lse2));
          float p1 = ex2(fmaf(__uint_as_float(sv[h2][x + 1]), c2, -lse2));
          if (c >= lim) p0 = 0.f;
          if (c + 1 >= lim) p1 = 0.f;
          const float d0 = p0 * (__uint_as_float(dv[h2][x]) - dpv);
          const float d1 = p1 * (__uint_as_float(dv[h2][x + 1]) - dpv);
          pk[16 * h2 + (x >> 1)] = pack_bf16x2(d0, d1);
        }
      tmem_st32(tS, pk);  // dS (bf16 pairs) over the first 32 columns of S
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[qPFull0 + t]);
    }
    // ------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[qDQFull0 + t], 0, g.err));
    if (ok) {
      tc_fence_after();
      // own mode: the row's past partials.  The chosen past blocks fill slots 1..np of the
      // row (the selection's padding is at the end), so partial q has the id row*(k-1) + q.
      int np = 0;
      const int64_t pbase = qrow >= 0 ? qrow * (g.k - 1) : 0;
      if constexpr (kOwn) {
        if (qrow >= 0) {
          bool run = true;
#pragma unroll
          for (int q = 0; q < kMaxTopK - 1; ++q) {
            const int32_t b = q + 1 < g.k ? __ldg(a.sel + qrow * g.k + q + 1) : -1;
            run = run && b >= 0 && b < i_blk;
            np += run ? 1 : 0;
          }
        }
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tDQ + c * 32, o);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] = __uint_as_float(o[x]) * g.scale;
        if constexpr (kOwn) {
          for (int q = 0; q < np; ++q) {
            const float4* src = reinterpret_cast<const float4*>(a.dq_part + (pbase + q) * D + c * 32);
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const float4 f = __ldg(src + x);
              v[4 * x] += f.x;
              v[4 * x + 1] += f.y;
              v[4 * x + 2] += f.z;
              v[4 * x + 3] += f.w;
            }
          }
          if (qrow >= 0) {
            uint4* dst = reinterpret_cast<uint4*>(a.dQ + qrow * D + c * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_uint4(pack_bf16x2(v[8 * x], v[8 * x + 1]), pack_bf16x2(v[8 * x + 2], v[8 * x + 3]),
                                  pack_bf16x2(v[8 * x + 4], v[8 * x + 5]), pack_bf16x2(v[8 * x + 6], v[8 * x + 7]));
          }
        } else {
          if (e >= 0) {
            float4* dst = reinterpret_cast<float4*>(a.dq_part + (int64_t)e * D + c * 32);
#pragma unroll
            for (int x = 0; x < 8; ++x) dst[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
          }
        }
      }
    }
  } else if (warp == 8) {
    // ========================================================= TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if constexpr (kOwn) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmDO);
        mbar_expect_tx(&bars[qQFull], 4 * L::kTile);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh) {
            tma_load_3d(smem + L::kQ + t * L::kTile + hh * kQRows * 128, &tmQ, &bars[qQFull], hh * 64, hd[t], q0[t]);
            tma_load_3d(smem + L::kDO + t * L::kTile + hh * kQRows * 128, &tmDO, &bars[qQFull], hh * 64, hd[t],
                        q0[t]);
          }
      }
      for (int j = 0; j < nchunks && ok; ++j) {
        const int st = j & 1, u = j >> 1;
        if (u > 0) ok = mbar_wait(&bars[qKVEmpty0 + st], (u - 1) & 1, g.err);
        if (!ok) break;
        const int tok = key0 + j * kQBN;
        mbar_expect_tx(&bars[qKVFull0 + st], 2 * L::kChunk);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh) {
          tma_load_3d(smem + L::kK0 + st * L::kChunk + hh * kQBN * 128, &tmK, &bars[qKVFull0 + st], hh * 64, gk, tok);
          tma_load_3d(smem + L::kV0 + st * L::kChunk + hh * kQBN * 128, &tmV, &bars[qKVFull0 + st], hh * 64, gk, tok);
        }
      }
    }
  } else {
    // ========================================================= MMA issuer (warp 9)
    constexpr uint32_t idS = idesc_bf16(kQRows, kQBN, false, false);
    constexpr uint32_t idQ = idesc_bf16(kQRows, D, false, true);
    const uint32_t sQ = smem_u32(smem + L::kQ);
    const uint32_t sG = smem_u32(smem + L::kDO);
    const uint32_t sK0 = smem_u32(smem + L::kK0);
    const uint32_t sV0 = smem_u32(smem + L::kV0);
    auto issue_s = [&](int t, int j) {  // S_t = Q_t K_j^T and dP_t = dO_t V_j^T
      const uint32_t qb = sQ + t * L::kTile, gb = sG + t * L::kTile;
      const uint32_t kb = sK0 + (j & 1) * L::kChunk, vb = sV0 + (j & 1) * L::kChunk;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t aoff = (kk >> 2) * (kQRows * 128) + (kk & 3) * 32;
        const uint32_t boff = (kk >> 2) * (kQBN * 128) + (kk & 3) * 32;
        mma_bf16_ss_warp(tmem + kQColS + t * kQBN, sdesc_sw128(qb + aoff, 16, 1024), sdesc_sw128(kb + boff, 16, 1024),
                         idS, kk > 0 ? 1u : 0u);
        mma_bf16_ss_warp(tmem + kQColDP + t * kQBN, sdesc_sw128(gb + aoff, 16, 1024),
                         sdesc_sw128(vb + boff, 16, 1024), idS, kk > 0 ? 1u : 0u);
      }
      mma_commit_warp(&bars[qSFull0 + t]);
    };
    auto issue_dq = [&](int t, int j) {  // dQ_t += dS_t K_j (dS from TMEM)
      const uint32_t kb = sK0 + (j & 1) * L::kChunk;
#pragma unroll
      for (int kk = 0; kk < kQBN / 16; ++kk)
        mma_bf16_ts_warp(tmem + kQColDQ + t * 128, tmem + kQColS + t * kQBN + kk * 8,
                         sdesc_sw128(kb + kk * 2048, kQBN * 128, 1024), idQ, (j > 0 || kk > 0) ? 1u : 0u);
    };
    ok = mbar_wait_warp(&bars[qQFull], 0, g.err) && mbar_wait_warp(&bars[qKVFull0], 0, g.err);
    if (ok) {
      tc_fence_after();
      issue_s(0, 0);
      issue_s(1, 0);
    }
    for (int j = 0; j < nchunks && ok; ++j) {
      const bool more = j + 1 < nchunks;
      ok = mbar_wait_warp(&bars[qPFull0], j & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      issue_dq(0, j);
      if (!more) mma_commit_warp(&bars[qDQFull0]);
      if (more) {
        ok = mbar_wait_warp(&bars[qKVFull0 + ((j + 1) & 1)], ((j + 1) >> 1) & 1, g.err);
        if (!ok) break;
        tc_fence_after();
        issue_s(0, j + 1);
      }
      ok = mbar_wait_warp(&bars[qPFull1], j & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      issue_dq(1, j);
      mma_commit_warp(&bars[qKVEmpty0 + (j & 1)]);
      if (!more) mma_commit_warp(&bars[qDQFull1]);
      if (more) issue_s(1, j + 1);
    }
    mma_commit_warp(&bars[qDone]);
    mbar_wait_warp(&bars[qDone], 0, g.err);
  }

  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =====================================================================================
// dK / dV kernel
// =====================================================================================
constexpr int kKVThreads = 288;  // warps 0-3 keys (TMEM lanes), 4-7 row gather, 8 TMA + MMA
constexpr int kKeys = 128;       // keys per CTA (M)
constexpr int kSub = 64;         // query rows per sub-tile (N of S^T)
constexpr int kStages = 4;       // gathered sub-tiles in flight
constexpr uint32_t kKColS = 0;     // S^T of buffer b at 64 b (P^T over its first 32 columns, dS^T over the next 32)
constexpr uint32_t kKColDP = 128;  // dP^T of buffer b at 128 + 64 b
constexpr uint32_t kKColDV = 256;  // dV, then dK at 256 + D

template <int D>
struct KVLayout {
  static constexpr int kTile = kKeys * D * 2;   // [128 x D]
  static constexpr int kSubT = kSub * D * 2;    // [64 x D]
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ0 = kV + kTile;              // kStages stages
  static constexpr int kG0 = kQ0 + kStages * kSubT;   // kStages stages
  static constexpr int kLse = kG0 + kStages * kSubT;  // [kStages][64] fp32 (natural-log LSE)
  static constexpr int kDp = kLse + kStages * kSub * 4;
  static constexpr int kBar = kDp + kStages * kSub * 4;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024 > 120 * 1024 ? kBytes + 1024 : 120 * 1024;  // one CTA per SM
};

enum KBar { kbKVFull = 0, kbStFull0, kbStFree0 = kbStFull0 + kStages, kbSFull0 = kbStFree0 + kStages, kbSFull1,
            kbPFull0, kbPFull1, kbDone, kbNumBars };

// Rows of sub-tile n of a dK/dV CTA: the bucket's routed rows first, then the own block's
// rows (per query head of the group, 64 tokens at a time, from the key tile onward).
struct KVWalk {
  int32_t slot0;     // first routed slot of the bucket
  int32_t n_routed;  // routed rows
  int n_rsub;        // routed sub-tiles
  int32_t tok0;      // first own token that can see the key tile
  int32_t tok_end;   // end of the own block's tokens
  int n_osub_h;      // own sub-tiles per query head
  int total;         // all sub-tiles
};

// Row r of sub-tile n: the (token, head) row of Q/dO/LSE, or -1 for an empty slot.
// own_sub: -1 for routed sub-tiles, else the index of the 64-token step inside the head.
__device__ __forceinline__ int64_t kv_row(const Geom& g, const int32_t* rows, const KVWalk& w, int gk, int n, int r,
                                         int* own_sub) {
  if (n < w.n_rsub) {
    *own_sub = -1;
    const int32_t idx = n * kSub + r;
    if (idx >= w.n_routed) return -1;
    const int32_t e = __ldg(rows + w.slot0 + idx);
    return e >= 0 ? (int64_t)(e / (g.k - 1)) : -1;
  }
  const int o = n - w.n_rsub;
  const int hh = o / w.n_osub_h, sub = o - hh * w.n_osub_h;
  *own_sub = sub;
  const int32_t t = w.tok0 + sub * kSub + r;
  if (t >= w.tok_end) return -1;
  return (int64_t)t * g.Hq + gk * g.G + hh;
}

template <int D>
__global__ void __launch_bounds__(kKVThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, BwdArgs a) {
  using L = KVLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kbNumBars * 8);
  float* s_lse = reinterpret_cast<float*>(smem + L::kLse);
  float* s_dp = reinterpret_cast<float*>(smem + L::kDp);
  const Geom& g = a.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ------------------------------------------------------------- work item
  // Blocks in ascending order, so the CTAs of early blocks (which later queries may choose,
  // hence the larger buckets) start first; inside a block: sequence, KV head, key tile.
  const int per_blk = g.bs / kKeys;
  int64_t idx = blockIdx.x;
  const int kt = (int)(idx % per_blk);
  idx /= per_blk;
  const int gk = (int)(idx % g.Hkv);
  idx /= g.Hkv;
  const int s = (int)(idx % g.num_seqs);
  const int b = (int)(idx / g.num_seqs);
  const int32_t ts = seq_start(g, s), te = seq_end(g, s);
  const int32_t blk0 = ts + b * g.bs;
  const int32_t key0 = blk0 + kt * kKeys;
  if (key0 >= te) return;
  const int32_t blk_end = min(blk0 + g.bs, te);
  KVWalk w;
  w.slot0 = 0;
  w.n_routed = 0;
  if (g.k > 1) {
    const int64_t bk = ((int64_t)gk * g.num_seqs + s) * g.MB + b;
    w.n_routed = __ldg(a.counts + bk);
    w.slot0 = __ldg(a.tile_off + bk) * kPastTileRows;
  }
  w.n_rsub = (w.n_routed + kSub - 1) / kSub;
  w.tok0 = key0;
  w.tok_end = blk_end;
  w.n_osub_h = (blk_end - key0 + kSub - 1) / kSub;
  w.total = w.n_rsub + g.G * w.n_osub_h;

  // ------------------------------------------------------------- setup
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    mbar_init(&bars[kbKVFull], 1);
    for (int q = 0; q < kStages; ++q) {
      mbar_init(&bars[kbStFull0 + q], 128);  // one (asynchronous) arrival per gather thread
      mbar_init(&bars[kbStFree0 + q], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bars[kbSFull0 + q], 1);
      mbar_init(&bars[kbPFull0 + q], kKeys);
    }
    mbar_init(&bars[kbDone], 1);
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  const int N = w.total;

  if (warp < 4) {
    // ========================================================= keys: P^T, dS^T, epilogue
    const int k = tid;  // key = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float c2 = g.scale_log2;
    for (int n = 0; n < N && ok; ++n) {
      const int buf = n & 1, st = n % kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kbSFull0 + buf], (n >> 1) & 1, g.err) &&
                                       mbar_wait(&bars[kbStFull0 + st], (n / kStages) & 1, g.err));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[2][32], dv[2][32];
      const uint32_t tS = tmem + lane_off + kKColS + buf * kSub;
      const uint32_t tDP = tmem + lane_off + kKColDP + buf * kSub;
      tmem_ld32(tS, sv[0]);
      tmem_ld32(tS + 32, sv[1]);
      tmem_ld32(tDP, dv[0]);
      tmem_ld32(tDP + 32, dv[1]);
      tmem_wait_ld();
      // own sub-tiles: row r (token tok0 + sub*64 + r) sees key k iff k <= sub*64 + r
      int own_sub = -1;
      if (n >= w.n_rsub) own_sub = (n - w.n_rsub) % w.n_osub_h;
      const int rmin = own_sub >= 0 ? k - own_sub * kSub : 0;  // first visible row
      // an empty row has Q = dO = 0 and LSE = Dp = 0: its P is 1 but dS and P dO vanish
      const float* lse = s_lse + st * kSub;
      const float* dpv = s_dp + st * kSub;
      uint32_t pp[32], pd[32];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const int r = h2 * 32 + x;
          float p0 = ex2(fmaf(__uint_as_float(sv[h2][x]), c2, lse[r] * -kLog2e));
          float p1 = ex2(fmaf(__uint_as_float(sv[h2][x + 1]), c2, lse[r + 1] * -kLog2e));
          if (r < rmin) p0 = 0.f;
          if (r + 1 < rmin) p1 = 0.f;
          const float d0 = p0 * (__uint_as_float(dv[h2][x]) - dpv[r]);
          const float d1 = p1 * (__uint_as_float(dv[h2][x + 1]) - dpv[r + 1]);
          pp[16 * h2 + (x >> 1)] = pack_bf16x2(p0, p1);
          pd[16 * h2 + (x >> 1)] = pack_bf16x2(d0, d1);
        }
      tmem_st32(tS, pp);
      tmem_st32(tS + 32, pd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[kbPFull0 + buf]);
    }
    // ------------------------------------------------------- epilogue: dV, dK rows
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kbDone], 0, g.err));
    if (ok) {
      tc_fence_after();
      const int32_t key = key0 + k;
      const bool live = key < blk_end;
#pragma unroll
      for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
        __nv_bfloat16* dst = (which ? a.dK : a.dV) + ((int64_t)key * g.Hkv + gk) * D;
        const float mul = which ? g.scale : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + kKColDV + which * D + c * 32, o);
          tmem_wait_ld();
          if (live) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              float v[8];
#pragma unroll
              for (int y = 0; y < 8; ++y) v[y] = N > 0 ? __uint_as_float(o[8 * x + y]) * mul : 0.f;
              d4[x] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                 pack_bf16x2(v[6], v[7]));
            }
          }
        }
      }
    }
  } else if (warp < 8) {
    // ========================================================= row gather (128 threads)
    // Thread (r, which) copies row r of Q (which 0) or dO (which 1) of every sub-tile, and
    // that row's LSE or Dp; the copies of kStages sub-tiles are in flight at once, each
    // stage's barrier receiving the thread's arrival when its copies have landed.  The
    // (token, head) row of each slot is looked up two sub-tiles ahead.
    const int p = tid - 128;
    const int r = p >> 1, which = p & 1;
    int own_sub;
    int64_t q_a = N > 0 ? kv_row(g, a.rows, w, gk, 0, r, &own_sub) : -1;
    int64_t q_b = N > 1 ? kv_row(g, a.rows, w, gk, 1, r, &own_sub) : -1;
    for (int n = 0; n < N && ok; ++n) {
      const int st = n % kStages, u = n / kStages;
      const int64_t qrow = q_a;
      q_a = q_b;
      q_b = n + 2 < N ? kv_row(g, a.rows, w, gk, n + 2, r, &own_sub) : -1;
      if (u > 0) ok = mbar_wait(&bars[kbStFree0 + st], (u - 1) & 1, g.err);
      if (!ok) break;
      const __nv_bfloat16* src = (which ? a.dO : a.Q) + (qrow >= 0 ? qrow * D : 0);
      const uint32_t nb = qrow >= 0 ? 16u : 0u;
      const uint32_t dstb = smem_u32(smem + (which ? L::kG0 : L::kQ0) + st * L::kSubT);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) cp_async_16(dstb + sw128_offset(r, c, kSub), src + c * 8, nb);
      const float* sv = (which ? a.Dp : a.LSE) + (qrow >= 0 ? qrow : 0);
      cp_async_4(smem_u32((which ? s_dp : s_lse) + st * kSub + r), sv, qrow >= 0 ? 4u : 0u);
      cp_async_arrive_noinc(&bars[kbStFull0 + st]);
    }
    cp_async_wait_all();  // nothing of this thread is in flight when the CTA ends
  } else {
    // ========================================================= TMA + MMA issuer (warp 8)
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(&bars[kbKVFull], 2 * L::kTile);
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        tma_load_3d(smem + L::kK + hh * kKeys * 128, &tmK, &bars[kbKVFull], hh * 64, gk, key0);
        tma_load_3d(smem + L::kV + hh * kKeys * 128, &tmV, &bars[kbKVFull], hh * 64, gk, key0);
      }
    }
    __syncwarp();
    constexpr uint32_t idS = idesc_bf16(kKeys, kSub, false, false);
    constexpr uint32_t idG = idesc_bf16(kKeys, D, false, true);
    const uint32_t sK = smem_u32(smem + L::kK);
    const uint32_t sV = smem_u32(smem + L::kV);
    const uint32_t sQ0 = smem_u32(smem + L::kQ0);
    const uint32_t sG0 = smem_u32(smem + L::kG0);
    auto issue_s = [&](int n) {  // S^T = K Q_n^T, dP^T = V dO_n^T into TMEM buffer n & 1
      const int st = n % kStages, buf = n & 1;
      const uint32_t qb = sQ0 + st * L::kSubT, gb = sG0 + st * L::kSubT;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t aoff = (kk >> 2) * (kKeys * 128) + (kk & 3) * 32;
        const uint32_t boff = (kk >> 2) * (kSub * 128) + (kk & 3) * 32;
        mma_bf16_ss_warp(tmem + kKColS + buf * kSub, sdesc_sw128(sK + aoff, 16, 1024),
                         sdesc_sw128(qb + boff, 16, 1024), idS, kk > 0 ? 1u : 0u);
        mma_bf16_ss_warp(tmem + kKColDP + buf * kSub, sdesc_sw128(sV + aoff, 16, 1024),
                         sdesc_sw128(gb + boff, 16, 1024), idS, kk > 0 ? 1u : 0u);
      }
      mma_commit_warp(&bars[kbSFull0 + buf]);
    };
    auto issue_acc = [&](int n) {  // dV += P^T dO_n, dK += dS^T Q_n
      const int st = n % kStages, buf = n & 1;
      const uint32_t qb = sQ0 + st * L::kSubT, gb = sG0 + st * L::kSubT;
#pragma unroll
      for (int kk = 0; kk < kSub / 16; ++kk) {
        const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
        mma_bf16_ts_warp(tmem + kKColDV, tmem + kKColS + buf * kSub + kk * 8,
                         sdesc_sw128(gb + kk * 2048, kSub * 128, 1024), idG, acc);
        mma_bf16_ts_warp(tmem + kKColDV + D, tmem + kKColS + buf * kSub + 32 + kk * 8,
                         sdesc_sw128(qb + kk * 2048, kSub * 128, 1024), idG, acc);
      }
      mma_commit_warp(&bars[kbStFree0 + st]);
    };
    // the gathered rows were written by cp.async (generic proxy): fence before the MMAs read them
    ok = mbar_wait_warp(&bars[kbKVFull], 0, g.err);
    if (ok && N > 0) {
      ok = mbar_wait_warp(&bars[kbStFull0], 0, g.err);
      if (ok) {
        fence_proxy_async_smem();
        tc_fence_after();
        issue_s(0);
      }
    }
    for (int n = 0; n < N && ok; ++n) {
      if (n + 1 < N) {
        ok = mbar_wait_warp(&bars[kbStFull0 + ((n + 1) % kStages)], ((n + 1) / kStages) & 1, g.err);
        if (!ok) break;
        fence_proxy_async_smem();
        tc_fence_after();
        issue_s(n + 1);
      }
      ok = mbar_wait_warp(&bars[kbPFull0 + (n & 1)], (n >> 1) & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      issue_acc(n);
    }
    mma_commit_warp(&bars[kbDone]);
    mbar_wait_warp(&bars[kbDone], 0, g.err);
  }

  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_bwd_d(const Geom& g, const BwdArgs& a, const __nv_bfloat16* K, const __nv_bfloat16* V,
                         cudaStream_t st) {
  CUtensorMap tq, tg, tk64, tv64, tk128, tv128;
  cudaError_t e;
  if ((e = make_rows_map(&tq, a.Q, (uint64_t)g.T, g.Hq, D, kQRows)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tg, a.dO, (uint64_t)g.T, g.Hq, D, kQRows)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tk64, K, (uint64_t)g.T, g.Hkv, D, kQBN)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tv64, V, (uint64_t)g.T, g.Hkv, D, kQBN)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tk128, K, (uint64_t)g.T, g.Hkv, D, kKeys)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tv128, V, (uint64_t)g.T, g.Hkv, D, kKeys)) != cudaSuccess) return e;
  // dQ partials of the routed slots
  if (g.k > 1 && g.R > 0) {
    const int smem = QLayout<D>::kAlloc;
    if ((e = cudaFuncSetAttribute(bwd_dq_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    bwd_dq_kernel<D, false><<<(unsigned)past_tiles(g), kQThreads, smem, st>>>(tq, tg, tk64, tv64, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // own block + the partials: final dQ
  {
    const int smem = QLayout<D>::kAlloc;
    if ((e = cudaFuncSetAttribute(bwd_dq_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    const int per_blk = g.bs / kQRows;
    const dim3 grid = a.own_head_pairs
                          ? dim3((unsigned)(g.MB * per_blk), (unsigned)g.num_seqs, (unsigned)(g.Hq / 2))
                          : dim3((unsigned)(g.MB * ((per_blk + 1) / 2)), (unsigned)g.num_seqs, (unsigned)g.Hq);
    bwd_dq_kernel<D, true><<<grid, kQThreads, smem, st>>>(tq, tg, tk64, tv64, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // dK, dV
  {
    const int smem = KVLayout<D>::kAlloc;
    if ((e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    const int64_t nct = (int64_t)g.MB * g.num_seqs * g.Hkv * (g.bs / kKeys);
    bwd_dkdv_kernel<D><<<(unsigned)nct, kKVThreads, smem, st>>>(tk128, tv128, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_attn_bwd(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                            const __nv_bfloat16* O, const float* LSE, const __nv_bfloat16* dO, const int32_t* sel,
                            const Work& w, float* Dp, float* dq_part, __nv_bfloat16* dQ, __nv_bfloat16* dK,
                            __nv_bfloat16* dV, cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  const int64_t rows = (int64_t)g.T * g.Hq;
  const int64_t want = (rows + 7) / 8;
  bwd_prep_kernel<<<(unsigned)(want < 148 * 32 ? want : 148 * 32), 256, 0, st>>>(O, dO, Dp, rows, g.D);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (g.k > 1) {
    e = launch_route(g, sel, w, st);
    if (e != cudaSuccess) return e;
  }
  BwdArgs a{g, Q, dO, LSE, Dp, sel, w.counts, w.tile_off, w.tile_bucket, w.rows, dq_part, dQ, dK, dV,
            (g.G % 2 == 0) ? 1 : 0};
  if (g.D == 64) return launch_bwd_d<64>(g, a, K, V, st);
  return launch_bwd_d<128>(g, a, K, V, st);
}

}  // namespace moba
