// MoBA own-block attention + merge, and the mask-based form, on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA).  (The past blocks are in attn_past.cu.)
//
// Two modes share the body of attn_tc_kernel:
//   own  : a CTA takes two tiles of 128 tokens (two heads, or two consecutive tiles of one
//          head) inside one block.  Each row's past partials are merged FIRST: they become
//          the starting state (m, l, O) of the online softmax, which then runs over the
//          block's keys up to the diagonal (causal mask on the diagonal chunk) and ends with
//          the final O (bf16) and LSE.
//   naive: the mask-based form of the same attention (MoBA README, "Implementation
//          Details": moba_naive builds the block mask and runs masked attention).  Tiles as
//          in own mode, but every causal key of the sequence is scored; a row's keys outside
//          its selected blocks get zero weight.  Dense causal cost: a baseline only.
// (youleyou.com, "Kimi发布MoBA突破性实现无限上下文", section "PyTorch实现关键要点": attention
// runs on the own block and on the selected blocks separately and the results are merged by
// online softmax; zhuoshang.net, "MoBA是什么？…", section "MoBA的技术原理": causal mask inside
// the current block.)
//
// Two 128-row query tiles per CTA.  Per 128-key chunk j of tile t:
//   S_t = Q_t K_j^T   (tcgen05 SS MMA, fp32 in TMEM)
//   softmax of S_t in registers (one thread per row = TMEM lane), P_t (bf16) written back
//   over the first half of S_t's TMEM columns
//   O_t += P_t V_j    (tcgen05 TS MMA, A read from TMEM, fp32 accumulator in TMEM)
// The tensor core works on one tile while the other tile's softmax runs.
// Warp roles: warps 0-3 softmax + epilogue of tile 0, warps 4-7 of tile 1, warp 8 TMA
// producer (K/V chunks, two stages), warp 9 TMEM owner + MMA issuer (the whole warp runs the
// issue loop; one elected lane issues each tcgen05.mma), warps 10-11 register donors.
#include <cudaTypedefs.h>
#include <float.h>

#include "attn_common.cuh"

namespace moba {

namespace {
template <int D>
struct Layout {
  static constexpr int kTile = kRows * D * 2;  // bytes of a [128 x D] bf16 tile
  static constexpr int kQ = 0;                 // two tiles
  static constexpr int kK0 = kQ + 2 * kTile;   // two stages
  static constexpr int kV0 = kK0 + 2 * kTile;  // two stages
  static constexpr int kBar = kV0 + 2 * kTile;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

enum Bar {
  kQFull = 0, kKFull0, kKFull1, kKEmpty0, kKEmpty1, kVFull0, kVFull1, kVEmpty0, kVEmpty1,
  kSFull0, kSFull1, kPFull0, kPFull1, kOFull0, kOFull1, kDone, kNumBars
};

// One tile's row source and causal geometry.
struct TileInfo {
  int32_t q0;  // first token
  int h;       // query head
  int nrows;   // valid rows (0..128)
  int diag;    // index of the diagonal chunk
};

enum Mode : int { kModeOwn = 1, kModeNaive = 2 };

template <int D, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars * 8);
  const Geom& g = a.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr bool kNaive = kMode == kModeNaive;

  // ------------------------------------------------------------- work item
  int gk, s, i_blk = 0, nchunks;
  int32_t key0;
  TileInfo ti[2];
  {
    const int per_blk = g.bs / kRows;
    s = blockIdx.y;
    const int32_t ts = seq_start(g, s), te = seq_end(g, s);
    // Own mode: the tiles of a block run together, so its K/V chunks are shared through L2
    // (the GPU runs under its power cap, and DRAM traffic saved there speeds up the other
    // kernels), and inside a block the longest tiles (the last ones) start first.  Naive
    // mode: the work grows with the block index, so the grid runs backwards.
    const int bx = kNaive ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
    if (a.own_head_pairs) {
      int qt;
      if constexpr (kNaive) {
        i_blk = bx / per_blk;
        qt = bx - i_blk * per_blk;
      } else {
        i_blk = bx / per_blk;
        qt = per_blk - 1 - (bx - i_blk * per_blk);
      }
      const int32_t q0 = ts + i_blk * g.bs + qt * kRows;
      if (q0 >= te) return;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        ti[t].h = 2 * blockIdx.z + t;
        ti[t].q0 = q0;
        ti[t].nrows = min(kRows, te - q0);
        ti[t].diag = qt;
      }
      nchunks = qt + 1;
    } else {
      const int pairs = (per_blk + 1) / 2;
      int qp;
      if constexpr (kNaive) {
        i_blk = bx / pairs;
        qp = bx - i_blk * pairs;
      } else {
        i_blk = bx / pairs;
        qp = pairs - 1 - (bx - i_blk * pairs);
      }
      const int32_t q0 = ts + i_blk * g.bs + 2 * qp * kRows;
      if (q0 >= te) return;
      const int qt1 = 2 * qp + 1;
      const bool has1 = qt1 < per_blk && q0 + kRows < te;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        ti[t].h = blockIdx.z;
        ti[t].q0 = q0 + t * kRows;
        ti[t].nrows = (t == 0 || has1) ? max(0, min(kRows, te - ti[t].q0)) : 0;
        ti[t].diag = 2 * qp + t;
      }
      nchunks = has1 ? qt1 + 1 : 2 * qp + 1;
    }
    gk = ti[0].h / g.G;
    key0 = ts + i_blk * g.bs;
    if constexpr (kNaive) {  // every earlier block's chunks come first
      const int before = i_blk * (g.bs / kBN);
      key0 = ts;
      nchunks += before;
#pragma unroll
      for (int t = 0; t < 2; ++t) ti[t].diag += before;
    }
  }

  // ------------------------------------------------------------- early loads
  // Own mode: each softmax thread reads its row's selection and the LSEs of its past
  // partials before the setup below.  The chosen past blocks fill slots 1..np of the row
  // (the selection's padding is at the end), so partial q of the row has the id
  // (row * (top_k - 1) + q).
  int np = 0;                 // own mode: past partials of this thread's row
  float pmax = -INFINITY;     // own mode: their largest LSE, log2 units
  bool folded = false;        // own mode: the row's partials come folded (one partial in mo/mlse)
  if (!kNaive && warp < 8) {
    const int t = warp >> 2, r = tid & (kRows - 1);
    if (r < ti[t].nrows) {
      const int64_t qrow = (int64_t)(ti[t].q0 + r) * g.Hq + ti[t].h;
      bool run = true;
#pragma unroll
      for (int q = 0; q < kMaxTopK - 1; ++q) {
        const int32_t b = q + 1 < g.k ? __ldg(a.sel + qrow * g.k + q + 1) : -1;
        run = run && b >= 0 && b < i_blk;
        np += run ? 1 : 0;
      }
      if (a.premerged && np >= 2) {
        folded = true;
        np = 1;
        pmax = __ldg(a.mlse + qrow) * kLog2e;
      } else {
        for (int q = 0; q < np; ++q) pmax = fmaxf(pmax, __ldg(a.part_lse + qrow * (g.k - 1) + q) * kLog2e);
      }
    }
  }
  auto load_k = [&](int j) {  // K of chunk j into stage j & 1 (TMA producer)
    const int st = j & 1;
    const int tok = key0 + j * kBN;
    mbar_expect_tx(&bars[kKFull0 + st], L::kTile);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh)
      tma_load_3d(smem + L::kK0 + st * L::kTile + hh * kRows * 128, &tmK, &bars[kKFull0 + st], hh * 64, gk, tok);
  };
  auto load_v = [&](int j) {
    const int st = j & 1;
    const int tok = key0 + j * kBN;
    mbar_expect_tx(&bars[kVFull0 + st], L::kTile);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh)
      tma_load_3d(smem + L::kV0 + st * L::kTile + hh * kRows * 128, &tmV, &bars[kVFull0 + st], hh * 64, gk, tok);
  };

  // ------------------------------------------------------------- setup
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    mbar_init(&bars[kQFull], 1);  // one TMA transaction
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bars[kKFull0 + q], 1);
      mbar_init(&bars[kKEmpty0 + q], 1);
      mbar_init(&bars[kVFull0 + q], 1);
      mbar_init(&bars[kVEmpty0 + q], 1);
      mbar_init(&bars[kSFull0 + q], 1);
      mbar_init(&bars[kPFull0 + q], kRows);
      mbar_init(&bars[kOFull0 + q], 1);
    }
    mbar_init(&bars[kDone], 1);
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  if (warp >= 8) regs_dec<kOtherRegs>(); else regs_inc<kSoftmaxRegs>();

  if (warp < 8) {
    // ========================================================= softmax warpgroups
    const int t = warp >> 2;           // tile
    const int r = tid & (kRows - 1);   // row = TMEM lane
    const TileInfo& T_ = ti[t];
    int64_t qrow = -1;  // this row's (token, head) row of Q, O and LSE
    if (r < T_.nrows) qrow = (int64_t)(T_.q0 + r) * g.Hq + T_.h;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS + t * kBN;
    const uint32_t tP = tS + kColP;
    const uint32_t tO = tmem + lane_off + kColO + t * 128;
    const float c2 = g.scale_log2;
    float m = -INFINITY, l = 0.f;
    {
      // Merge first: the row's past partials (normalised O_q and LSE_q, written by the
      // past-block attention before this kernel runs) become the starting state of the
      // online softmax, in its log2 units: m = max_q LSE_q log2(e), w_q = 2^(LSE_q log2(e) - m),
      // l = sum_q w_q, O = sum_q w_q O_q (the past keys' share of sum_k 2^(s_k c2 - m) v_k).
      // The own block's chunks then continue the same online softmax; the O accumulator is
      // written here, before the first PV MMA (which accumulates onto it).
      const int64_t pbase = qrow >= 0 ? qrow * (g.k - 1) : 0;
      m = pmax;
      const int npmax = __reduce_max_sync(0xffffffffu, np);
      for (int q0 = 0; q0 < npmax || q0 == 0; q0 += 2) {  // warp-uniform: TMEM access is per warp
        uint4 hv[2][D / 8];
        float w[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int q = q0 + h2;
          const bool have = q < np;
          w[h2] = have ? ex2(__ldg(folded ? a.mlse + qrow : a.part_lse + pbase + q) * kLog2e - m) : 0.f;
          const __half* srow = !have ? a.part_o : (folded ? a.mo + qrow * D : a.part_o + (pbase + q) * D);
          const uint4* src = reinterpret_cast<const uint4*>(srow);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) hv[h2][c] = have ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        }
        l += w[0] + w[1];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (q0 > 0) {
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = 0u;
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const __half2* hp = reinterpret_cast<const __half2*>(&hv[h2][c * 4]);
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const float2 f = __half22float2(hp[x]);
              o[2 * x] = __float_as_uint(fmaf(w[h2], f.x, __uint_as_float(o[2 * x])));
              o[2 * x + 1] = __float_as_uint(fmaf(w[h2], f.y, __uint_as_float(o[2 * x + 1])));
            }
          }
          tmem_st32(tO + c * 32, o);
        }
        tmem_wait_st();
      }
    }
    // naive mode: this row's selected blocks (own block in slot 0; -1 pads)
    int32_t rsel[kNaive ? kMaxTopK : 1];
    if constexpr (kNaive) {
#pragma unroll
      for (int q = 0; q < kMaxTopK; ++q) rsel[q] = (qrow >= 0 && q < g.k) ? __ldg(a.sel + qrow * g.k + q) : -1;
    }
    for (int j = 0; j < nchunks && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kSFull0 + t], j & 1, g.err));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
      tmem_wait_ld();
      // scaled-logit row max (log2 units); the causal mask applies to the diagonal chunk only
      // (keys after the diagonal chunk, in the query-tile-pair layout, are all masked)
      bool masked = j >= T_.diag;
      int lim = j == T_.diag ? r + 1 : (masked ? 0 : kBN);
      if constexpr (kNaive) {  // keys of a block the row did not select get zero weight
        const int32_t blk = (j * kBN) / g.bs;
        bool on = false;
#pragma unroll
        for (int q = 0; q < kMaxTopK; ++q) on |= rsel[q] == blk;
        if (!on) lim = 0;
        masked = !__all_sync(0xffffffffu, lim == kBN);
      }
      // eight independent running maxima keep the dependency chain short
      float mv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mv[q] = -INFINITY;
      if (!masked) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int x = 0; x < 32; x += 2)
            mv[(x >> 1) & 7] = max3(mv[(x >> 1) & 7], __uint_as_float(sr[c][x]), __uint_as_float(sr[c][x + 1]));
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (c * 32 + x < lim) mv[x & 7] = fmaxf(mv[x & 7], __uint_as_float(sr[c][x]));
      }
      float mx = fmaxf(fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3])), fmaxf(fmaxf(mv[4], mv[5]), fmaxf(mv[6], mv[7])));
      mx *= c2;
      // running max: rescale the TMEM accumulator only when it grows by more than 2^8
      // (p <= 256 otherwise, harmless in fp32 sums and bf16 P).  At this point the previous
      // PV of this tile has completed: the MMA that produced this S was issued after it.
      if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {  // m may start at -inf
        const float m_new = fmaxf(m, mx);
        // naive mode: a row whose keys so far were all masked has m = m_new = -inf (its O and
        // l are still zero); its factor must not become 2^(-inf + inf)
        const float alpha = (kNaive && m_new == -INFINITY) ? 1.f : ex2(m - m_new);
        l *= alpha;
        m = m_new;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      // p = 2^(s*c2 - m); P (bf16 pairs) overwrites the first 64 S columns (S is in registers).
      // Unmasked chunks work on pairs with f32x2 arithmetic and send a share of the
      // exponentials to the FMA pipe; the diagonal chunk keeps the plain scalar form.
      float rv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) rv[q] = 0.f;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t pk[32];
        if (!masked) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int c = 2 * cc + h2;
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              const int pi = x >> 1;
              float u0, u1, p0, p1;
              fma2(u0, u1, __uint_as_float(sr[c][x]), __uint_as_float(sr[c][x + 1]), c2, c2, -m, -m);
              if (pi % kPolyDen < kPolyNum) {
                exp2_poly2(p0, p1, u0, u1);
              } else {
                p0 = ex2(u0);
                p1 = ex2(u1);
              }
              const int q = 2 * (pi & 3);
              add2(rv[q], rv[q + 1], rv[q], rv[q + 1], p0, p1);
              pk[16 * h2 + pi] = pack_bf16x2(p0, p1);
            }
          }
        } else {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int c = 2 * cc + h2;
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              float p0 = ex2(fmaf(__uint_as_float(sr[c][x]), c2, -m));
              float p1 = ex2(fmaf(__uint_as_float(sr[c][x + 1]), c2, -m));
              if (c * 32 + x >= lim) p0 = 0.f;
              if (c * 32 + x + 1 >= lim) p1 = 0.f;
              rv[x & 7] += p0;
              rv[(x & 7) + 1] += p1;
              pk[16 * h2 + (x >> 1)] = pack_bf16x2(p0, p1);
            }
          }
        }
        tmem_st32(tP + cc * 32, pk);
      }
      const float rs = ((rv[0] + rv[1]) + (rv[2] + rv[3])) + ((rv[4] + rv[5]) + (rv[6] + rv[7]));
      l += rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[kPFull0 + t]);
    }
    // ------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kOFull0 + t], 0, g.err));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const float lse_row = (m + __log2f(l)) * kLn2;
      // The final O row (bf16) and LSE: the past partials were merged in at the start.
      // Each thread stages its own row (rows padded by 16 bytes so the row-per-thread 16-byte
      // writes spread over the banks) and hands it to the TMA engine as one bulk copy.  The
      // copies drain to memory on their own; the thread only waits until the engine has read
      // the staged row.  Tile 0's warps stage in the Q and K buffers (free: the O barrier
      // implies every QK^T MMA completed); tile 1's warps, whose O barrier follows the last
      // MMA of the CTA, continue into the V buffers.
      constexpr int kStgBytes = D * 2 + 16;
      static_assert(8 * 32 * kStgBytes <= L::kBar && 4 * 32 * kStgBytes <= L::kV0, "staging rows");
      uint8_t* srow = smem + L::kQ + (warp * 32 + lane) * kStgBytes;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        uint32_t hv[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float v0 = __uint_as_float(o[x]) * inv_l, v1 = __uint_as_float(o[x + 1]) * inv_l;
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
          hv[x >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
        }
#pragma unroll
        for (int x = 0; x < 16; x += 4)
          *reinterpret_cast<uint4*>(srow + c * 64 + x * 4) = make_uint4(hv[x], hv[x + 1], hv[x + 2], hv[x + 3]);
      }
      if (qrow >= 0) {
        a.LSE[qrow] = lse_row;
        fence_proxy_async_smem();
        bulk_store_s2g(a.O + qrow * D, smem_u32(srow), D * 2);
        bulk_commit();
        bulk_wait_read_all();
      }
    }
  } else if (warp == 8) {
    // ========================================================= TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      {  // both Q tiles: 128 consecutive tokens of one head each
        prefetch_tmap(&tmQ);
        mbar_expect_tx(&bars[kQFull], 2 * L::kTile);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d(smem + L::kQ + t * L::kTile + hh * kRows * 128, &tmQ, &bars[kQFull], hh * 64, ti[t].h,
                        ti[t].q0);
      }
      for (int j = 0; j < nchunks && ok; ++j) {
        const int st = j & 1, u = j >> 1;
        if (u > 0) ok = mbar_wait(&bars[kKEmpty0 + st], (u - 1) & 1, g.err);
        if (!ok) break;
        load_k(j);
        if (u > 0) ok = mbar_wait(&bars[kVEmpty0 + st], (u - 1) & 1, g.err);
        if (!ok) break;
        load_v(j);
      }
    }
  } else if (warp == 9) {
    // ========================================================= MMA issuer (whole warp, one elected lane issues)
    constexpr uint32_t idS = idesc_bf16(kRows, kBN, false, false);
    constexpr uint32_t idO = idesc_bf16(kRows, D, false, true);
    const uint32_t sQ = smem_u32(smem + L::kQ);
    const uint32_t sK0 = smem_u32(smem + L::kK0);
    const uint32_t sV0 = smem_u32(smem + L::kV0);
    auto issue_s = [&](int t, int j) {
      const uint32_t qb = sQ + t * L::kTile, kb = sK0 + (j & 1) * L::kTile;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
        mma_bf16_ss_warp(tmem + kColS + t * kBN, sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                         idS, kk > 0 ? 1u : 0u);
      }
      mma_commit_warp(&bars[kSFull0 + t]);
    };
    auto issue_pv = [&](int t, int j) {
      const uint32_t vb = sV0 + (j & 1) * L::kTile;
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        mma_bf16_ts_warp(tmem + kColO + t * 128, tmem + kColS + t * kBN + kColP + kk * 8,
                         sdesc_sw128(vb + kk * 2048, kRows * 128, 1024), idO, 1u);  // O starts from the merge
    };
    ok = mbar_wait_warp(&bars[kQFull], 0, g.err) && mbar_wait_warp(&bars[kKFull0], 0, g.err);
    if (ok) {
      tc_fence_after();
      issue_s(0, 0);
      issue_s(1, 0);
      mma_commit_warp(&bars[kKEmpty0]);
    }
    for (int j = 0; j < nchunks && ok; ++j) {
      const bool more = j + 1 < nchunks;
      ok = mbar_wait_warp(&bars[kVFull0 + (j & 1)], (j >> 1) & 1, g.err) &&
           mbar_wait_warp(&bars[kPFull0], j & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      issue_pv(0, j);
      if (!more) mma_commit_warp(&bars[kOFull0]);
      if (more) {
        ok = mbar_wait_warp(&bars[kKFull0 + ((j + 1) & 1)], ((j + 1) >> 1) & 1, g.err);
        if (!ok) break;
        tc_fence_after();
        issue_s(0, j + 1);
      }
      ok = mbar_wait_warp(&bars[kPFull1], j & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      issue_pv(1, j);
      mma_commit_warp(&bars[kVEmpty0 + (j & 1)]);
      if (!more) mma_commit_warp(&bars[kOFull1]);
      if (more) {
        issue_s(1, j + 1);
        mma_commit_warp(&bars[kKEmpty0 + ((j + 1) & 1)]);
      }
    }
    mma_commit_warp(&bars[kDone]);
    mbar_wait_warp(&bars[kDone], 0, g.err);
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int kMode>
cudaError_t launch_tc(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                      const int32_t* sel, const Work& w, __nv_bfloat16* O, float* LSE, dim3 grid, int head_pairs,
                      cudaStream_t st, int premerged = 0) {
  CUtensorMap tq, tk, tv;
  cudaError_t e = make_rows_map(&tk, K, (uint64_t)g.T, g.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  e = make_rows_map(&tq, Q, (uint64_t)g.T, g.Hq, D, kRows);
  if (e != cudaSuccess) return e;
  e = make_rows_map(&tv, V, (uint64_t)g.T, g.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  AttnArgs a{g, Q, sel, w.tile_off, w.tile_bucket, w.rows, w.part_o, w.part_lse, O, LSE, head_pairs, premerged,
             w.merged_o, w.merged_lse};
  const int smem = Layout<D>::kAlloc;
  e = cudaFuncSetAttribute(attn_tc_kernel<D, kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // the setmaxnreg split must fit in what the launch reserves, or the increase never returns
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_tc_kernel<D, kMode>);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
  attn_tc_kernel<D, kMode><<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}


}  // namespace

namespace {
// Grid of the own-block and naive modes: tile pairs (two heads of a group, or two
// consecutive tiles of one head) x sequences x head pairs (or heads).
dim3 own_grid(const Geom& g, int* head_pairs) {
  const int per_blk = g.bs / kRows;
  *head_pairs = (g.G % 2 == 0) ? 1 : 0;
  return *head_pairs ? dim3((unsigned)(g.MB * per_blk), (unsigned)g.num_seqs, (unsigned)(g.Hq / 2))
                     : dim3((unsigned)(g.MB * ((per_blk + 1) / 2)), (unsigned)g.num_seqs, (unsigned)g.Hq);
}
}  // namespace

namespace {
// When a row can have more than two past partials, they are folded before the own-block
// kernel runs: one warp per (token, head) row with two or more partials loads all of them
// at once (a lane holds D/32 elements of each, so every partial row is one coalesced read),
// merges them by online softmax (M = max LSE_q, w_q = e^(LSE_q - M), O = sum w_q O_q /
// sum w_q, LSE = M + ln sum w_q) and writes the result to the row's entry of mo / mlse.
// The own-block kernel then merges one partial per row: a single round trip instead of one
// per two partials.  The partials themselves are left as they are.

template <int D>
__global__ void __launch_bounds__(256) premerge_kernel(Geom g, const int32_t* __restrict__ sel,
                                                       const __half* __restrict__ part_o,
                                                       const float* __restrict__ part_lse, __half* __restrict__ mo,
                                                       float* __restrict__ mlse) {
  constexpr int kDL = D / 32;  // elements of a partial row per lane
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)g.T * g.Hq;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int km1 = g.k - 1;
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows; row += nwarps) {
    const int32_t t = (int32_t)(row / g.Hq);
    const int s = find_seq(g, t);
    const int i = (t - seq_start(g, s)) / g.bs;
    const int64_t base = row * km1;
    // One round trip per row: lane q reads slot q's block and LSE, and every lane reads its
    // share of all km1 partial rows at once (in bounds whether or not a slot is used; the
    // unused ones are excluded by a select below, never multiplied in).
    const int32_t b = lane < km1 ? __ldg(sel + row * g.k + 1 + lane) : -1;
    const float lq = lane < km1 ? __ldg(part_lse + base + lane) : -INFINITY;
    uint32_t raw[kMaxTopK - 1][kDL / 2];
#pragma unroll
    for (int q = 0; q < kMaxTopK - 1; ++q) {
      const __half* src = part_o + (base + (q < km1 ? q : 0)) * D + lane * kDL;
      if constexpr (kDL == 4) {
        const uint2 v = q < km1 ? __ldg(reinterpret_cast<const uint2*>(src)) : make_uint2(0u, 0u);
        raw[q][0] = v.x;
        raw[q][1] = v.y;
      } else {
        raw[q][0] = q < km1 ? __ldg(reinterpret_cast<const uint32_t*>(src)) : 0u;
      }
    }
    // the chosen past blocks fill the first np slots
    const uint32_t bad = __ballot_sync(0xffffffffu, !(b >= 0 && b < i));
    const int np = min(km1, __ffs(bad) - 1);
    if (np < 2) continue;  // the own-block kernel reads a lone partial where it is
    float M = lane < np ? lq : -INFINITY;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float wl = lane < np ? __expf(lq - M) : 0.f;
    float L = wl;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float acc[kDL];
#pragma unroll
    for (int x = 0; x < kDL; ++x) acc[x] = 0.f;
#pragma unroll
    for (int q = 0; q < kMaxTopK - 1; ++q) {
      const float w = __shfl_sync(0xffffffffu, wl, q);
      if (q < np) {
#pragma unroll
        for (int x = 0; x < kDL / 2; ++x) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&raw[q][x]));
          acc[2 * x] = fmaf(w, f.x, acc[2 * x]);
          acc[2 * x + 1] = fmaf(w, f.y, acc[2 * x + 1]);
        }
      }
    }
    const float inv = 1.f / L;
    __half2* dst = reinterpret_cast<__half2*>(mo + row * D + lane * kDL);
#pragma unroll
    for (int x = 0; x < kDL / 2; ++x) dst[x] = __floats2half2_rn(acc[2 * x] * inv, acc[2 * x + 1] * inv);
    if (lane == 0) mlse[row] = M + __logf(L);
  }
}
}  // namespace

cudaError_t launch_attn_self(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const int32_t* sel, const Work& w,
                             __nv_bfloat16* O, float* LSE, cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  const int head_pairs = (g.G % 2 == 0) ? 1 : 0;
  int premerged = 0;
  if (premerge_used(g)) {
    const int64_t rows = (int64_t)g.T * g.Hq;
    const int64_t want = (rows + 7) / 8;
    const unsigned blocks = (unsigned)(want < 148 * 64 ? want : 148 * 64);
    if (g.D == 64) premerge_kernel<64><<<blocks, 256, 0, st>>>(g, sel, w.part_o, w.part_lse, w.merged_o, w.merged_lse);
    else premerge_kernel<128><<<blocks, 256, 0, st>>>(g, sel, w.part_o, w.part_lse, w.merged_o, w.merged_lse);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    premerged = 1;
  }
  int hp = 0;
  const dim3 grid = own_grid(g, &hp);
  if (g.D == 64) return launch_tc<64, kModeOwn>(g, Q, K, V, sel, w, O, LSE, grid, head_pairs, st, premerged);
  return launch_tc<128, kModeOwn>(g, Q, K, V, sel, w, O, LSE, grid, head_pairs, st, premerged);
}

cudaError_t launch_attn_naive(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                              const __nv_bfloat16* V, const int32_t* sel, __nv_bfloat16* O, float* LSE,
                              cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  int head_pairs = 0;
  const dim3 grid = own_grid(g, &head_pairs);
  Work w{};
  if (g.D == 64) return launch_tc<64, kModeNaive>(g, Q, K, V, sel, w, O, LSE, grid, head_pairs, st);
  return launch_tc<128, kModeNaive>(g, Q, K, V, sel, w, O, LSE, grid, head_pairs, st);
}

int launches_per_forward(const Geom& g) {
  // pool + gate (Kbar split, scores/top-k) + (route count, scan, scatter + past attention
  // when top_k > 1) + (partial pre-merge when a row can have more than two partials) +
  // own block/merge
  return 3 + (g.k > 1 ? 4 : 0) + (premerge_used(g) ? 1 : 0) + 1;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}
}  // namespace

// A [rows, heads, D] bf16 tensor viewed as dims (d, head, row); boxes of 64 d x 1 head x
// box_rows rows with the 128-byte swizzle, i.e. the canonical 128-byte-swizzled atoms of the
// MMA operands (K-major for Q, K, Kbar; MN-major for V).  Out-of-range rows read as zeros.
cudaError_t make_rows_map(CUtensorMap* m, const void* base, uint64_t rows, int heads, int D, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace moba
